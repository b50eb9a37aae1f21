// fa_prefill_common.cuh -- device pieces of the prefill kernel (fa_prefill_sm100.cu): kernel
// parameters, bounded waits, the varlen work-unit finder, rows without keys, the row max, the
// exponential/row-sum/pack step of the softmax, the output row writer, TMA map creation.
#pragma once
#include <cudaTypedefs.h>

#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P and O may grow by up to 2^8
constexpr uint64_t kDrainLimitNs = 200000000ull;
constexpr int kEmuEvery = 8;  // of every kEmuEvery column pairs, kEmu take the FMA-pipe polynomial

struct FwdParams {
  void* o;
  float* lse;
  const int* cu;
  int* status;
  int B, H, Nq, Nk;
  int num_units;  // dense: work units (groups of Q tiles) per (batch, head)
  float scale_log2;
  int causal;
  int prefix;  // causal only: keys [0, prefix) of a sequence are visible to all its queries
  int head_group;  // dense: heads whose work units are ordered together, longest first
  int tma_out;     // 16-bit O: full tiles are written through shared memory by a TMA store
};

// Bounded wait used only on the abort path: ignores the abort flag, has its own limit.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_addr(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > kDrainLimitNs) return;
  }
}

// Wait by every lane of a warp; true only if all lanes saw the phase complete.  (Polling by one
// lane with a broadcast was measured slower in the prefill.)
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Varlen: map a linear slot to (sequence, unit of kUnitRows query rows) by a warp-wide scan of
// per-sequence unit counts.  Within a sequence the last unit (the one with the most causal key
// blocks) comes first.  Invalid cu_seqlens are reported through the status word.
template <int kUnitRows>
__device__ void find_varlen_unit(const FwdParams& p, int slot, int lane, int& out_b, int& out_unit) {
  const int total = p.Nq;
  int base = 0, fb = -1, fm = -1;
  bool bad = false;
  for (int c = 0; c < p.B; c += 32) {
    const int bb = c + lane;
    int len = 0;
    if (bb < p.B) {
      const int lo = p.cu[bb], hi = p.cu[bb + 1];
      if (lo < 0 || hi < lo || hi > total) bad = true;
      else len = hi - lo;
    }
    const int nt = (len + kUnitRows - 1) / kUnitRows;
    int incl = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const int excl = incl - nt;
    const bool mine = nt > 0 && slot >= base + excl && slot < base + incl;
    const unsigned bal = __ballot_sync(0xffffffffu, mine);
    if (bal != 0u) {
      const int src = __ffs(bal) - 1;
      fb = c + src;
      fm = base + __shfl_sync(0xffffffffu, incl, src) - 1 - slot;
      break;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(p.status, kStatusCuSeqlens);
  out_b = fb;
  out_unit = fm;
}

// Elements of the O and LSE buffers (the bounds of the debug build's index checks).
template <int D>
__device__ __forceinline__ long long o_elems(const FwdParams& p) {
  return static_cast<long long>(p.cu == nullptr ? p.B : 1) * p.Nq * p.H * D;
}
__device__ __forceinline__ long long lse_elems(const FwdParams& p) {
  return static_cast<long long>(p.cu == nullptr ? p.B : 1) * p.H * p.Nq;
}

// Index of a row's LSE: [B, H, Nq] dense, [H, total] packed varlen.
__device__ __forceinline__ size_t lse_index(const FwdParams& p, int b, int h, int q_row0, int qi) {
  return (p.cu == nullptr) ? (static_cast<size_t>(b) * p.H + h) * p.Nq + qi
                           : static_cast<size_t>(h) * p.Nq + q_row0 + qi;
}

// O and LSE of a row that sees no key at all.
template <int D, bool kOutF32>
__device__ void write_empty_row(const FwdParams& p, int b, int h, int q_row0, int qi) {
  const size_t orow = (static_cast<size_t>(q_row0 + qi) * p.H + h) * D;
  const size_t li0 = lse_index(p, b, h, q_row0, qi);
  if (!idx_ok(p.status, orow, D, o_elems<D>(p)) || !idx_ok(p.status, li0, 1, lse_elems(p))) return;
  if constexpr (kOutF32) {
    float4* out = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow);
    for (int d = 0; d < D / 4; ++d) out[d] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    uint4* out = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + orow);
    for (int d = 0; d < D / 8; ++d) out[d] = make_uint4(0, 0, 0, 0);
  }
  p.lse[li0] = -INFINITY;
}

// P for 32 score columns (chunk ch of the row): x = s * scale * log2(e) - m, p = 2^x (on the MUFU
// unit, or -- for kEmu of every kEmuEvery column pairs -- by the FMA-pipe polynomial), row-sum
// accumulation in two packed fp32 chains, and conversion to the input type (two 16-bit values per
// 32-bit word, key order).
template <bool kFp16, int kEmu, int N>
__device__ __forceinline__ void exp_chunk(const uint32_t (&sr)[N], int ch, uint64_t sl2x2, uint64_t negm,
                                          uint64_t& acc0, uint64_t& acc1, uint32_t (&pk)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = ch * 32 + 2 * i;
    const uint64_t x = f2_fma(f2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, negm);
    uint64_t pe;
    if ((i % kEmuEvery) < kEmu) {
      pe = exp2_poly_pair(x);
    } else {
      float x0, x1;
      f2_split(x, x0, x1);
      pe = f2(ex2(x0), ex2(x1));
    }
    if (i & 1) acc1 = f2_add(acc1, pe);
    else acc0 = f2_add(acc0, pe);
    float p0, p1;
    f2_split(pe, p0, p1);
    pk[i] = pack2<kFp16>(p0, p1);
  }
}

// Row max of N raw scores: independent chains of 3-input max, one per 32 columns.
template <int N>
__device__ __forceinline__ float row_max(const uint32_t (&sr)[N]) {
  static_assert(N % 32 == 0, "whole 32-column chunks");
  float mxc[N / 32];
#pragma unroll
  for (int k = 0; k < N / 32; ++k) {
    const int b0 = 32 * k;
    float mm = fmax3(__uint_as_float(sr[b0]), __uint_as_float(sr[b0 + 1]), __uint_as_float(sr[b0 + 2]));
#pragma unroll
    for (int i = 3; i < 31; i += 2) mm = fmax3(mm, __uint_as_float(sr[b0 + i]), __uint_as_float(sr[b0 + i + 1]));
    mxc[k] = fmaxf(mm, __uint_as_float(sr[b0 + 31]));
  }
  float mx = mxc[0];
#pragma unroll
  for (int k = 1; k < N / 32; ++k) mx = fmaxf(mx, mxc[k]);
  return mx;
}

// Writes O / l (and LSE = (m + log2 l) ln 2) of one row from its fp32 accumulator in TMEM; rows
// without any visible key get O = 0, LSE = -inf.
template <int D, bool kFp16, bool kOutF32>
__device__ __forceinline__ void write_row(const FwdParams& p, uint32_t o_taddr, int b, int h, int q_row0, int qi,
                                          bool store, float m_run, float l_run) {
  const bool empty = (m_run == -INFINITY);
  const float inv_l = empty ? 0.f : 1.f / l_run;
  const size_t orow = (static_cast<size_t>(q_row0 + qi) * p.H + h) * D;
#ifdef FA_DEBUG
  if (store) store = idx_ok(p.status, orow, D, o_elems<D>(p)) && idx_ok(p.status, lse_index(p, b, h, q_row0, qi), 1, lse_elems(p));
#endif
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t orr[32];
    tmem_ld32_sync(o_taddr + ch * 32, orr);
    if (store) {
      if constexpr (kOutF32) {
        float4* out = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow + ch * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i)
          out[i] = make_float4(__uint_as_float(orr[4 * i]) * inv_l, __uint_as_float(orr[4 * i + 1]) * inv_l,
                               __uint_as_float(orr[4 * i + 2]) * inv_l, __uint_as_float(orr[4 * i + 3]) * inv_l);
      } else {
        uint4* out = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + orow + ch * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float* f = reinterpret_cast<const float*>(orr + 8 * i);
          out[i] = make_uint4(pack2<kFp16>(f[0] * inv_l, f[1] * inv_l), pack2<kFp16>(f[2] * inv_l, f[3] * inv_l),
                              pack2<kFp16>(f[4] * inv_l, f[5] * inv_l), pack2<kFp16>(f[6] * inv_l, f[7] * inv_l));
        }
      }
    }
  }
  if (store) p.lse[lse_index(p, b, h, q_row0, qi)] = empty ? -INFINITY : (m_run + lg2(l_run)) * kLn2;
}

// Normalises one row of O (O / l, from its fp32 accumulator in TMEM) into a 16-bit tile in shared
// memory laid out as the TMA tile box reads and writes it: 64-column panels of 128-byte rows, the
// 16-byte chunks of row r XOR-ed with r mod 8 (128-byte swizzle).
template <int D, bool kFp16>
__device__ __forceinline__ void stage_row(uint32_t o_taddr, uint8_t* tile, int r, float m_run, float l_run) {
  const bool empty = (m_run == -INFINITY);
  const float inv_l = empty ? 0.f : 1.f / l_run;
  const uint32_t base = smem_addr(tile) + r * 128;
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    uint32_t orr[32];
    tmem_ld32_sync(o_taddr + ch * 32, orr);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float* f = reinterpret_cast<const float*>(orr + 8 * i);
      const int col = ch * 32 + 8 * i;  // first of 8 output columns = one 16-byte chunk
      const uint32_t addr = base + (col >> 6) * (128 * 128) + ((((col & 63) >> 3) ^ (r & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                   "r"(pack2<kFp16>(f[0] * inv_l, f[1] * inv_l)), "r"(pack2<kFp16>(f[2] * inv_l, f[3] * inv_l)),
                   "r"(pack2<kFp16>(f[4] * inv_l, f[5] * inv_l)), "r"(pack2<kFp16>(f[6] * inv_l, f[7] * inv_l))
                   : "memory");
    }
  }
}

// 3-D TMA map over a [rows, H, D] 16-bit tensor: box = 64 columns x 1 head x box_rows rows, 128-byte
// swizzle.
bool make_tma_map(CUtensorMap* map, const void* base, int rows, int H, int D, bool fp16, int box_rows);

}  // namespace fa
