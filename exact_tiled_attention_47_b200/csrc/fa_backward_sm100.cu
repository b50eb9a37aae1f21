// fa_backward_sm100.cu -- gradients of exact attention on B200 tensor cores (tcgen05 + TMEM + TMA).
//
// "轻松读懂FlashAttention 上", end of section "Softmax求解重构": the forward pass keeps O and the
// softmax statistics so that the backward pass can recompute S and P instead of reading them back.
// With the natural-log LSE of the forward pass, P = 2^(S*scale*log2(e) - LSE*log2(e)) needs no
// running max.  For an upstream gradient dO of L = sum(dO * O) (the derivative of the forward
// definition):  dV = P^T dO,  dP = dO V^T,  dS = P * (dP - Drow) with Drow_i = sum_d dO_id O_id,
// dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three kernels, no atomics:
//   bwd_rowterm_kernel  Drow[b,h,i] (fp32), one thread per (b, i, h) row.
//   bwd_dq_kernel       CTA = one 128-row query tile.  Per key block j: S = Q K_j^T and
//                       dP = dO V_j^T into TMEM, the four compute warps (thread = query row) form dS
//                       32 columns at a time and write it (bf16/fp16) over the first 64 columns of
//                       dP, then dQ += dS K_j accumulates in TMEM.  dQ * scale is written at the end.
//   bwd_dkdv_kernel     CTA = one 128-row key tile.  Per query block i: S^T = K Q_i^T and
//                       dP^T = V dO_i^T into TMEM, the compute warps (thread = key row) form P^T and
//                       dS^T 32 query columns at a time (the block's LSE and Drow come through shared
//                       memory) and write them over S^T and dP^T, then dV += P^T dO_i and
//                       dK += dS^T Q_i accumulate in TMEM.  dV and dK * scale are written at the end.
// Both recompute S and dP (two more GEMMs than the minimum) so that each gradient is owned by one
// CTA and accumulates in TMEM.  Each streamed 128-row block is processed as two 64-column halves that
// form two independent pipelines: warps 0-3 compute half 0 and warps 4-7 half 1 (the same TMEM lanes,
// different columns), warp 8 is the TMA producer, and warp 9 owns TMEM and issues every tcgen05.mma
// from one thread.  For each half it issues S and dP (N = 64), waits for that half's P/dS, issues the
// half's gradient products (K = 64) and at once the next block's S and dP of the same half, so the
// tensor core works on one half while the other half's softmax-derivative runs (the tensor core runs
// one thread's MMAs in order, which orders each half's next S/dP after the products that read its
// P/dS columns).  The MMA forms are those of the forward kernel: SS with both operands K-major (S, dP)
// and TS with the A operand in TMEM and an N-major B in shared memory (dQ, dV, dK).  Causal runs skip
// fully masked blocks; masking is applied on the blocks that cross the diagonal and at the sequence
// ends.  The masks and layouts are those of the forward kernel: causal (bottom-right aligned), the
// prefix-LM mask (keys [0, prefix) visible to every query of the sequence) and packed varlen
// sequences indexed through cu_seqlens (LSE and Drow [H, total]).
#include <cudaTypedefs.h>

#include <algorithm>

#include "fa_prefill_common.cuh"

namespace fa {
namespace {

constexpr int kBT = 128;  // rows per tile (queries or keys)
constexpr int kHalf = 64;  // columns of a half block
// Column groups per half block: the half's 64 columns are split between kCG warps on each quarter of
// the TMEM lanes (the elementwise work needs no exchange between them: P comes from the stored LSE).
// Two groups (16 compute warps, 88-92 registers) gave the same gradients bit for bit but were 3-4 %
// slower than one at both head dims, so one is the default.
#ifndef FA_BWD_CG
#define FA_BWD_CG 1
#endif
constexpr int kCG = FA_BWD_CG;
static_assert(kCG == 1 || kCG == 2 || kCG == 4, "column groups: 1, 2 or 4");
constexpr int kChunksPerGroup = 4 / kCG;  // 16-column chunks per warp and block half
constexpr int kComputeWarps = 8 * kCG;
constexpr int kThreads = (kComputeWarps + 2) * 32;
constexpr int kProducerWarp = kComputeWarps;
constexpr int kMmaWarp = kComputeWarps + 1;
// Where chunk c (16 columns) of a half keeps its packed 16-bit P or dS: inside the columns its own
// column group has already read, so no group overwrites values another group has yet to load.
__host__ __device__ constexpr uint32_t packed_col(int c) {
  return static_cast<uint32_t>(16 * kChunksPerGroup * (c / kChunksPerGroup) + 8 * (c % kChunksPerGroup));
}
constexpr uint32_t kTmemCols = 512;
constexpr int kPanelBytes = kBT * 64 * 2;  // one 64-column (128-byte) swizzle panel of a tile
constexpr int kMaxStages = 3;  // streamed-tile stages: 3 at D = 64, 2 at D = 128 (shared memory)
constexpr uint32_t kColS = 0, kColDP = 128, kColA = 256;  // S (P over it), dP (dS over it), accumulators

template <int D>
struct BwdCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kBT * D * 2;
  static constexpr int kSt = (D == 64) ? 3 : 2;
  static constexpr int kUsed = (2 + 2 * kSt) * kTileBytes + 2 * kSt * kBT * 4 + 256 + 1024;
  // at least 120 KB so that one CTA (which takes all 512 TMEM columns) runs per SM
  static constexpr int kSmemBytes = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
};
static_assert(BwdCfg<128>::kSmemBytes <= 232448, "shared memory budget");

struct BwdParams {
  const float* lse;   // [B, H, Nq]
  const float* drow;  // [B, H, Nq]
  void* g0;           // dq (dq kernel) or dk (dkdv kernel)
  void* g1;           // dv (dkdv kernel)
  long long g0_n, g1_n;  // elements of g0 and g1 (bounds of the debug index checks)
  int* status;
  const int* cu;  // packed varlen: int32[B + 1] sequence starts (nullptr: dense [B, N, H, D])
  int B, H, Nq, Nk;  // varlen: Nq = Nk = total packed rows
  int num_tiles;  // dense: query tiles (dq) or key tiles (dkdv) per (b, h); varlen: slots per head
  float scale, scale_log2;
  int causal;
  int prefix;  // causal only: keys [0, prefix) of a sequence are visible to all of its queries
  int head_group;  // dense: (b, h) heads whose tiles are ordered together, most work first
};

// The CTA's (batch item, head, 128-row tile) and its sequence: rows [row0, row0 + L) of the packed
// query / key tensors; head-major order.  Dense: tiles of one (b, h) are consecutive, the tile with
// the most causal work first (dq: the last query tile; dk/dv: the first key tile).  Varlen: slots of
// one head are consecutive, sequences in order, tiles found by a warp-wide scan of cu_seqlens; spare
// slots get b = -1.
struct BwdUnit {
  int b, h, tile;
  int q_row0, k_row0, Lq, Lk;
};

template <bool kLastFirst>
__device__ __forceinline__ BwdUnit bwd_unit(const BwdParams& p, int warp, int lane, int* sh_b, int* sh_t) {
  BwdUnit u;
  if (p.cu == nullptr) {
    // groups of head_group heads (their streamed tiles fit in L2) one after another; inside a group
    // the tiles with the most causal work of all its heads first, heads fastest
    const int bhs = p.B * p.H;
    const int per_group = p.head_group * p.num_tiles;
    const int grp = static_cast<int>(blockIdx.x / per_group), w = static_cast<int>(blockIdx.x % per_group);
    const int gsz = min(p.head_group, bhs - grp * p.head_group);
    const int bh = grp * p.head_group + w % gsz;
    const int t = w / gsz;
    u.tile = kLastFirst ? p.num_tiles - 1 - t : t;
    u.b = bh / p.H;
    u.h = bh % p.H;
    u.q_row0 = u.b * p.Nq;
    u.k_row0 = u.b * p.Nk;
    u.Lq = p.Nq;
    u.Lk = p.Nk;
    return u;
  }
  u.h = static_cast<int>(blockIdx.x / p.num_tiles);
  const int slot = static_cast<int>(blockIdx.x % p.num_tiles);
  if (warp == 0) {
    FwdParams f{};  // the unit finder reads cu, B, Nq and status
    f.cu = p.cu;
    f.B = p.B;
    f.Nq = p.Nq;
    f.status = p.status;
    int fb, fm;
    find_varlen_unit<kBT>(f, slot, lane, fb, fm);  // fm counts the sequence's tiles from its last
    if (lane == 0) {
      *sh_b = fb;
      *sh_t = fm;
    }
  }
  __syncthreads();
  u.b = *sh_b;
  u.tile = *sh_t;
  if (u.b < 0) return u;
  u.q_row0 = u.k_row0 = p.cu[u.b];
  u.Lq = u.Lk = p.cu[u.b + 1] - p.cu[u.b];
  if (!kLastFirst) u.tile = (u.Lq + kBT - 1) / kBT - 1 - u.tile;
  return u;
}

struct BwdBars {
  uint64_t fixed_full;                           // the CTA's own tiles (Q + dO, or K + V)
  uint64_t st_full[kMaxStages], st_empty[kMaxStages];  // streamed tiles (K + V, or Q + dO)
  uint64_t stat_full[kMaxStages];                      // dK/dV: the streamed block's LSE and Drow in shared memory
  uint64_t s_full[2], p_full[2];                 // per half block
  uint64_t o_done, drain;
  uint32_t tmem_base;
  int abort_flag;
  int unit_b, unit_t;
};
static_assert(sizeof(BwdBars) <= 256, "barrier block too large");

// ------------------------------------------------------------------------------------------------
// Drow = sum_d dO * O per row

template <bool kFp16, int D>
__global__ void __launch_bounds__(256) bwd_rowterm_kernel(const void* o, const void* dout, float* drow, int B,
                                                          int H, int N, int* status) {
  const long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;  // (b, i, h) row
  const long long rows = static_cast<long long>(B) * N * H;
  if (r >= rows) return;
  if (!idx_ok(status, r * D, D, rows * D)) return;
  const uint4* a = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(o) + r * D);
  const uint4* g = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(dout) + r * D);
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 x = a[c], y = g[c];
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 xf = unpack2<kFp16>(xs[e]), yf = unpack2<kFp16>(ys[e]);
      acc = fmaf(xf.x, yf.x, fmaf(xf.y, yf.y, acc));
    }
  }
  const int h = static_cast<int>(r % H);
  const long long bi = r / H;
  const int i = static_cast<int>(bi % N);
  const int b = static_cast<int>(bi / N);
  const size_t di = (static_cast<size_t>(b) * H + h) * N + i;
  if (idx_ok(status, di, 1, rows)) drow[di] = acc;
}

// ------------------------------------------------------------------------------------------------
// shared pieces

// Load of 16 TMEM columns without the wait: the registers are defined only after tmem_wait_ld_pair,
// which names them as read-write operands so that no use can be scheduled between load and wait.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : FA_R8(0), FA_R8(8)
      : "r"(taddr)
      : "memory");
}

#define FA_RW8(a, i) "+r"(a[i + 0]), "+r"(a[i + 1]), "+r"(a[i + 2]), "+r"(a[i + 3]), "+r"(a[i + 4]), \
                     "+r"(a[i + 5]), "+r"(a[i + 6]), "+r"(a[i + 7])
__device__ __forceinline__ void tmem_wait_ld_pair(uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : FA_RW8(a, 0), FA_RW8(a, 8), FA_RW8(b, 0), FA_RW8(b, 8)
               :
               : "memory");
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
               FA_W8(0)
               : "memory");
}

// The MMA thread issues every product of the CTA, and at N = 64 an MMA takes about 64 cycles of
// issue (twice its tensor work), so the per-MMA instruction count matters: every shared-memory
// descriptor is derived from one built once per tile buffer by adding a constant offset (its start
// address field, bits 0-13 in 16-byte units, cannot carry: shared memory ends below 2^18 bytes).
__device__ __forceinline__ uint64_t desc_kmajor(const void* tile) { return smem_desc_sw128(smem_addr(tile), 16, 1024); }
__device__ __forceinline__ uint64_t desc_nmajor(const void* tile) {
  return smem_desc_sw128(smem_addr(tile), kPanelBytes, 1024);
}
// offset (16-byte units) of K step kk in a K-major tile: 16-element steps advance 32 bytes inside a
// 128-byte row; every 4 steps move to the next 64-column panel
__host__ __device__ constexpr uint32_t kstep_off(int kk) {
  return static_cast<uint32_t>(((kk >> 2) * kPanelBytes + (kk & 3) * 32) >> 4);
}

// Two independent products d0 = a0 b0^T and d1 = a1 b1^T (both operands K-major in shared memory,
// K = D) with their K steps interleaved.
template <int D>
__device__ __forceinline__ void mma_kk2(uint32_t d0, uint64_t a0, uint64_t b0, uint32_t d1, uint64_t a1, uint64_t b1,
                                        uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    mma_ss(d0, a0 + kstep_off(kk), b0 + kstep_off(kk), idesc, kk > 0 ? 1u : 0u);
    mma_ss(d1, a1 + kstep_off(kk), b1 + kstep_off(kk), idesc, kk > 0 ? 1u : 0u);
  }
}

// d += A (TMEM, 128 x 64 packed 16-bit, chunk kk at packed_col(kk)) * B (shared, N-major: the 64 rows
// of a half block, b the descriptor of its first row); 16 rows = two 8-row swizzle atoms = 2048 bytes
__device__ __forceinline__ void mma_tn_half(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                            bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < kHalf / 16; ++kk)
    mma_ts(d_tmem, a_tmem + packed_col(kk), b + ((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
}

// Two independent TS products with their K steps interleaved.
__device__ __forceinline__ void mma_tn_half2(uint32_t d0, uint32_t a0, uint64_t b0, uint32_t d1, uint32_t a1,
                                             uint64_t b1, uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < kHalf / 16; ++kk) {
    mma_ts(d0, a0 + packed_col(kk), b0 + ((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
    mma_ts(d1, a1 + packed_col(kk), b1 + ((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// Byte offset of row 64 in a 128-row swizzled tile (rows are 128 bytes in every 64-column panel).
constexpr uint32_t kHalfRowOff = kHalf * 128;

// Every lane of the warp loads (tcgen05.ld is warp-collective); only lanes with store write the row.
// Columns [32 * ch_lo, 32 * ch_hi) of the row.
template <int D, bool kFp16, bool kOutF32>
__device__ __forceinline__ void store_grad_row(void* out, size_t row_elem, uint32_t taddr, float mul, bool store,
                                               int* status, long long out_n, int ch_lo = 0, int ch_hi = D / 32) {
  if (store) store = idx_ok(status, row_elem, D, out_n);
#pragma unroll
  for (int ch = 0; ch < D / 32; ++ch) {
    if (ch < ch_lo || ch >= ch_hi) continue;
    uint32_t r[32];
    tmem_ld32_sync(taddr + ch * 32, r);
    if (!store) continue;
    if constexpr (kOutF32) {
      float4* o4 = reinterpret_cast<float4*>(static_cast<float*>(out) + row_elem + ch * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        o4[i] = make_float4(__uint_as_float(r[4 * i]) * mul, __uint_as_float(r[4 * i + 1]) * mul,
                            __uint_as_float(r[4 * i + 2]) * mul, __uint_as_float(r[4 * i + 3]) * mul);
    } else {
      uint4* o4 = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + row_elem + ch * 32);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float* f = reinterpret_cast<const float*>(r + 8 * i);
        o4[i] = make_uint4(pack2<kFp16>(f[0] * mul, f[1] * mul), pack2<kFp16>(f[2] * mul, f[3] * mul),
                           pack2<kFp16>(f[4] * mul, f[5] * mul), pack2<kFp16>(f[6] * mul, f[7] * mul));
      }
    }
  }
}

__device__ __forceinline__ void bwd_setup(BwdBars* bars, int warp) {
  if (threadIdx.x == 0) {
    mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&bars->st_full[s], 1);
      mbar_init(&bars->st_empty[s], 1);
      mbar_init(&bars->stat_full[s], 1);
    }
    for (int hh = 0; hh < 2; ++hh) {
      mbar_init(&bars->s_full[hh], 1);
      mbar_init(&bars->p_full[hh], 4 * kCG);
    }
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

__device__ __forceinline__ void bwd_teardown(BwdBars* bars, int warp, uint32_t tbase) {
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// ------------------------------------------------------------------------------------------------
// dQ: one query tile per CTA, walking the key blocks it sees

template <int D, bool kFp16, bool kOutF32>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                  const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sDO = smem + C::kTileBytes;
  auto sK = [&](int st) { return smem + (2 + st) * C::kTileBytes; };
  auto sV = [&](int st) { return smem + (2 + C::kSt + st) * C::kTileBytes; };
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + (2 + 2 * C::kSt) * C::kTileBytes + 2 * C::kSt * kBT * 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const BwdUnit u = bwd_unit<true>(p, warp, lane, &bars->unit_b, &bars->unit_t);
  if (u.b < 0) return;  // spare varlen slot (uniform across the CTA)
  const int b = u.b, h = u.h;
  const int m0 = u.tile * kBT;
  const int Lq = u.Lq, Lk = u.Lk, diag = Lk - Lq;
  int kv_end = Lk;
#ifndef FA_DEBUG
  if (p.causal) kv_end = min(Lk, max(p.prefix, m0 + kBT + diag));
#endif
  const int n = (m0 < Lq && kv_end > 0) ? (kv_end + kBT - 1) / kBT : 0;
  if (n == 0) {  // no row of the tile sees a key: dQ = 0
    if (warp < 4) {
      const int qi = m0 + warp * 32 + lane;
      if (qi < Lq) {
        const size_t row = (static_cast<size_t>(u.q_row0 + qi) * p.H + h) * D;
        for (int d = 0; d < D && idx_ok(p.status, row, D, p.g0_n); ++d) {
          if constexpr (kOutF32) static_cast<float*>(p.g0)[row + d] = 0.f;
          else static_cast<uint16_t*>(p.g0)[row + d] = 0;
        }
      }
    }
    return;
  }
  bwd_setup(bars, warp);
  const uint32_t tbase = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      const uint64_t keep = l2_policy_evict_last();
      mbar_arrive_expect_tx(&bars->fixed_full, 2 * C::kTileBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn) {
        tma_load_3d(&tm_q, &bars->fixed_full, sQ + pn * kPanelBytes, pn * 64, h, u.q_row0 + m0);
        tma_load_3d(&tm_do, &bars->fixed_full, sDO + pn * kPanelBytes, pn * 64, h, u.q_row0 + m0);
      }
      int issued = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        const int st = j % C::kSt;
        if (!(ok = mbar_wait(&bars->st_empty[st], ((j / C::kSt) & 1) ^ 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(&bars->st_full[st], 2 * C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn) {
          tma_load_3d_hint(&tm_k, &bars->st_full[st], sK(st) + pn * kPanelBytes, pn * 64, h, u.k_row0 + j * kBT, keep);
          tma_load_3d_hint(&tm_v, &bars->st_full[st], sV(st) + pn * kPanelBytes, pn * 64, h, u.k_row0 + j * kBT, keep);
        }
        issued = j + 1;
      }
      if (!ok) {
        drain_wait(&bars->fixed_full, 0);
        for (int j = max(0, issued - C::kSt); j < issued; ++j) drain_wait(&bars->st_full[j % C::kSt], (j / C::kSt) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr int fmt = kFp16 ? 0 : 1;
      constexpr uint32_t idesc_s = instr_desc_f16(kBT, kHalf, fmt, 0);
      constexpr uint32_t idesc_g = instr_desc_f16(kBT, D, fmt, 1);
      const uint64_t d_q = desc_kmajor(sQ), d_do = desc_kmajor(sDO);
      const uint64_t d_k = desc_kmajor(sK(0)), d_v = desc_kmajor(sV(0)), d_kn = desc_nmajor(sK(0));
      // offset (16-byte units) of half hh of stage st's tile from stage 0's
      auto half_off = [&](int st, int hh) { return static_cast<uint64_t>((st * C::kTileBytes + kHalfRowOff * hh) >> 4); };
      // S = Q K_j^T and dP = dO V_j^T of half hh (keys 64 hh .. 64 hh + 63 of block j)
      auto issue_s = [&](int st, int hh) {
        mma_kk2<D>(tbase + kColS + kHalf * hh, d_q, d_k + half_off(st, hh), tbase + kColDP + kHalf * hh, d_do,
                   d_v + half_off(st, hh), idesc_s);
        mma_commit(&bars->s_full[hh]);
      };
      bool ok = mbar_wait(&bars->fixed_full, 0, abort_flag, p.status) &&
                mbar_wait(&bars->st_full[0], 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(0, 1);
      }
      for (int j = 0; ok && j < n; ++j) {
        const int st = j % C::kSt;
        for (int hh = 0; hh < 2; ++hh) {
          if (!(ok = mbar_wait(&bars->p_full[hh], j & 1, abort_flag, p.status))) break;
          tc_fence_after();
          // dQ += dS_hh K_j[hh]
          mma_tn_half(tbase + kColA, tbase + kColDP + kHalf * hh, d_kn + half_off(st, hh), idesc_g, j > 0 || hh > 0);
          if (hh == 1) mma_commit(&bars->st_empty[st]);  // every product reading stage st is issued
          if (j + 1 < n) {
            const int st1 = (j + 1) % C::kSt;
            if (hh == 0 && !(ok = mbar_wait(&bars->st_full[st1], ((j + 1) / C::kSt) & 1, abort_flag, p.status)))
              break;
            tc_fence_after();
            issue_s(st1, hh);
          }
        }
      }
      if (ok) mma_commit(&bars->o_done);
      mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
  } else {
    const int hh = warp / (4 * kCG);          // half of every key block this warp works on
    const int cg = (warp >> 2) % kCG;          // its column group within the half
    const int c_lo = cg * kChunksPerGroup;     // first 16-column chunk of the group
    const int r = (warp & 3) * 32 + lane;
    const int qi = m0 + r;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    // keys [0, row_lim) are visible to this row; tile_lim is the smallest row_lim of the tile
    const int row_lim = p.causal ? min(Lk, max(p.prefix, qi + 1 + diag)) : Lk;
    const int tile_lim = p.causal ? min(Lk, max(p.prefix, m0 + 1 + diag)) : Lk;
    // LSE and Drow: [B, H, Nq] dense, [H, total] varlen
    const size_t stat = (p.cu == nullptr ? (static_cast<size_t>(b) * p.H + h) * p.Nq
                                         : static_cast<size_t>(h) * p.Nq + u.q_row0) + min(qi, Lq - 1);
    const bool stat_in = idx_ok(p.status, stat, 1, static_cast<long long>(p.cu == nullptr ? p.B : 1) * p.H * p.Nq);
    const float lse = stat_in ? p.lse[stat] : -INFINITY;
    // rows without keys (LSE = -inf) and rows past the end get P = 0
    const float lse2 = (qi < Lq && lse != -INFINITY) ? lse * kLog2e : INFINITY;
    const float dr = (qi < Lq && stat_in) ? p.drow[stat] : 0.f;
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!(ok = warp_wait(&bars->s_full[hh], j & 1, abort_flag, p.status))) break;
      tc_fence_after();
      const bool masked = (j + 1) * kBT > tile_lim;
      const int lim = row_lim - j * kBT;
      // the group's key columns of the half in 16-column chunks; chunk c+1 is loaded while chunk c is
      // computed
      const uint32_t cs = lane_base + kColS + kHalf * hh, cd = lane_base + kColDP + kHalf * hh;
      uint32_t sb[2][16], db[2][16];
      tmem_ld16_async(cs + 16 * c_lo, sb[0]);
      tmem_ld16_async(cd + 16 * c_lo, db[0]);
      tmem_wait_ld_pair(sb[0], db[0]);
#pragma unroll
      for (int ci = 0; ci < kChunksPerGroup; ++ci) {
        const int c = c_lo + ci, cur = ci & 1;
        if (ci + 1 < kChunksPerGroup) {
          tmem_ld16_async(cs + 16 * (c + 1), sb[cur ^ 1]);
          tmem_ld16_async(cd + 16 * (c + 1), db[cur ^ 1]);
        }
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c0 = kHalf * hh + 16 * c + 2 * i;  // key column in the block
          float p0 = ex2(fmaf(__uint_as_float(sb[cur][2 * i]), sl2, -lse2));
          float p1 = ex2(fmaf(__uint_as_float(sb[cur][2 * i + 1]), sl2, -lse2));
          if (masked) {
            if (c0 >= lim) p0 = 0.f;
            if (c0 + 1 >= lim) p1 = 0.f;
          }
          pk[i] = pack2<kFp16>(p0 * (__uint_as_float(db[cur][2 * i]) - dr), p1 * (__uint_as_float(db[cur][2 * i + 1]) - dr));
        }
        tmem_st8(cd + packed_col(c), pk);  // dS over dP columns this group has already read
        if (ci + 1 < kChunksPerGroup) tmem_wait_ld_pair(sb[cur ^ 1], db[cur ^ 1]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[hh]);
    }
    if (ok) ok = warp_wait(&bars->o_done, 0, abort_flag, p.status);
    if (ok) {
      tc_fence_after();
      const size_t row = static_cast<size_t>(u.q_row0 + min(qi, Lq - 1)) * p.H + h;
      // the 2 kCG groups of warps on this lane quarter store their shares of the row's 32-column chunks
      const int gi = hh * kCG + cg;
      store_grad_row<D, kFp16, kOutF32>(p.g0, row * D, lane_base + kColA, p.scale, qi < Lq, p.status, p.g0_n,
                                        gi * (D / 32) / (2 * kCG), (gi + 1) * (D / 32) / (2 * kCG));
    }
  }
  bwd_teardown(bars, warp, tbase);
}

// ------------------------------------------------------------------------------------------------
// dK, dV: one key tile per CTA, walking the query blocks that see it

template <int D, bool kFp16, bool kOutF32>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sK = smem;
  uint8_t* sV = smem + C::kTileBytes;
  auto sQ = [&](int st) { return smem + (2 + st) * C::kTileBytes; };
  auto sDO = [&](int st) { return smem + (2 + C::kSt + st) * C::kTileBytes; };
  float* sStat = reinterpret_cast<float*>(smem + (2 + 2 * C::kSt) * C::kTileBytes);  // [stage][lse2 | drow][128]
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + (2 + 2 * C::kSt) * C::kTileBytes + 2 * C::kSt * kBT * 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const BwdUnit u = bwd_unit<false>(p, warp, lane, &bars->unit_b, &bars->unit_t);
  if (u.b < 0) return;  // spare varlen slot (uniform across the CTA)
  const int b = u.b, h = u.h;
  const int n0 = u.tile * kBT;
  const int Lq = u.Lq, Lk = u.Lk, diag = Lk - Lq;
  // query blocks that see any key of this tile: every query if the tile starts inside the prefix,
  // else q >= k - diag for the tile's first key k = n0 (causal)
  bool skip = p.causal && n0 >= p.prefix;
#ifdef FA_DEBUG
  skip = false;  // the debug build walks every query block and lets the mask zero the invisible ones
#endif
  const int i_first = skip ? max(0, n0 - diag) / kBT : 0;
  const int nq_blocks = (Lq + kBT - 1) / kBT;
  const int n = (n0 >= Lk || (skip && n0 - diag > Lq - 1)) ? 0 : nq_blocks - i_first;
  if (n <= 0) {  // no query sees this tile: dK = dV = 0
    if (warp < 4) {
      const int kj = n0 + warp * 32 + lane;
      if (kj < Lk) {
        const size_t row = (static_cast<size_t>(u.k_row0 + kj) * p.H + h) * D;
        for (int d = 0; d < D && idx_ok(p.status, row, D, p.g0_n) && idx_ok(p.status, row, D, p.g1_n); ++d) {
          if constexpr (kOutF32) {
            static_cast<float*>(p.g0)[row + d] = 0.f;
            static_cast<float*>(p.g1)[row + d] = 0.f;
          } else {
            static_cast<uint16_t*>(p.g0)[row + d] = 0;
            static_cast<uint16_t*>(p.g1)[row + d] = 0;
          }
        }
      }
    }
    return;
  }
  bwd_setup(bars, warp);
  const uint32_t tbase = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  if (warp == kProducerWarp) {
    const uint64_t keep = l2_policy_evict_last();
    if (lane == 0) {
      mbar_arrive_expect_tx(&bars->fixed_full, 2 * C::kTileBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn) {
        tma_load_3d(&tm_k, &bars->fixed_full, sK + pn * kPanelBytes, pn * 64, h, u.k_row0 + n0);
        tma_load_3d(&tm_v, &bars->fixed_full, sV + pn * kPanelBytes, pn * 64, h, u.k_row0 + n0);
      }
    }
    int issued = 0;
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      const int i = i_first + jj, st = jj % C::kSt;
      if (!(ok = warp_wait(&bars->st_empty[st], ((jj / C::kSt) & 1) ^ 1, abort_flag, p.status))) break;
      if (lane == 0) {  // the tiles first, so their copies overlap the loads of the row statistics
        mbar_arrive_expect_tx(&bars->st_full[st], 2 * C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn) {
          tma_load_3d_hint(&tm_q, &bars->st_full[st], sQ(st) + pn * kPanelBytes, pn * 64, h, u.q_row0 + i * kBT, keep);
          tma_load_3d_hint(&tm_do, &bars->st_full[st], sDO(st) + pn * kPanelBytes, pn * 64, h, u.q_row0 + i * kBT, keep);
        }
      }
      issued = jj + 1;
      // the block's LSE (log2 units; +inf for rows without keys or past the end, so P = 0) and Drow:
      // all eight loads of a lane are independent and in flight together
      float* stat = sStat + st * 2 * kBT;
      // LSE and Drow: [B, H, Nq] dense, [H, total] varlen
      const size_t base = p.cu == nullptr ? (static_cast<size_t>(b) * p.H + h) * p.Nq
                                          : static_cast<size_t>(h) * p.Nq + u.q_row0;
      const long long stat_n = static_cast<long long>(p.cu == nullptr ? p.B : 1) * p.H * p.Nq;
      float lv[4], dv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qi = i * kBT + lane + 32 * e;
        const bool in = qi < Lq && idx_ok(p.status, base + qi, 1, stat_n);
        lv[e] = in ? p.lse[base + qi] : -INFINITY;
        dv[e] = in ? p.drow[base + qi] : 0.f;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        stat[lane + 32 * e] = (lv[e] != -INFINITY) ? lv[e] * kLog2e : INFINITY;
        stat[kBT + lane + 32 * e] = dv[e];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->stat_full[st]);  // release: orders the warp's stores above
    }
    if (!ok && lane == 0) {
      drain_wait(&bars->fixed_full, 0);
      for (int jj = max(0, issued - C::kSt); jj < issued; ++jj) drain_wait(&bars->st_full[jj % C::kSt], (jj / C::kSt) & 1);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr int fmt = kFp16 ? 0 : 1;
      constexpr uint32_t idesc_s = instr_desc_f16(kBT, kHalf, fmt, 0);
      constexpr uint32_t idesc_g = instr_desc_f16(kBT, D, fmt, 1);
      const uint64_t d_k = desc_kmajor(sK), d_v = desc_kmajor(sV);
      const uint64_t d_q = desc_kmajor(sQ(0)), d_do = desc_kmajor(sDO(0));
      const uint64_t d_qn = desc_nmajor(sQ(0)), d_don = desc_nmajor(sDO(0));
      // offset (16-byte units) of half hh of stage st's tile from stage 0's
      auto half_off = [&](int st, int hh) { return static_cast<uint64_t>((st * C::kTileBytes + kHalfRowOff * hh) >> 4); };
      // S^T = K Q_i^T and dP^T = V dO_i^T of half hh (queries 64 hh .. 64 hh + 63 of block i)
      auto issue_s = [&](int st, int hh) {
        mma_kk2<D>(tbase + kColS + kHalf * hh, d_k, d_q + half_off(st, hh), tbase + kColDP + kHalf * hh, d_v,
                   d_do + half_off(st, hh), idesc_s);
        mma_commit(&bars->s_full[hh]);
      };
      bool ok = mbar_wait(&bars->fixed_full, 0, abort_flag, p.status) &&
                mbar_wait(&bars->st_full[0], 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(0, 1);
      }
      for (int jj = 0; ok && jj < n; ++jj) {
        const int st = jj % C::kSt;
        for (int hh = 0; hh < 2; ++hh) {
          if (!(ok = mbar_wait(&bars->p_full[hh], jj & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const bool acc = jj > 0 || hh > 0;
          // dV += P^T_hh dO_i[hh],  dK += dS^T_hh Q_i[hh]
          mma_tn_half2(tbase + kColA, tbase + kColS + kHalf * hh, d_don + half_off(st, hh), tbase + kColA + D,
                       tbase + kColDP + kHalf * hh, d_qn + half_off(st, hh), idesc_g, acc);
          if (hh == 1) mma_commit(&bars->st_empty[st]);  // every product reading stage st is issued
          if (jj + 1 < n) {
            const int st1 = (jj + 1) % C::kSt;
            if (hh == 0 && !(ok = mbar_wait(&bars->st_full[st1], ((jj + 1) / C::kSt) & 1, abort_flag, p.status)))
              break;
            tc_fence_after();
            issue_s(st1, hh);
          }
        }
      }
      if (ok) mma_commit(&bars->o_done);
      mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
  } else {
    const int hh = warp / (4 * kCG);          // half of every query block this warp works on
    const int cg = (warp >> 2) % kCG;          // its column group within the half
    const int c_lo = cg * kChunksPerGroup;     // first 16-column chunk of the group
    const int r = (warp & 3) * 32 + lane;
    const int kj = n0 + r;  // this thread's key
    const uint32_t lane_base = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      const int i = i_first + jj, st = jj % C::kSt;
      if (!(ok = warp_wait(&bars->s_full[hh], jj & 1, abort_flag, p.status))) break;
      // the stage's LSE/Drow (this stage cannot be refilled before this block's P V products)
      if (!(ok = warp_wait(&bars->stat_full[st], (jj / C::kSt) & 1, abort_flag, p.status))) break;
      tc_fence_after();
      const float* stat = sStat + st * 2 * kBT;
      // key kj is visible to query q iff kj < prefix or q >= kj - diag (causal); the whole block is
      // visible iff its first query already sees the tile's last key; queries past the sequence end
      // have P = 0 through their +inf LSE
      const bool masked = p.causal && (i * kBT + diag < n0 + kBT - 1);
      const int q_lo = (kj < p.prefix) ? -kBT : kj - diag - i * kBT;  // columns c < q_lo are masked
      // the group's query columns of the half in 16-column chunks; chunk c+1 is loaded while chunk c
      // is computed
      const uint32_t cs = lane_base + kColS + kHalf * hh, cd = lane_base + kColDP + kHalf * hh;
      uint32_t sb[2][16], db[2][16];
      tmem_ld16_async(cs + 16 * c_lo, sb[0]);
      tmem_ld16_async(cd + 16 * c_lo, db[0]);
      tmem_wait_ld_pair(sb[0], db[0]);
#pragma unroll
      for (int ci = 0; ci < kChunksPerGroup; ++ci) {
        const int c = c_lo + ci, cur = ci & 1;
        if (ci + 1 < kChunksPerGroup) {
          tmem_ld16_async(cs + 16 * (c + 1), sb[cur ^ 1]);
          tmem_ld16_async(cd + 16 * (c + 1), db[cur ^ 1]);
        }
        uint32_t pk[8], dk[8];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int c0 = kHalf * hh + 16 * c + 4 * q4;  // query column in the block
          const float4 l2 = *reinterpret_cast<const float4*>(stat + c0);
          const float4 dr = *reinterpret_cast<const float4*>(stat + kBT + c0);
          const float lv[4] = {l2.x, l2.y, l2.z, l2.w}, dv[4] = {dr.x, dr.y, dr.z, dr.w};
          float pv[4], dsv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float pe = ex2(fmaf(__uint_as_float(sb[cur][4 * q4 + e]), sl2, -lv[e]));
            if (masked && c0 + e < q_lo) pe = 0.f;
            pv[e] = pe;
            dsv[e] = pe * (__uint_as_float(db[cur][4 * q4 + e]) - dv[e]);
          }
          pk[2 * q4] = pack2<kFp16>(pv[0], pv[1]);
          pk[2 * q4 + 1] = pack2<kFp16>(pv[2], pv[3]);
          dk[2 * q4] = pack2<kFp16>(dsv[0], dsv[1]);
          dk[2 * q4 + 1] = pack2<kFp16>(dsv[2], dsv[3]);
        }
        tmem_st8(cs + packed_col(c), pk);  // P^T over S^T columns this group has already read
        tmem_st8(cd + packed_col(c), dk);  // dS^T over dP^T columns this group has already read
        if (ci + 1 < kChunksPerGroup) tmem_wait_ld_pair(sb[cur ^ 1], db[cur ^ 1]);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full[hh]);
    }
    if (ok) ok = warp_wait(&bars->o_done, 0, abort_flag, p.status);
    if (ok) {
      tc_fence_after();
      const size_t row = (static_cast<size_t>(u.k_row0 + min(kj, Lk - 1)) * p.H + h) * D;
      // warps of half 0 store dV, those of half 1 dK, each column group its share of the 32-column chunks
      const int ch_lo = cg * (D / 32) / kCG, ch_hi = (cg + 1) * (D / 32) / kCG;
      if (hh == 0)
        store_grad_row<D, kFp16, kOutF32>(p.g1, row, lane_base + kColA, 1.f, kj < Lk, p.status, p.g1_n, ch_lo, ch_hi);
      else
        store_grad_row<D, kFp16, kOutF32>(p.g0, row, lane_base + kColA + D, p.scale, kj < Lk, p.status, p.g0_n, ch_lo,
                                          ch_hi);
    }
  }
  bwd_teardown(bars, warp, tbase);
}

template <int D, bool kFp16, bool kOutF32>
int launch_bwd_t(const BackwardArgs& a, const CUtensorMap (&m)[4], BwdParams p, cudaStream_t stream) {
  const int smem = BwdCfg<D>::kSmemBytes;
  const bool varlen = a.cu_seqlens != nullptr;
  const size_t rows = static_cast<size_t>(varlen ? 1 : a.B) * a.Nq * a.H;
  // varlen rows are those of one batch item of Nq = total rows: Drow [H, total]
  bwd_rowterm_kernel<kFp16, D><<<static_cast<unsigned>((rows + 255) / 256), 256, 0, stream>>>(
      a.o, a.dout, a.drow, varlen ? 1 : a.B, a.H, a.Nq, a.status);
  auto kq = bwd_dq_kernel<D, kFp16, kOutF32>;
  auto kkv = bwd_dkdv_kernel<D, kFp16, kOutF32>;
  // the shared-memory opt-in is a per-device (per-context) attribute: raised once
  static PerContext<int> configured;
  int unused = 0;
  const int ce = configured.get(&unused, [&](int*) {
    cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    return static_cast<int>(e);
  });
  if (ce != 0) return ce;
  BwdParams pq = p;
  pq.g0 = a.dq;
  pq.g0_n = static_cast<long long>(varlen ? 1 : a.B) * a.Nq * a.H * D;
  // dense: tiles per (b, h); varlen: slots per head, enough for the sum over the sequences of
  // ceil(len / 128) <= total / 128 + B (spare slots exit at once)
  pq.num_tiles = varlen ? a.Nq / kBT + a.B : (a.Nq + kBT - 1) / kBT;
  kq<<<static_cast<unsigned>(pq.num_tiles * (varlen ? 1 : a.B) * a.H), kThreads, smem, stream>>>(m[0], m[1], m[2], m[3], pq);
  BwdParams pk = p;
  pk.g0 = a.dk;
  pk.g1 = a.dv;
  pk.g0_n = pk.g1_n = static_cast<long long>(varlen ? 1 : a.B) * a.Nk * a.H * D;
  pk.num_tiles = varlen ? a.Nk / kBT + a.B : (a.Nk + kBT - 1) / kBT;
  kkv<<<static_cast<unsigned>(pk.num_tiles * (varlen ? 1 : a.B) * a.H), kThreads, smem, stream>>>(m[0], m[1], m[2], m[3], pk);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_backward(const BackwardArgs& a, cudaStream_t stream) {
  CUtensorMap m[4];
  const int rows_q = a.cu_seqlens != nullptr ? a.Nq : a.B * a.Nq;
  const int rows_k = a.cu_seqlens != nullptr ? a.Nk : a.B * a.Nk;
  if (!make_tma_map(&m[0], a.q, rows_q, a.H, a.D, a.fp16, kBT) ||
      !make_tma_map(&m[1], a.dout, rows_q, a.H, a.D, a.fp16, kBT) ||
      !make_tma_map(&m[2], a.k, rows_k, a.H, a.D, a.fp16, kBT) ||
      !make_tma_map(&m[3], a.v, rows_k, a.H, a.D, a.fp16, kBT))
    return static_cast<int>(cudaErrorInvalidValue);
  BwdParams p;
  p.lse = a.lse;
  p.drow = a.drow;
  p.g0 = p.g1 = nullptr;
  p.g0_n = p.g1_n = 0;
  p.status = a.status;
  p.B = a.B;
  p.H = a.H;
  p.Nq = a.Nq;
  p.Nk = a.Nk;
  p.num_tiles = 0;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal ? 1 : 0;
  p.prefix = a.causal ? a.prefix : 0;
  p.cu = a.cu_seqlens;
  // about 64 MB of streamed tiles (K and V for dQ, Q and dO for dK/dV) per head group
  const long long stream_head = 2LL * std::max(a.Nq, a.Nk) * a.D * 2;
  p.head_group = static_cast<int>(
      std::max(1LL, std::min<long long>(static_cast<long long>(a.B) * a.H, (64LL << 20) / stream_head)));
#ifdef FA_BWD_HEAD_GROUP  // tuning: a fixed head-group size
  p.head_group = FA_BWD_HEAD_GROUP;
#endif
  if (a.D == 64) {
    if (a.fp16) return a.g_fp32 ? launch_bwd_t<64, true, true>(a, m, p, stream) : launch_bwd_t<64, true, false>(a, m, p, stream);
    return a.g_fp32 ? launch_bwd_t<64, false, true>(a, m, p, stream) : launch_bwd_t<64, false, false>(a, m, p, stream);
  }
  if (a.fp16) return a.g_fp32 ? launch_bwd_t<128, true, true>(a, m, p, stream) : launch_bwd_t<128, true, false>(a, m, p, stream);
  return a.g_fp32 ? launch_bwd_t<128, false, true>(a, m, p, stream) : launch_bwd_t<128, false, false>(a, m, p, stream);
}

}  // namespace fa
