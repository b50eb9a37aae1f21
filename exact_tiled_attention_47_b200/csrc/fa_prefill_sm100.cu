// fa_prefill_sm100.cu -- exact tiled attention forward on B200 tensor cores (tcgen05 + TMEM + TMA).
//
// The method (Ascend CANN ops-transformer FlashAttention article, sections "原理" and "代码讲解"):
// cut Q into row blocks and K/V into key blocks; for every Q block walk the K/V blocks, form the
// block scores, keep a running row max m and row sum l, rescale the output accumulator when m grows,
// add P_j V_j, and divide by l at the end.  S and P never leave the chip.
//
// Mapping to sm_100a.  One CTA owns two 128-row Q tiles (256 rows) of one (batch, head), so every
// K/V tile brought into shared memory feeds both, and the tensor core alternates between the tiles
// while the other tile's softmax runs ("ping-pong"):
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1: thread r of a warpgroup owns query
//               row r (TMEM lane r).  Per key block it reads its 128 scores with tcgen05.ld, masks
//               them (causal diagonal / key-length tail only), updates the running max m and sum l,
//               computes P = 2^(S*scale*log2(e) - m) -- part of the exponentials on the MUFU unit,
//               part with a polynomial on the FMA pipe -- writes P (bf16/fp16) to TMEM, and at the end
//               writes O / l and the LSE.  O is rescaled only when m grew by more than 2^8 since the
//               last rescale; until then P and l use the stale max, which is exact because O and l
//               share it.
//   warp 8      TMA producer: Q tiles once, then K_j and V_j through rings of 128-byte-swizzled
//               shared-memory stages tracked by mbarriers.
//   warp 9      owns the tensor memory and issues every tcgen05.mma from one thread, in the order
//               S0(0) S1(0) | PV0(j) S0(j+1) PV1(j) S1(j+1) | ...  The commit that signals S_t(j+1)
//               covers all earlier MMAs, so it also tells softmax t that PV_t(j) is done (its P
//               buffer is free and O_t is stable).
//   warps 10-11 idle.
// TMEM (512 columns): S0 [0,128) S1 [128,256); D=64: O0 [256,320) O1 [320,384) P0 [384,448)
// P1 [448,512); D=128: O0 [256,384) O1 [384,512) and P_t in the upper half of S_t (P is written
// only after the whole S row was read; the next S_t is issued after the PV_t that reads P_t).
// Causal runs stop at the last key block the tile's last row can see; fully masked blocks are never
// loaded or multiplied.  Work units are issued longest first.
#include <cudaTypedefs.h>

#include <mutex>

#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per block
constexpr int kTiles = 2;
constexpr int kThreads = 384;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;  // owns TMEM; issues the MMAs of tile 0 (warp 10 those of tile 1)
constexpr uint32_t kTmemCols = 512;
constexpr int kPanelBytes = kBM * 64 * 2;  // one 64-column (128-byte) swizzle panel of a tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P and O may grow by up to 2^8
constexpr uint64_t kDrainLimitNs = 200000000ull;
// Registers: launched with kLaunchRegs per thread; the two softmax warpgroups then take
// kSoftmaxRegs and the producer/MMA warpgroup gives back down to kControlRegs.  The split must not
// exceed the launch allocation (256 * 216 + 128 * 72 = 384 * 168), else setmaxnreg.inc would wait
// forever; the host refuses to launch if the compiled register count differs from kLaunchRegs.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(256 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kEmuEvery = 8;  // of every kEmuEvery column pairs ...
// ... this many take the polynomial exp2 (the MUFU unit is the tighter limit at D = 64, where the
// MMA work per score is half that of D = 128)
template <int D>
constexpr int emu_pairs() {
#ifdef FA_EMU_PAIRS
  return FA_EMU_PAIRS;
#else
  return D == 64 ? 1 : 1;
#endif
}

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kBM * D * 2;
#ifndef FA_KSTAGES_128
#define FA_KSTAGES_128 2
#endif
#ifndef FA_VSTAGES_128
#define FA_VSTAGES_128 2
#endif
  static constexpr int kKStages = (D == 64) ? 4 : FA_KSTAGES_128;
  static constexpr int kVStages = (D == 64) ? 4 : FA_VSTAGES_128;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTiles * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 384 + 1024;  // barriers + alignment slack
  // With P in its own TMEM columns (D = 64) the next S of a tile is issued as soon as the softmax
  // has read the current one; with P aliased into S (D = 128) it must follow the P*V product.
#ifndef FA_FORCE_LATE_S
#define FA_FORCE_LATE_S 0
#endif
  static constexpr bool kEarlyS = (D == 64) && !FA_FORCE_LATE_S;
  __device__ static constexpr uint32_t col_s(int t) { return t ? 128u : 0u; }
  __device__ static constexpr uint32_t col_o(int t) { return t ? ((D == 64) ? 320u : 384u) : 256u; }
  __device__ static constexpr uint32_t col_p(int t) {
    return t ? ((D == 64) ? 448u : 192u) : ((D == 64) ? 384u : 64u);
  }
};

struct Bars {
  uint64_t q_full[2];
  uint64_t k_full[4], v_full[4];
  uint64_t k_empty[2][4], v_empty[2][4];  // per tile: its MMAs no longer read the stage
  uint64_t s_full[2], s_free[2], p_full[2], o_done[2];
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
  int tile_b, tile_pair;
};
static_assert(sizeof(Bars) <= 384, "barrier block too large");

struct FwdParams {
  void* o;
  float* lse;
  const int* cu;
  int* status;
  int B, H, Nq, Nk;
  int num_pairs;  // dense: ceil(Nq / 256)
  float scale_log2;
  int causal;
};

// Bounded wait used only on the abort path: ignores the abort flag, has its own limit.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_addr(bar);
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (global_timer_ns() - t0 > kDrainLimitNs) return;
  }
}

// Wait by every lane of a warp; true only if all lanes saw the phase complete.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status) {
  const bool ok = mbar_wait(bar, parity, abort_flag, status);
  return __all_sync(0xffffffffu, ok);
}

// Varlen: map a linear slot to (sequence, 256-row pair) by a warp-wide scan of per-sequence counts.
__device__ void find_varlen_pair(const FwdParams& p, int slot, int lane, int& out_b, int& out_pair) {
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
    const int nt = (len + kTiles * kBM - 1) / (kTiles * kBM);
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
      fm = slot - base - __shfl_sync(0xffffffffu, excl, src);
      break;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(p.status, kStatusCuSeqlens);
  out_b = fb;
  out_pair = fm;
}

// O and LSE of rows that see no key at all.
template <int D, bool kOutF32>
__device__ void write_empty_row(const FwdParams& p, int b, int h, int q_row0, int qi) {
  const size_t orow = (static_cast<size_t>(q_row0 + qi) * p.H + h) * D;
  if constexpr (kOutF32) {
    float4* out = reinterpret_cast<float4*>(static_cast<float*>(p.o) + orow);
    for (int d = 0; d < D / 4; ++d) out[d] = make_float4(0.f, 0.f, 0.f, 0.f);
  } else {
    uint4* out = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.o) + orow);
    for (int d = 0; d < D / 8; ++d) out[d] = make_uint4(0, 0, 0, 0);
  }
  const size_t li = (p.cu == nullptr) ? (static_cast<size_t>(b) * p.H + h) * p.Nq + qi
                                      : static_cast<size_t>(h) * p.Nq + q_row0 + qi;
  p.lse[li] = -INFINITY;
}

// P for 32 score columns (chunk ch of the row): x = s * scale * log2(e) - m, p = 2^x (on the MUFU
// unit, or -- for kEmu of every kEmuEvery column pairs when kMixed -- by the FMA-pipe
// polynomial), row-sum accumulation in two packed fp32 chains, conversion to the input type and a
// 16-column TMEM store (two 16-bit values per 32-bit column, the layout the P*V MMA reads).
#ifndef FA_PACKED_MUFU
#define FA_PACKED_MUFU 1
#endif
template <bool kMixed, bool kFp16, int kEmu>
__device__ __forceinline__ void exp_chunk_regs(const uint32_t (&sr)[128], int ch, uint64_t sl2x2, uint64_t negm,
                                               uint64_t& acc0, uint64_t& acc1, uint32_t (&pk)[16]) {
#if !FA_PACKED_MUFU
  float sl2, nm, u;
  f2_split(sl2x2, sl2, u);
  f2_split(negm, nm, u);
  float sa = 0.f, sb = 0.f;
#endif
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = ch * 32 + 2 * i;
    float p0, p1;
    if (kMixed && (i % kEmuEvery) < kEmu) {
      const uint64_t x = f2_fma(f2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, negm);
      const uint64_t pe = exp2_poly_pair(x);
      if (i & 1) acc1 = f2_add(acc1, pe);
      else acc0 = f2_add(acc0, pe);
      f2_split(pe, p0, p1);
    } else {
#if FA_PACKED_MUFU
      const uint64_t x = f2_fma(f2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])), sl2x2, negm);
      float x0, x1;
      f2_split(x, x0, x1);
      const uint64_t pe = f2(ex2(x0), ex2(x1));
      if (i & 1) acc1 = f2_add(acc1, pe);
      else acc0 = f2_add(acc0, pe);
      f2_split(pe, p0, p1);
#else
      p0 = ex2(fmaf(__uint_as_float(sr[c]), sl2, nm));
      p1 = ex2(fmaf(__uint_as_float(sr[c + 1]), sl2, nm));
      sa += p0;
      sb += p1;
#endif
    }
    pk[i] = pack2<kFp16>(p0, p1);
  }
#if !FA_PACKED_MUFU
  acc0 = f2_add(acc0, f2(sa, sb));
#endif
}

template <bool kMixed, bool kFp16, int kEmu>
__device__ __forceinline__ void exp_chunk(const uint32_t (&sr)[128], int ch, uint64_t sl2x2, uint64_t negm,
                                          uint64_t& acc0, uint64_t& acc1, uint32_t p_addr) {
  uint32_t pk[16];
  exp_chunk_regs<kMixed, kFp16, kEmu>(sr, ch, sl2x2, negm, acc0, acc1, pk);
  tmem_st16(p_addr + ch * 16, pk);
}

template <int D, bool kFp16, bool kOutF32>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const FwdParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Bars* bars = reinterpret_cast<Bars*>(smem + C::kBarOff);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work unit: (b, h, pair of Q tiles) -----------------------------------------------------
  int b, h, pair;
  if (p.cu == nullptr) {
    // all pairs of one (b, h) are consecutive, so they run together and share its K/V in L2;
    // within a head the pair with the most key blocks (causal) goes first
    const int bh = static_cast<int>(blockIdx.x / p.num_pairs);
    pair = p.num_pairs - 1 - static_cast<int>(blockIdx.x % p.num_pairs);
    b = bh / p.H;
    h = bh % p.H;
  } else {
    h = blockIdx.x % p.H;
    const int slot = blockIdx.x / p.H;
    if (warp == 0) {
      int fb, fm;
      find_varlen_pair(p, slot, lane, fb, fm);
      if (lane == 0) {
        bars->tile_b = fb;
        bars->tile_pair = fm;
      }
    }
    __syncthreads();
    b = bars->tile_b;
    pair = bars->tile_pair;
    if (b < 0) return;  // spare slot (uniform across the CTA)
  }
  int q_row0, k_row0, Lq, Lk;
  if (p.cu == nullptr) {
    q_row0 = b * p.Nq;
    k_row0 = b * p.Nk;
    Lq = p.Nq;
    Lk = p.Nk;
  } else {
    q_row0 = k_row0 = p.cu[b];
    Lq = Lk = p.cu[b + 1] - p.cu[b];
  }
  const int m0 = pair * (kTiles * kBM);
  const int diag = Lk - Lq;  // bottom-right causal alignment
  // key blocks each tile needs (0: the tile is past the end, or no row of it sees a key)
  auto blocks_of = [&](int t) {
    const int first = m0 + t * kBM;
    int kv_end = Lk;
    if (p.causal) kv_end = min(Lk, first + kBM + diag);
    return (first < Lq && kv_end > 0) ? (kv_end + kBN - 1) / kBN : 0;
  };
  const int n_kv0 = blocks_of(0), n_kv1 = blocks_of(1);
  auto n_kv = [&](int t) { return t ? n_kv1 : n_kv0; };
  const int n_max = max(n_kv0, n_kv1);

  // softmax warps of tiles without any visible key write O = 0, LSE = -inf directly
  if (warp < 8) {
    const int t = warp >> 2;
    if (n_kv(t) == 0) {
      const int qi = m0 + t * kBM + (warp & 3) * 32 + lane;
      if (qi < Lq) write_empty_row<D, kOutF32>(p, b, h, q_row0, qi);
    }
  }
  if (n_max == 0) return;  // uniform

  // ---- setup ----------------------------------------------------------------------------------
  if (threadIdx.x == 0) {
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(&bars->q_full[t], 1);
      mbar_init(&bars->s_full[t], 1);
      mbar_init(&bars->s_free[t], 4);
      mbar_init(&bars->p_full[t], 4);
      mbar_init(&bars->o_done[t], 1);
    }
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[0][s], 1);
      mbar_init(&bars->k_empty[1][s], 1);
    }
    for (int s = 0; s < C::kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[0][s], 1);
      mbar_init(&bars->v_empty[1][s], 1);
    }
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
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
  const uint32_t tbase = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  auto sQ = [&](int t) { return smem + C::kQOff + t * C::kTileBytes; };
  auto sK = [&](int st) { return smem + C::kKOff + st * C::kTileBytes; };
  auto sV = [&](int st) { return smem + C::kVOff + st * C::kTileBytes; };

  if (warp >= 8) {
    regs_decrease<kControlRegs>();
  if (warp == kProducerWarp) {
    // ================================ TMA producer ===============================================
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      const uint64_t keep = l2_policy_evict_last();
      for (int t = 0; t < kTiles; ++t) {
        if (n_kv(t) == 0) continue;
        mbar_arrive_expect_tx(&bars->q_full[t], C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d(&tmap_q, &bars->q_full[t], sQ(t) + pn * kPanelBytes, pn * 64, h, q_row0 + m0 + t * kBM);
      }
      int k_issued = 0, v_issued = 0;  // blocks whose K / V copies were started
      bool ok = true;
      for (int j = 0; j < n_max; ++j) {
        const int ks = j % C::kKStages, vs = j % C::kVStages;
        // the stage's previous block must no longer be read by any tile that used it
        const int jk = j - C::kKStages, jv = j - C::kVStages;
        for (int t = 0; t < kTiles && ok && jk >= 0; ++t)
          if (jk < n_kv(t)) ok = mbar_wait(&bars->k_empty[t][ks], (jk / C::kKStages) & 1, abort_flag, p.status);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars->k_full[ks], C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d_hint(&tmap_k, &bars->k_full[ks], sK(ks) + pn * kPanelBytes, pn * 64, h, k_row0 + j * kBN, keep);
        k_issued = j + 1;
        for (int t = 0; t < kTiles && ok && jv >= 0; ++t)
          if (jv < n_kv(t)) ok = mbar_wait(&bars->v_empty[t][vs], (jv / C::kVStages) & 1, abort_flag, p.status);
        if (!ok) break;
        mbar_arrive_expect_tx(&bars->v_full[vs], C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d_hint(&tmap_v, &bars->v_full[vs], sV(vs) + pn * kPanelBytes, pn * 64, h, k_row0 + j * kBN, keep);
        v_issued = j + 1;
      }
      if (!ok) {  // let every copy this thread started land before the CTA exits
        for (int t = 0; t < kTiles; ++t)
          if (n_kv(t) > 0) drain_wait(&bars->q_full[t], 0);
        // the newest copy into each stage is the last one that can still be in flight
        for (int j = max(0, k_issued - C::kKStages); j < k_issued; ++j)
          drain_wait(&bars->k_full[j % C::kKStages], (j / C::kKStages) & 1);
        for (int j = max(0, v_issued - C::kVStages); j < v_issued; ++j)
          drain_wait(&bars->v_full[j % C::kVStages], (j / C::kVStages) & 1);
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp + 1) {
    // ================================ MMA issuers ================================================
    // Early S (D = 64): one issuing thread per tile (warp 9 for tile 0, warp 10 for tile 1), so
    // neither tile's S or P*V waits behind the other's; the tensor core runs both streams in arrival
    // order.  Late S (D = 128, P aliased into S): one thread (warp 9) issues both tiles in the order
    // PV0(j) S0(j+1) PV1(j) S1(j+1), which keeps each tile's S right behind its own P*V.
    // A commit covers only the issuing thread's earlier MMAs.
    constexpr int fmt = kFp16 ? 0 : 1;
    constexpr uint32_t idesc_qk = instr_desc_f16(kBM, kBN, fmt, 0);
    constexpr uint32_t idesc_pv = instr_desc_f16(kBM, D, fmt, 1);
    auto issue_s = [&](int t, int j) {
      const uint32_t sQa = smem_addr(sQ(t));
      const uint32_t sKa = smem_addr(sK(j % C::kKStages));
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        // K-major, 128B swizzle: 16-element K steps advance 32 bytes inside a 128-byte row;
        // every 4 steps move to the next 64-column panel.  SBO = 8 rows * 128 B.
        const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
        mma_ss(tbase + C::col_s(t), smem_desc_sw128(sQa + off, 16, 1024), smem_desc_sw128(sKa + off, 16, 1024),
               idesc_qk, kk > 0 ? 1u : 0u);
      }
      mma_commit(&bars->s_full[t]);
      mma_commit(&bars->k_empty[t][j % C::kKStages]);
    };
    auto issue_pv = [&](int t, int j) {
      const uint32_t sVa = smem_addr(sV(j % C::kVStages));
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk) {
        // V is N-major (head dim contiguous): 16 keys = two 8-row swizzle atoms = 2048 bytes;
        // LBO = distance between the 64-column panels, SBO = 8 rows * 128 B.
        mma_ts(tbase + C::col_o(t), tbase + C::col_p(t) + kk * 8,
               smem_desc_sw128(sVa + kk * 2048, kPanelBytes, 1024), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(&bars->v_empty[t][j % C::kVStages]);
    };
    auto wait_k = [&](int j) {
      return mbar_wait(&bars->k_full[j % C::kKStages], (j / C::kKStages) & 1, abort_flag, p.status);
    };
    auto wait_v = [&](int j) {
      return mbar_wait(&bars->v_full[j % C::kVStages], (j / C::kVStages) & 1, abort_flag, p.status);
    };
    if constexpr (C::kEarlyS) {
      const int t = warp - kMmaWarp;
      const int n = n_kv(t);
      if (lane == 0 && n > 0) {
        bool ok = mbar_wait(&bars->q_full[t], 0, abort_flag, p.status) && wait_k(0);
        if (ok) {
          tc_fence_after();
          issue_s(t, 0);
        }
        for (int j = 0; ok && j < n; ++j) {
          // S_t(j+1) as soon as softmax t has read S_t(j); then P_t(j) V_j.
          if (j + 1 < n) {
            if (!(ok = wait_k(j + 1) && mbar_wait(&bars->s_free[t], j & 1, abort_flag, p.status))) break;
            tc_fence_after();
            issue_s(t, j + 1);
          }
          if (!(ok = wait_v(j) && mbar_wait(&bars->p_full[t], j & 1, abort_flag, p.status))) break;
          tc_fence_after();
          issue_pv(t, j);
          mma_commit(&bars->o_done[t]);
        }
        // no tensor-core work of this thread may still be in flight when TMEM and SMEM are released
        mma_commit(&bars->drain[t]);
        drain_wait(&bars->drain[t], 0);
      }
    } else if (warp == kMmaWarp && lane == 0) {
      bool ok = true;
      for (int t = 0; t < kTiles && ok; ++t)
        if (n_kv(t) > 0) ok = mbar_wait(&bars->q_full[t], 0, abort_flag, p.status);
      if (ok) ok = wait_k(0);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < kTiles; ++t)
          if (n_kv(t) > 0) issue_s(t, 0);
      }
      for (int j = 0; ok && j < n_max; ++j) {
        if (!(ok = wait_v(j))) break;
        bool k_next_ready = false;
        for (int t = 0; t < kTiles; ++t) {
          if (j >= n_kv(t)) continue;
          if (!(ok = mbar_wait(&bars->p_full[t], j & 1, abort_flag, p.status))) break;
          tc_fence_after();
          issue_pv(t, j);
          if (j + 1 < n_kv(t)) {  // P_t aliases S_t: S_t(j+1) follows P_t(j) V_j
            if (!k_next_ready && !(ok = wait_k(j + 1))) break;
            k_next_ready = true;
            tc_fence_after();
            issue_s(t, j + 1);
          } else {
            mma_commit(&bars->o_done[t]);
          }
        }
      }
      mma_commit(&bars->drain[0]);
      drain_wait(&bars->drain[0], 0);
    }
  }
  } else {
    regs_increase<kSoftmaxRegs>();
    // ================================ softmax / epilogue =========================================
    const int t = warp >> 2;
    const int n = n_kv(t);
    if (n > 0) {
      const int quarter = warp & 3;
      const int r = quarter * 32 + lane;
      const uint32_t lane_base = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
      const int tile_m0 = m0 + t * kBM;
      const int qi = tile_m0 + r;
      const int row_lim = p.causal ? min(Lk, qi + 1 + diag) : Lk;         // keys [0,row_lim) visible
      const int tile_lim = p.causal ? min(Lk, tile_m0 + 1 + diag) : Lk;   // smallest row_lim of the tile
      const float sl2 = p.scale_log2;
      const uint64_t sl2x2 = f2(sl2, sl2);
      float m_run = -INFINITY;
      uint64_t lsum = f2(0.f, 0.f);
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        if (!(ok = warp_wait(&bars->s_full[t], j & 1, abort_flag, p.status))) break;
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128_sync(lane_base + C::col_s(t), sr);
        if constexpr (C::kEarlyS) {  // S_t may now be overwritten by the next block's scores
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bars->s_free[t]);
        }
        const bool masked = (j + 1) * kBN > tile_lim;
        if (masked) {
          const int lim = row_lim - j * kBN;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        // row max (raw score units): four independent chains of 3-input max, one per 32 columns
        float mxc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int b0 = 32 * k;
          float m = fmax3(__uint_as_float(sr[b0]), __uint_as_float(sr[b0 + 1]), __uint_as_float(sr[b0 + 2]));
#pragma unroll
          for (int i = 3; i < 31; i += 2) m = fmax3(m, __uint_as_float(sr[b0 + i]), __uint_as_float(sr[b0 + i + 1]));
          mxc[k] = fmaxf(m, __uint_as_float(sr[b0 + 31]));
        }
        const float mx = fmaxf(fmax3(mxc[0], mxc[1], mxc[2]), mxc[3]);
        const float m_new = fmaxf(m_run, mx * sl2);
        // Rescale O only when the max grew by more than the threshold (warp-uniform decision); with
        // early S the multiplication of O waits below until P_t(j-1) V has landed in O.
        const bool need = m_new > m_run + kRescaleThreshold;
        float alpha = 1.f;
        bool rescale = false;
        if (j == 0) {
          m_run = m_new;
        } else if (__any_sync(0xffffffffu, need)) {
          rescale = true;
          if (need) {
            alpha = ex2(m_run - m_new);  // m_run = -inf only for rows without any key
            float l0, l1;
            f2_split(lsum, l0, l1);
            lsum = f2(l0 * alpha, l1 * alpha);
            m_run = m_new;
          }
        }
        const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
        const uint64_t negm = f2(-m_use, -m_use);
        uint64_t acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
        const uint32_t p_addr = lane_base + C::col_p(t);
        // First half of P into registers; with early S the previous P_t V product may still be
        // reading the P_t columns, so only then wait for it (it normally finished long before).
        uint32_t pk0[16], pk1[16];
#ifndef FA_UNIFIED_EXP
#define FA_UNIFIED_EXP 0
#endif
        if (masked && !FA_UNIFIED_EXP) {
          exp_chunk_regs<false, kFp16, 0>(sr, 0, sl2x2, negm, acc0, acc1, pk0);
          exp_chunk_regs<false, kFp16, 0>(sr, 1, sl2x2, negm, acc0, acc1, pk1);
        } else {
          exp_chunk_regs<true, kFp16, emu_pairs<D>()>(sr, 0, sl2x2, negm, acc0, acc1, pk0);
          exp_chunk_regs<true, kFp16, emu_pairs<D>()>(sr, 1, sl2x2, negm, acc0, acc1, pk1);
        }
        if constexpr (C::kEarlyS) {
          if (j > 0 && !(ok = warp_wait(&bars->o_done[t], (j - 1) & 1, abort_flag, p.status))) break;
          tc_fence_after();
        }
        if (rescale) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t orr[32];
            tmem_ld32_sync(lane_base + C::col_o(t) + ch * 32, orr);
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st32(lane_base + C::col_o(t) + ch * 32, orr);
          }
        }
        tmem_st16(p_addr, pk0);
        tmem_st16(p_addr + 16, pk1);
        if (masked && !FA_UNIFIED_EXP) {
#pragma unroll
          for (int ch = 2; ch < 4; ++ch) exp_chunk<false, kFp16, 0>(sr, ch, sl2x2, negm, acc0, acc1, p_addr);
        } else {
#pragma unroll
          for (int ch = 2; ch < 4; ++ch) exp_chunk<true, kFp16, emu_pairs<D>()>(sr, ch, sl2x2, negm, acc0, acc1, p_addr);
        }
        lsum = f2_add(lsum, f2_add(acc0, acc1));
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[t]);
      }
      // the last P_t V product (o_done is committed once per block with early S, once in total otherwise)
      if (ok) ok = warp_wait(&bars->o_done[t], C::kEarlyS ? ((n - 1) & 1) : 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        float l0, l1;
        f2_split(lsum, l0, l1);
        const float l_run = l0 + l1;
        const bool empty = (m_run == -INFINITY);
        const float inv_l = empty ? 0.f : 1.f / l_run;
        const bool store = qi < Lq;
        const size_t orow = (static_cast<size_t>(q_row0 + qi) * p.H + h) * D;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t orr[32];
          tmem_ld32_sync(lane_base + C::col_o(t) + ch * 32, orr);
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
        if (store) {
          const size_t li = (p.cu == nullptr) ? (static_cast<size_t>(b) * p.H + h) * p.Nq + qi
                                              : static_cast<size_t>(h) * p.Nq + q_row0 + qi;
          p.lse[li] = empty ? -INFINITY : (m_run + lg2(l_run)) * kLn2;
        }
      }
    }
  }

  // ---- teardown -------------------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// ---------------------------------------------------------------------------------------------
// host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3-D map over a [rows, H, D] 16-bit tensor: box = 64 columns x 1 head x 128 rows, 128B swizzle.
bool make_map(CUtensorMap* map, const void* base, int rows, int H, int D, bool fp16) {
  auto encode = get_encode_fn();
  if (!encode) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(kBM)};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kFp16, bool kOutF32>
int launch_t(const PrefillArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
             const FwdParams& p, cudaStream_t stream) {
  auto kern = fa_fwd_kernel<D, kFp16, kOutF32>;
  const int smem = Cfg<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return static_cast<int>(e);
  cudaFuncAttributes fattr;
  e = cudaFuncGetAttributes(&fattr, kern);
  if (e != cudaSuccess) return static_cast<int>(e);
  if (fattr.numRegs != kLaunchRegs) return static_cast<int>(cudaErrorInvalidConfiguration);
  long long blocks;
  if (a.cu_seqlens == nullptr)
    blocks = static_cast<long long>(p.num_pairs) * a.B * a.H;
  else
    blocks = (static_cast<long long>(a.Nq) / (kTiles * kBM) + a.B) * a.H;
  if (blocks > 0x7fffffffLL) return static_cast<int>(cudaErrorInvalidConfiguration);
  kern<<<static_cast<unsigned>(blocks), kThreads, smem, stream>>>(mq, mk, mv, p);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
  const bool varlen = a.cu_seqlens != nullptr;
  const int rows_q = varlen ? a.Nq : a.B * a.Nq;
  const int rows_k = varlen ? a.Nk : a.B * a.Nk;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, a.q, rows_q, a.H, a.D, a.fp16) || !make_map(&mk, a.k, rows_k, a.H, a.D, a.fp16) ||
      !make_map(&mv, a.v, rows_k, a.H, a.D, a.fp16))
    return static_cast<int>(cudaErrorInvalidValue);
  FwdParams p;
  p.o = a.o;
  p.lse = a.lse;
  p.cu = a.cu_seqlens;
  p.status = a.status;
  p.B = a.B;
  p.H = a.H;
  p.Nq = a.Nq;
  p.Nk = a.Nk;
  p.num_pairs = (a.Nq + kTiles * kBM - 1) / (kTiles * kBM);
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal ? 1 : 0;
  if (a.D == 64) {
    if (a.fp16) return a.o_fp32 ? launch_t<64, true, true>(a, mq, mk, mv, p, stream) : launch_t<64, true, false>(a, mq, mk, mv, p, stream);
    return a.o_fp32 ? launch_t<64, false, true>(a, mq, mk, mv, p, stream) : launch_t<64, false, false>(a, mq, mk, mv, p, stream);
  }
  if (a.fp16) return a.o_fp32 ? launch_t<128, true, true>(a, mq, mk, mv, p, stream) : launch_t<128, true, false>(a, mq, mk, mv, p, stream);
  return a.o_fp32 ? launch_t<128, false, true>(a, mq, mk, mv, p, stream) : launch_t<128, false, false>(a, mq, mk, mv, p, stream);
}

}  // namespace fa
