// fa_prefill_sm100.cu -- exact tiled attention forward on B200 tensor cores (tcgen05 + TMEM + TMA).
//
// The method (Ascend CANN ops-transformer FlashAttention article, sections "原理" and "代码讲解"):
// cut Q into row blocks and K/V into key blocks; for every Q block walk the K/V blocks, form the
// block scores, keep a running row max m and row sum l, rescale the output accumulator when m grows,
// add P_j V_j, and divide by l at the end.  S and P never leave the chip.
//
// Mapping to sm_100a.  One CTA owns two 128-row Q tiles (256 rows) of one (batch, head), so every
// K/V tile brought into shared memory feeds both, and each SM sub-partition runs two independent
// softmax warps (one per tile) that cover each other's waits:
//   warps 0-3   softmax of tile 0, warps 4-7 softmax of tile 1: thread r of a warpgroup owns query
//               row r (TMEM lane r).  Per key block it reads its 128 scores with tcgen05.ld (which
//               frees the S buffer for the next block's scores at once), masks them (causal diagonal
//               / key-length tail only), updates the running max m, computes
//               P = 2^(S*scale*log2(e) - m) -- part of the exponentials on the MUFU unit, part with a
//               polynomial on the FMA pipe -- into registers, accumulates l, then (once the previous
//               P*V product has released the P buffer) rescales O if needed and stores P, and at the
//               end writes O / l and the LSE.  O is rescaled only when m grew by more than 2^8 since
//               the last rescale; until then P and l use the stale max, which is exact because O and
//               l share it.
//   warp 8      TMA producer: Q tiles once, then K_j and V_j through rings of 128-byte-swizzled
//               shared-memory stages tracked by mbarriers.
//   warps 9-10  MMA issuers, one thread per tile (warp 9 also owns the tensor memory): S_t(j+1) as
//               soon as softmax t has read S_t(j), then P_t(j) V_j as soon as P_t(j) is stored.
//   warp 11     idle.
// Tensor memory (512 columns): S0 [0,128) S1 [128,256); D = 64: O0 [256,320) O1 [320,384) and P0
// [384,448) P1 [448,512) (two 16-bit values per 32-bit column, the A operand of P*V read from TMEM);
// D = 128: O0 [256,384) O1 [384,512) and P in shared memory (K-major, 128-byte swizzle, the A operand
// of P*V read from shared memory), which leaves no room for more than one K stage.
// Causal runs (optionally with a prefix of keys every query sees, the prefix-LM mask) stop at the last
// key block the tile's last row can see; fully masked blocks are never loaded or multiplied.  The pairs of one head run back to back (longest causal pair first) and
// share its K/V in L2.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "fa_prefill_common.cuh"

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
// Registers: launched with kLaunchRegs per thread; the two softmax warpgroups then take
// kSoftmaxRegs and the producer/MMA warpgroup gives back down to kControlRegs.  The split must not
// exceed the launch allocation (256 * 216 + 128 * 72 = 384 * 168), else setmaxnreg.inc would wait
// forever.  The build checks (ptxas report) that every instantiation is compiled to exactly
// kLaunchRegs registers, and the host confirms it once per device before the first launch.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 216;
constexpr int kControlRegs = 72;
static_assert(256 * kSoftmaxRegs + 128 * kControlRegs <= kThreads * kLaunchRegs, "register split");
// Of every kEmuEvery column pairs of exponentials, kEmuPairs run on the FMA pipe (measured best of
// 0..3 for both head dims).
#ifndef FA_EMU_PAIRS
#define FA_EMU_PAIRS 1
#endif
constexpr int kEmuPairs = FA_EMU_PAIRS;

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kBM * D * 2;
  // P of D = 128 lives in shared memory (tensor memory holds S0 S1 O0 O1)
  static constexpr bool kPSmem = (D == 128);
  static constexpr int kPBytes = kBM * kBN * 2;  // one tile's P, bf16/fp16
  // D = 128 has room for three 32 KB K/V stages next to Q and P: one K stage (K_{j+1} is loaded
  // once both S(j) are done and is needed a whole softmax step later) and two V stages (V_j is
  // needed at the end of step j, and a single stage would wait for the slower tile's P V).
  static constexpr int kKStages = (D == 64) ? 4 : 1;
  static constexpr int kVStages = (D == 64) ? 4 : 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTiles * kTileBytes;
  static constexpr int kVOff = kKOff + kKStages * kTileBytes;
  static constexpr int kPOff = kVOff + kVStages * kTileBytes;
  static constexpr int kBarOff = kPOff + (kPSmem ? kTiles * kPBytes : 0);
  static constexpr int kSmemBytes = kBarOff + 384 + 1024;  // barriers + alignment slack
  __device__ static constexpr uint32_t col_s(int t) { return t ? 128u : 0u; }
  __device__ static constexpr uint32_t col_o(int t) { return 256u + (t ? static_cast<uint32_t>(D) : 0u); }
  __device__ static constexpr uint32_t col_p(int t) { return t ? 448u : 384u; }  // D = 64 only
};
static_assert(Cfg<64>::kSmemBytes <= 232448 && Cfg<128>::kSmemBytes <= 232448, "shared memory budget");

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

// Row r of a K-major, 128-byte-swizzled P tile in shared memory: 32 keys (chunk ch) = four 16-byte
// groups of 8 keys; within the 1024-byte atom of 8 rows the group index is XOR-ed with r mod 8.
__device__ __forceinline__ void store_p_smem(uint32_t tile_base, int r, int ch, const uint32_t (&pk)[16]) {
  const uint32_t row = tile_base + (ch >> 1) * kPanelBytes + r * 128;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t grp = static_cast<uint32_t>(((ch & 1) * 4 + q) ^ (r & 7));
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + grp * 16), "r"(pk[4 * q]),
                 "r"(pk[4 * q + 1]), "r"(pk[4 * q + 2]), "r"(pk[4 * q + 3])
                 : "memory");
  }
}

template <int D, bool kFp16, bool kOutF32>
__global__ void __launch_bounds__(kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o,
                  const FwdParams p) {
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
    // Groups of head_group (b, h) heads run one after another, so the K/V of the heads in flight
    // stay in L2; inside a group the pairs with the most key blocks (causal) of all its heads come
    // first, heads fastest, so that the longest units start early and none is left for the end.
    const int bhs = p.B * p.H;
    const int per_group = p.head_group * p.num_units;
    const int grp = static_cast<int>(blockIdx.x / per_group), w = static_cast<int>(blockIdx.x % per_group);
    const int gsz = min(p.head_group, bhs - grp * p.head_group);
    const int bh = grp * p.head_group + w % gsz;
    pair = p.num_units - 1 - w / gsz;
    b = bh / p.H;
    h = bh % p.H;
  } else {
    h = blockIdx.x % p.H;
    const int slot = blockIdx.x / p.H;
    if (warp == 0) {
      int fb, fm;
      find_varlen_unit<kTiles * kBM>(p, slot, lane, fb, fm);
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
#ifndef FA_DEBUG  // the debug build walks every key block and lets the mask zero the invisible ones
    if (p.causal) kv_end = min(Lk, max(p.prefix, first + kBM + diag));
#endif
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
      mbar_init(&bars->drain[t], 1);
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
  auto sP = [&](int t) { return smem + C::kPOff + t * C::kPBytes; };

  if (warp >= 8) {
    regs_decrease<kControlRegs>();
    if (warp == kProducerWarp) {
      // ================================ TMA producer =============================================
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
      // ================================ MMA issuers ==============================================
      // One issuing thread per tile, so neither tile's S or P*V waits behind the other's; the tensor
      // core runs both streams in arrival order.  A commit covers only the issuing thread's earlier
      // MMAs, and that thread's MMAs complete in issue order.
      constexpr int fmt = kFp16 ? 0 : 1;
      constexpr uint32_t idesc_qk = instr_desc_f16(kBM, kBN, fmt, 0);
      constexpr uint32_t idesc_pv = instr_desc_f16(kBM, D, fmt, 1);
      const int t = warp - kMmaWarp;
      const int n = n_kv(t);
      auto issue_s = [&](int j) {
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
      auto issue_pv = [&](int j) {
        const uint32_t sVa = smem_addr(sV(j % C::kVStages));
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // V is N-major (head dim contiguous): 16 keys = two 8-row swizzle atoms = 2048 bytes;
          // LBO = distance between the 64-column panels, SBO = 8 rows * 128 B.
          const uint64_t vdesc = smem_desc_sw128(sVa + kk * 2048, kPanelBytes, 1024);
          if constexpr (C::kPSmem) {  // P K-major in shared memory, laid out like Q
            const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
            mma_ss(tbase + C::col_o(t), smem_desc_sw128(smem_addr(sP(t)) + off, 16, 1024), vdesc, idesc_pv,
                   (j > 0 || kk > 0) ? 1u : 0u);
          } else {
            mma_ts(tbase + C::col_o(t), tbase + C::col_p(t) + kk * 8, vdesc, idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&bars->o_done[t]);
        mma_commit(&bars->v_empty[t][j % C::kVStages]);
      };
      auto wait_k = [&](int j) {
        return mbar_wait(&bars->k_full[j % C::kKStages], (j / C::kKStages) & 1, abort_flag, p.status);
      };
      auto wait_v = [&](int j) {
        return mbar_wait(&bars->v_full[j % C::kVStages], (j / C::kVStages) & 1, abort_flag, p.status);
      };
      if (lane == 0 && n > 0) {
        bool ok = mbar_wait(&bars->q_full[t], 0, abort_flag, p.status) && wait_k(0);
        if (ok) {
          tc_fence_after();
          issue_s(0);
        }
        for (int j = 0; ok && j < n; ++j) {
          // S_t(j+1) as soon as softmax t has read S_t(j); then P_t(j) V_j.
          if (j + 1 < n) {
            if (!(ok = mbar_wait(&bars->s_free[t], j & 1, abort_flag, p.status) && wait_k(j + 1))) break;
            tc_fence_after();
            issue_s(j + 1);
          }
          if (!(ok = mbar_wait(&bars->p_full[t], j & 1, abort_flag, p.status) && wait_v(j))) break;
          tc_fence_after();
          issue_pv(j);
        }
        // no tensor-core work of this thread may still be in flight when TMEM and SMEM are released
        mma_commit(&bars->drain[t]);
        drain_wait(&bars->drain[t], 0);
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
      // keys [0, row_lim) are visible to this row; tile_lim is the smallest row_lim of the tile
      const int row_lim = p.causal ? min(Lk, max(p.prefix, qi + 1 + diag)) : Lk;
      const int tile_lim = p.causal ? min(Lk, max(p.prefix, tile_m0 + 1 + diag)) : Lk;
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
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->s_free[t]);  // S_t may now be overwritten by S_t(j+1)
        const bool masked = (j + 1) * kBN > tile_lim;
        if (masked) {
          const int lim = row_lim - j * kBN;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        const float m_new = fmaxf(m_run, row_max(sr) * sl2);  // raw score units, scaled
        // Rescale O only when the max grew by more than the threshold (warp-uniform decision); the
        // multiplication of O waits below until P_t(j-1) V has landed in O.
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
        // All of P into registers first; the P buffer (and O) belong to P_t(j-1) V until that
        // product completes, which it normally has by the time the exponentials are done.
        uint32_t pk[4][16];
        if (masked) {  // masked scores are -inf: keep their P exact zeros (MUFU ex2(-inf) = 0)
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) exp_chunk<kFp16, 0>(sr, ch, sl2x2, negm, acc0, acc1, pk[ch]);
        } else {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) exp_chunk<kFp16, kEmuPairs>(sr, ch, sl2x2, negm, acc0, acc1, pk[ch]);
        }
        lsum = f2_add(lsum, f2_add(acc0, acc1));
        if (j > 0) {
          if (!(ok = warp_wait(&bars->o_done[t], (j - 1) & 1, abort_flag, p.status))) break;
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
        if constexpr (C::kPSmem) {
          const uint32_t pbase = smem_addr(sP(t));
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) store_p_smem(pbase, r, ch, pk[ch]);
          // generic-proxy stores must be visible to the tensor core (async proxy) before P V
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          if (rescale) {
            tmem_wait_st();
            tc_fence_before();
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) tmem_st16(lane_base + C::col_p(t) + ch * 16, pk[ch]);
          tmem_wait_st();
          tc_fence_before();
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->p_full[t]);
      }
      // the last P_t V product (the issuer's MMAs complete in order, so all earlier ones are done)
      if (ok) ok = warp_wait(&bars->o_done[t], (n - 1) & 1, abort_flag, p.status);
      float l0, l1;
      f2_split(lsum, l0, l1);
      if (!kOutF32 && p.tma_out && tile_m0 + kBM <= Lq) {
        // a full tile of 16-bit O: rows normalised into shared memory (the tile's Q buffer, which no
        // MMA reads any more), one TMA store per 64-column panel.  All four warps of the tile reach
        // the named barrier, whether or not their loop completed.
        if (ok) {
          tc_fence_after();
          stage_row<D, kFp16>(lane_base + C::col_o(t), sQ(t), r, m_run, l0 + l1);
          const size_t li = lse_index(p, b, h, q_row0, qi);
          if (idx_ok(p.status, li, 1, lse_elems(p))) p.lse[li] = (m_run == -INFINITY) ? -INFINITY : (m_run + lg2(l0 + l1)) * kLn2;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        named_barrier(1 + t, 128);
        if (quarter == 0 && lane == 0 && *abort_flag == 0) {
#pragma unroll
          for (int pn = 0; pn < C::kPanels; ++pn)
            tma_store_3d(&tmap_o, sQ(t) + pn * kPanelBytes, pn * 64, h, q_row0 + tile_m0);
          tma_store_commit();
          tma_store_wait_read();  // the buffer is released with the CTA
        }
      } else if (ok) {
        tc_fence_after();
        write_row<D, kFp16, kOutF32>(p, lane_base + C::col_o(t), b, h, q_row0, qi, qi < Lq, m_run, l0 + l1);
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

template <int D, bool kFp16, bool kOutF32>
int launch_t(const PrefillArgs& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
             const CUtensorMap& mo, const FwdParams& p, cudaStream_t stream) {
  auto kern = fa_fwd_kernel<D, kFp16, kOutF32>;
  const int smem = Cfg<D>::kSmemBytes;
  // Once per device and context: raise the shared-memory limit and confirm the register count the
  // build checked (the setmaxnreg split above needs exactly the launch allocation).
  static PerContext<int> configured;
  int unused = 0;
  const int ce = configured.get(&unused, [&](int*) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return static_cast<int>(e);
    cudaFuncAttributes fattr;
    e = cudaFuncGetAttributes(&fattr, kern);
    if (e != cudaSuccess) return static_cast<int>(e);
    return fattr.numRegs == kLaunchRegs ? 0 : static_cast<int>(cudaErrorInvalidConfiguration);
  });
  if (ce != 0) return ce;
  long long blocks;
  if (a.cu_seqlens == nullptr)
    blocks = static_cast<long long>(p.num_units) * a.B * a.H;
  else  // sum over sequences of ceil(len / 256) <= total / 256 + B; spare slots exit at once
    blocks = (static_cast<long long>(a.Nq) / (kTiles * kBM) + a.B) * a.H;
  if (blocks > 0x7fffffffLL) return static_cast<int>(cudaErrorInvalidConfiguration);
  kern<<<static_cast<unsigned>(blocks), kThreads, smem, stream>>>(mq, mk, mv, mo, p);
  return static_cast<int>(cudaGetLastError());
}

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

}  // namespace

bool make_tma_map(CUtensorMap* map, const void* base, int rows, int H, int D, bool fp16, int box_rows) {
  auto encode = get_encode_fn();
  if (!encode) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(H) * D * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(map, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
  const bool varlen = a.cu_seqlens != nullptr;
  const int rows_q = varlen ? a.Nq : a.B * a.Nq;
  const int rows_k = varlen ? a.Nk : a.B * a.Nk;
  CUtensorMap mq, mk, mv, mo;
  if (!make_tma_map(&mq, a.q, rows_q, a.H, a.D, a.fp16, kBM) || !make_tma_map(&mk, a.k, rows_k, a.H, a.D, a.fp16, kBN) ||
      !make_tma_map(&mv, a.v, rows_k, a.H, a.D, a.fp16, kBN))
    return static_cast<int>(cudaErrorInvalidValue);
  // 16-bit O is stored by TMA (same box as Q); an fp32 O keeps the per-thread stores
  if (a.o_fp32) mo = mq;
  else if (!make_tma_map(&mo, a.o, rows_q, a.H, a.D, a.fp16, kBM)) return static_cast<int>(cudaErrorInvalidValue);
  FwdParams p;
  p.o = a.o;
  p.lse = a.lse;
  p.cu = a.cu_seqlens;
  p.status = a.status;
  p.B = a.B;
  p.H = a.H;
  p.Nq = a.Nq;
  p.Nk = a.Nk;
  p.num_units = (a.Nq + kTiles * kBM - 1) / (kTiles * kBM);
  p.scale_log2 = a.scale * kLog2e;
  p.causal = a.causal ? 1 : 0;
  p.prefix = a.causal ? a.prefix : 0;
  // about FA_GROUP_KV_MB of K and V per head group (half of L2: measured best of 8-64 heads at
  // 2 MB per head), at least one head
#ifndef FA_GROUP_KV_MB
#define FA_GROUP_KV_MB 64
#endif
  const long long kv_head = 2LL * a.Nk * a.D * 2;
  p.head_group = static_cast<int>(
      std::max(1LL, std::min<long long>(static_cast<long long>(a.B) * a.H, (static_cast<long long>(FA_GROUP_KV_MB) << 20) / kv_head)));
#ifdef FA_HEAD_GROUP  // tuning: a fixed head-group size
  p.head_group = FA_HEAD_GROUP;
#endif
  p.tma_out = a.o_fp32 ? 0 : 1;
#ifdef FA_NO_TMA_OUT  // tuning: per-thread O stores for every tile
  p.tma_out = 0;
#endif
  if (a.D == 64) {
    if (a.fp16) return a.o_fp32 ? launch_t<64, true, true>(a, mq, mk, mv, mo, p, stream) : launch_t<64, true, false>(a, mq, mk, mv, mo, p, stream);
    return a.o_fp32 ? launch_t<64, false, true>(a, mq, mk, mv, mo, p, stream) : launch_t<64, false, false>(a, mq, mk, mv, mo, p, stream);
  }
  if (a.fp16) return a.o_fp32 ? launch_t<128, true, true>(a, mq, mk, mv, mo, p, stream) : launch_t<128, true, false>(a, mq, mk, mv, mo, p, stream);
  return a.o_fp32 ? launch_t<128, false, true>(a, mq, mk, mv, mo, p, stream) : launch_t<128, false, false>(a, mq, mk, mv, mo, p, stream);
}

}  // namespace fa
