// fa_prefill_sm100.cu -- exact tiled attention forward on B200 tensor cores (tcgen05 + TMEM + TMA).
//
// The method (Ascend CANN ops-transformer FlashAttention article, sections "原理" and "代码讲解"):
// cut Q into row blocks and K/V into key blocks; for every Q block walk the K/V blocks, form the
// block scores, keep a running row max m and row sum l, rescale the output accumulator when m grows,
// add P_j V_j, and divide by l at the end.  S and P never leave the chip.
//
// Mapping to sm_100a (one CTA per 128-row Q tile of one (batch, head)):
//   warp 0      TMA producer: the Q tile once, then K_j and V_j through a kStages-deep ring of
//               128-byte-swizzled shared-memory tiles tracked by mbarriers.
//   warp 1      owns the tensor memory and issues the tensor-core work from one thread:
//               S_j = Q K_j^T  (tcgen05.mma, both operands in shared memory, fp32 into TMEM), and
//               O  += P_j V_j  (tcgen05.mma, P read from TMEM, V from shared memory).
//               S is double-buffered in TMEM so S_{j+1} runs while the softmax works on S_j.
//   warps 2..5  softmax: thread r owns query row r (TMEM lane r).  It reads its 128 scores with
//               tcgen05.ld, applies the causal / key-length mask, updates m and l, computes
//               P = 2^(S*scale*log2(e) - m) with the MUFU ex2, rescales its O row in TMEM when m
//               grew, writes P (bf16/fp16) back to TMEM, and finally writes O / l and the LSE.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+D) P [384,448) (P packs two 16-bit values per
// 32-bit column).  Causal runs stop at the last key block that the tile's last row can see, so
// fully masked blocks are never loaded or multiplied.
#include <cudaTypedefs.h>

#include <mutex>

#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kBM = 128;  // query rows per tile
constexpr int kBN = 128;  // keys per tile
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColP = 384;
constexpr int kPanelBytes = kBM * 64 * 2;  // one 64-column (128-byte) swizzle panel of a tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint64_t kDrainLimitNs = 200000000ull;

template <int D>
struct Cfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kBM * D * 2;
  static constexpr int kStages = (D == 64) ? 4 : 2;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + kTileBytes;
  static constexpr int kVOff = kKOff + kStages * kTileBytes;
  static constexpr int kBarOff = kVOff + kStages * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;  // barriers + alignment slack
};

struct Bars {
  uint64_t q_full;
  uint64_t k_full[4], k_empty[4], v_full[4], v_empty[4];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full, o_done, drain;
  uint32_t tmem_base;
  int abort_flag;
  int tile_b, tile_m;
};
static_assert(sizeof(Bars) <= 256, "barrier block too large");

struct FwdParams {
  void* o;
  float* lse;
  const int* cu;
  int* status;
  int B, H, Nq, Nk;
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

// Varlen: map a linear tile slot to (sequence, row block) by a warp-wide scan of the tile counts.
__device__ void find_varlen_tile(const FwdParams& p, int lane, int& out_b, int& out_m) {
  const int tile = blockIdx.x;
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
    const int nt = (len + kBM - 1) / kBM;
    int incl = nt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const int excl = incl - nt;
    const bool mine = nt > 0 && tile >= base + excl && tile < base + incl;
    const unsigned bal = __ballot_sync(0xffffffffu, mine);
    if (bal != 0u) {
      const int src = __ffs(bal) - 1;
      fb = c + src;
      fm = tile - base - __shfl_sync(0xffffffffu, excl, src);
      break;
    }
    base += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_status(p.status, kStatusCuSeqlens);
  out_b = fb;
  out_m = fm;
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
  const int h = blockIdx.y;

  // ---- tile geometry --------------------------------------------------------------------------
  int b, m_block;
  if (p.cu == nullptr) {
    b = blockIdx.z;
    m_block = blockIdx.x;
  } else {
    if (warp == 0) {
      int fb, fm;
      find_varlen_tile(p, lane, fb, fm);
      if (lane == 0) {
        bars->tile_b = fb;
        bars->tile_m = fm;
      }
    }
    __syncthreads();
    b = bars->tile_b;
    m_block = bars->tile_m;
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
  const int m0 = m_block * kBM;
  int kv_end = Lk;
  if (p.causal) kv_end = min(Lk, m0 + kBM + (Lk - Lq));
  const int n_kv = kv_end > 0 ? (kv_end + kBN - 1) / kBN : 0;

  if (n_kv == 0) {  // no row of this tile sees any key: O = 0, LSE = -inf
    if (warp >= 2) {
      const int r = (warp & 3) * 32 + lane;
      const int qi = m0 + r;
      if (qi < Lq) {
        const size_t orow = (static_cast<size_t>(q_row0 + qi) * p.H + h) * D;
        if constexpr (kOutF32) {
          float* out = static_cast<float*>(p.o) + orow;
          for (int d = 0; d < D; d += 4) *reinterpret_cast<float4*>(out + d) = make_float4(0.f, 0.f, 0.f, 0.f);
        } else {
          uint16_t* out = static_cast<uint16_t*>(p.o) + orow;
          for (int d = 0; d < D; d += 8) *reinterpret_cast<uint4*>(out + d) = make_uint4(0, 0, 0, 0);
        }
        const size_t li = (p.cu == nullptr) ? (static_cast<size_t>(b) * p.H + h) * p.Nq + qi
                                            : static_cast<size_t>(h) * p.Nq + q_row0 + qi;
        p.lse[li] = -INFINITY;
      }
    }
    return;
  }

  // ---- setup ----------------------------------------------------------------------------------
  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->s_full[i], 1);
      mbar_init(&bars->s_free[i], 4);
    }
    mbar_init(&bars->p_full, 4);
    mbar_init(&bars->o_done, 1);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  uint8_t* sQ = smem + C::kQOff;
  auto sK = [&](int st) { return smem + C::kKOff + st * C::kTileBytes; };
  auto sV = [&](int st) { return smem + C::kVOff + st * C::kTileBytes; };

  if (warp == 0) {
    // ================================ TMA producer ===============================================
    if (lane == 0) {
      tma_prefetch_desc(&tmap_q);
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      const uint64_t keep = l2_policy_evict_last();
      mbar_arrive_expect_tx(&bars->q_full, C::kTileBytes);
#pragma unroll
      for (int pn = 0; pn < C::kPanels; ++pn)
        tma_load_3d(&tmap_q, &bars->q_full, sQ + pn * kPanelBytes, pn * 64, h, q_row0 + m0);
      int last_k[4] = {-1, -1, -1, -1}, last_v[4] = {-1, -1, -1, -1};
      bool ok = true;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::kStages;
        const uint32_t ph = (j / C::kStages) & 1;
        if (!(ok = mbar_wait(&bars->k_empty[st], ph ^ 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(&bars->k_full[st], C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d_hint(&tmap_k, &bars->k_full[st], sK(st) + pn * kPanelBytes, pn * 64, h,
                           k_row0 + j * kBN, keep);
        last_k[st] = j;
        if (!(ok = mbar_wait(&bars->v_empty[st], ph ^ 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(&bars->v_full[st], C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d_hint(&tmap_v, &bars->v_full[st], sV(st) + pn * kPanelBytes, pn * 64, h,
                           k_row0 + j * kBN, keep);
        last_v[st] = j;
      }
      if (!ok) {  // let every copy this thread started land before the CTA exits
        drain_wait(&bars->q_full, 0);
        for (int st = 0; st < C::kStages; ++st) {
          if (last_k[st] >= 0) drain_wait(&bars->k_full[st], (last_k[st] / C::kStages) & 1);
          if (last_v[st] >= 0) drain_wait(&bars->v_full[st], (last_v[st] / C::kStages) & 1);
        }
      }
    }
  } else if (warp == 1) {
    // ================================ MMA issuer =================================================
    if (lane == 0) {
      constexpr int fmt = kFp16 ? 0 : 1;
      constexpr uint32_t idesc_qk = instr_desc_f16(kBM, kBN, fmt, 0);
      constexpr uint32_t idesc_pv = instr_desc_f16(kBM, D, fmt, 1);
      const uint32_t sQa = smem_addr(sQ);
      bool ok = mbar_wait(&bars->q_full, 0, abort_flag, p.status);
      auto issue_s = [&](int j) -> bool {
        const int st = j % C::kStages;
        const uint32_t ph = (j / C::kStages) & 1;
        if (!mbar_wait(&bars->k_full[st], ph, abort_flag, p.status)) return false;
        if (j >= 2 && !mbar_wait(&bars->s_free[j & 1], ((j >> 1) - 1) & 1, abort_flag, p.status))
          return false;
        tc_fence_after();
        const uint32_t d_tmem = tbase + ((j & 1) ? kColS1 : kColS0);
        const uint32_t sKa = smem_addr(sK(st));
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          // K-major, 128B swizzle: 16-element K steps advance 32 bytes inside a 128-byte row;
          // every 4 steps move to the next 64-column panel.  SBO = 8 rows * 128 B.
          const uint32_t off = (kk >> 2) * kPanelBytes + (kk & 3) * 32;
          mma_ss(d_tmem, smem_desc_sw128(sQa + off, 16, 1024), smem_desc_sw128(sKa + off, 16, 1024),
                 idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&bars->s_full[j & 1]);
        mma_commit(&bars->k_empty[st]);
        return true;
      };
      auto issue_pv = [&](int i) -> bool {
        const int st = i % C::kStages;
        const uint32_t ph = (i / C::kStages) & 1;
        if (!mbar_wait(&bars->v_full[st], ph, abort_flag, p.status)) return false;
        if (!mbar_wait(&bars->p_full, i & 1, abort_flag, p.status)) return false;
        tc_fence_after();
        const uint32_t sVa = smem_addr(sV(st));
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // V is N-major (head dim contiguous): 16 keys = two 8-row swizzle atoms = 2048 bytes;
          // LBO = distance between the 64-column panels, SBO = 8 rows * 128 B.
          mma_ts(tbase + kColO, tbase + kColP + kk * 8, smem_desc_sw128(sVa + kk * 2048, kPanelBytes, 1024),
                 idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bars->o_done);
        mma_commit(&bars->v_empty[st]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int j = 1; ok && j <= n_kv; ++j) {
        if (j < n_kv) ok = issue_s(j);
        if (ok) ok = issue_pv(j - 1);
      }
      // no tensor-core work may still be in flight when TMEM and shared memory are released
      mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
  } else {
    // ================================ softmax / correction / epilogue ============================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tbase + (static_cast<uint32_t>(quarter * 32) << 16);
    const int qi = m0 + r;
    const int diag = Lk - Lq;  // bottom-right causal alignment
    const int row_lim = p.causal ? min(Lk, qi + 1 + diag) : Lk;      // keys [0,row_lim) visible
    const int tile_lim = p.causal ? min(Lk, m0 + 1 + diag) : Lk;     // smallest row_lim of the tile
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!(ok = warp_wait(&bars->s_full[j & 1], (j >> 1) & 1, abort_flag, p.status))) break;
      tc_fence_after();
      const uint32_t s_addr = lane_base + ((j & 1) ? kColS1 : kColS0);
      uint32_t sr[128];
      tmem_ld128_sync(s_addr, sr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->s_free[j & 1]);

      float s[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(sr[c]);
      if ((j + 1) * kBN > tile_lim) {
        const int lim = row_lim - j * kBN;
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < 128; ++c) mx = fmaxf(mx, s[c]);
      const float m_new = fmaxf(m_run, mx * sl2);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = ex2(m_run - m_use);
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = ex2(fmaf(s[c], sl2, -m_use));
        const float p1 = ex2(fmaf(s[c + 1], sl2, -m_use));
        rs0 += p0;
        rs1 += p1;
        pk[c >> 1] = pack2<kFp16>(p0, p1);
      }
      l_run = l_run * alpha + (rs0 + rs1);
      if (j > 0) {
        // PV of the previous block must be done: it reads the P buffer and accumulates into O.
        if (!(ok = warp_wait(&bars->o_done, (j - 1) & 1, abort_flag, p.status))) break;
        tc_fence_after();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t orr[32];
            tmem_ld32_sync(lane_base + kColO + ch * 32, orr);
#pragma unroll
            for (int i = 0; i < 32; ++i) orr[i] = __float_as_uint(__uint_as_float(orr[i]) * alpha);
            tmem_st32(lane_base + kColO + ch * 32, orr);
          }
        }
      }
      {
        uint32_t h0[32], h1[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          h0[i] = pk[i];
          h1[i] = pk[32 + i];
        }
        tmem_st32(lane_base + kColP, h0);
        tmem_st32(lane_base + kColP + 32, h1);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
      m_run = m_new;
    }
    if (ok) ok = warp_wait(&bars->o_done, (n_kv - 1) & 1, abort_flag, p.status);
    if (ok) {
      tc_fence_after();
      const float inv_l = l_run > 0.f ? 1.f / l_run : 0.f;
      const bool store = qi < Lq;
      const size_t orow = (static_cast<size_t>(q_row0 + qi) * p.H + h) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t orr[32];
        tmem_ld32_sync(lane_base + kColO + ch * 32, orr);
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
        p.lse[li] = l_run > 0.f ? (m_run + lg2(l_run)) * kLn2 : -INFINITY;
      }
    }
  }

  // ---- teardown -------------------------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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
  dim3 grid;
  if (a.cu_seqlens == nullptr)
    grid = dim3((a.Nq + kBM - 1) / kBM, a.H, a.B);
  else
    grid = dim3(a.Nq / kBM + a.B, a.H, 1);
  kern<<<grid, kThreads, smem, stream>>>(mq, mk, mv, p);
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
