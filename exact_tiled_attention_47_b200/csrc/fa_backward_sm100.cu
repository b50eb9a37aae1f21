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
//                       dP = dO V_j^T into TMEM, the eight compute warps (thread = query row, two
//                       warps per TMEM lane quarter, one per 64-column half) form dS and pack it
//                       (bf16/fp16) over the dP columns they have read, then dQ += dS K_j accumulates
//                       in TMEM.  dQ * scale is written at the end.
//   bwd_dkdv_kernel     CTA = one 128-row key tile.  Per query block i: S^T = K Q_i^T and
//                       dP^T = V dO_i^T into TMEM, the compute warps (thread = key row) form P^T and
//                       dS^T (the block's LSE and Drow come through shared memory) and pack both over
//                       the dP^T columns they have read, then dV += P^T dO_i and dK += dS^T Q_i
//                       accumulate in TMEM.  dV and dK * scale are written at the end.
// Both recompute S and dP (two more GEMMs than the minimum) so that each gradient is owned by one
// CTA and accumulates in TMEM.  Warp 8 is the TMA producer; warp 9 owns TMEM and issues S and dP
// (and dV) from one thread, warp 10 the products that read dS (dQ; dK).  A single thread issues an
// MMA about every 64 cycles whatever N up to 128 (measured), so S and dP are whole-block products
// (M = N = 128) and the schedule keeps the issue threads off the compute warps' path: S is released for the next block's S as soon as the
// compute warps hold it in registers, and dP goes into one of two TMEM buffers two blocks ahead
// (after the gradient products that read that buffer; with one buffer, as in dK/dV at D = 128,
// right after them).  The MMA forms are those of the forward kernel: SS with both operands K-major
// (S, dP) and TS with the A operand in TMEM and an N-major B in shared memory (dQ, dV, dK).  Causal
// runs skip fully masked blocks; masking is applied on the blocks that cross the diagonal and at
// the sequence ends.  The masks and layouts are those of the forward kernel: causal (bottom-right
// aligned), the prefix-LM mask (keys [0, prefix) visible to every query of the sequence) and packed
// varlen sequences indexed through cu_seqlens (LSE and Drow [H, total]).
#include <cudaTypedefs.h>

#include <algorithm>

#include "fa_prefill_common.cuh"

namespace fa {
namespace {

constexpr int kBT = 128;  // rows per tile (queries or keys)
// MMA-issuing threads: one issues S and dP (and owns TMEM); with two, a second issues the gradient
// products that read the compute warps' results (dQ; dK), since one thread issues an MMA only every
// ~64 cycles (two: +2 % at D = 128, no change at D = 64, measured)
#ifndef FA_BWD_ISSUERS
#define FA_BWD_ISSUERS 2
#endif
constexpr int kIssuers = FA_BWD_ISSUERS;
static_assert(kIssuers == 1 || kIssuers == 2, "one or two MMA issuers");
constexpr int kThreads = (9 + kIssuers) * 32;  // 8 compute warps, a TMA producer warp, the MMA warps
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;   // S and dP (and, with one issuer, everything); owns TMEM
constexpr int kMmaWarp2 = 10;  // with two issuers: the gradient products that read dS (dQ; dK)
constexpr uint32_t kTmemCols = 512;
constexpr int kPanelBytes = kBT * 64 * 2;  // one 64-column (128-byte) swizzle panel of a tile
constexpr int kMaxStages = 3;  // streamed-tile stages: 3 at D = 64, 2 at D = 128 (shared memory)
// Tensor memory: S (or S^T) in columns [0, 128), one or two dP (dP^T) buffers of 128 columns after it
// (the compute warps pack their 16-bit results into the dP columns they have read), then the
// accumulators (dQ; or dV and dK).
constexpr uint32_t kColS = 0, kColDP = 128;

template <int D>
struct BwdCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kBT * D * 2;
  static constexpr int kSt = (D == 64) ? 3 : 2;
  // dP buffers: two where they fit next to the accumulators (dQ: always; dK/dV: D = 64)
  template <bool kDkdv>
  static constexpr int kDPBufs = (!kDkdv || D == 64) ? 2 : 1;
  template <bool kDkdv>
  static constexpr uint32_t kColAcc = kColDP + 128 * kDPBufs<kDkdv>;
  static constexpr int kUsed = (2 + 2 * kSt) * kTileBytes + 2 * kSt * kBT * 4 + 256 + 1024;
  // at least 120 KB so that one CTA (which takes all 512 TMEM columns) runs per SM
  static constexpr int kSmemBytes = kUsed > 120 * 1024 ? kUsed : 120 * 1024;
  // dQ kernel: K and V stream through rings of their own, K three deep (S(j+1) is issued while
  // dQ(j) may still read K(j)), V three deep at D = 64 and two at D = 128, where shared memory ends
  // (V is read only by dP, which runs two blocks ahead; two V slots measured 2.6 % slower at D = 64)
  static constexpr int kKSt = 3, kVSt = (D == 64) ? 3 : 2;
  // rings of equal depth: the release of K(j) after dQ(j) also releases V(j) (dP(j) completed before
  // dQ(j) in the issuing thread's order), which saves one commit -- an MMA-pipe instruction -- per block
  static constexpr bool kJointKV = kKSt == kVSt;
  static constexpr int kDqUsed = (2 + kKSt + kVSt) * kTileBytes + 256 + 1024;
  static constexpr int kDqSmemBytes = kDqUsed > 120 * 1024 ? kDqUsed : 120 * 1024;
};
static_assert(BwdCfg<128>::kSmemBytes <= 232448 && BwdCfg<128>::kDqSmemBytes <= 232448, "shared memory budget");

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
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];  // dQ: the K and V rings
  uint64_t s_full;   // S and dP of the next block are in TMEM (one phase per block)
  uint64_t s_read;   // the compute warps hold the block's S in registers: S may be overwritten
  uint64_t p_full;   // the block's packed dS (and P^T) are in TMEM
  uint64_t o_done, drain, drain2;
  uint64_t g_done[2];  // two issuers: the block's dS-reading product (dQ; dK) has completed
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

// d = a b^T over K = D (both operands K-major in shared memory; a and b are descriptors)
template <int D>
__device__ __forceinline__ void mma_kk(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) mma_ss(d, a + kstep_off(kk), b + kstep_off(kk), idesc, kk > 0 ? 1u : 0u);
}

// Where 16-column chunk kk (0..7) of a block keeps its packed 16-bit values in the dP buffer: the
// compute warps of column half c = kk / 4 write chunk ci = kk % 4 over the dP columns they have just
// read.  dQ kernel: dS at 64 c + 8 ci.  dK/dV kernel: dS^T at 64 c + 16 ci and P^T 8 columns after it.
__host__ __device__ constexpr uint32_t ds_col_dq(int kk) { return static_cast<uint32_t>(64 * (kk >> 2) + 8 * (kk & 3)); }
__host__ __device__ constexpr uint32_t ds_col_dkdv(int kk) {
  return static_cast<uint32_t>(64 * (kk >> 2) + 16 * (kk & 3));
}

// packed product of fp32 pairs; with fma.rn.f32x2 and add.rn.f32x2 it rounds each lane as the scalar
// instruction does (round to nearest, subnormals kept), at one issue slot per pair
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_of(const uint32_t* x) { return f2(__uint_as_float(x[0]), __uint_as_float(x[1])); }

// d (+)= A (TMEM, 128 x 128 packed 16-bit, chunk kk at a_tmem + col(kk)) * B (shared, N-major 128
// rows from the descriptor b; 16 rows = two 8-row swizzle atoms = 2048 bytes).  Two products
// (d0, d1) have their K steps interleaved.
template <uint32_t (*col)(int)>
__device__ __forceinline__ void mma_tn(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < kBT / 16; ++kk)
    mma_ts(d, a + col(kk), b + ((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
}
template <uint32_t (*col)(int)>
__device__ __forceinline__ void mma_tn2(uint32_t d0, uint32_t a0, uint64_t b0, uint32_t d1, uint32_t a1, uint64_t b1,
                                        uint32_t idesc, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < kBT / 16; ++kk) {
    mma_ts(d0, a0 + col(kk), b0 + ((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
    mma_ts(d1, a1 + col(kk), b1 + ((kk * 2048) >> 4), idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}


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

// o_done_count: the issuing threads whose products accumulate into the CTA's gradients
__device__ __forceinline__ void bwd_setup(BwdBars* bars, int warp, int o_done_count) {
  if (threadIdx.x == 0) {
    mbar_init(&bars->fixed_full, 1);
    for (int s = 0; s < kMaxStages; ++s) {
      mbar_init(&bars->st_full[s], 1);
      mbar_init(&bars->st_empty[s], kIssuers);  // every issuing thread reads the streamed stage
      mbar_init(&bars->stat_full[s], 1);
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], kIssuers);  // K: S (first thread) and dQ (second thread)
    }
    for (int s = 0; s < 3; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->s_full, 1);
    mbar_init(&bars->s_read, 8);
    mbar_init(&bars->p_full, 8);
    mbar_init(&bars->o_done, o_done_count);
    mbar_init(&bars->drain, 1);
    mbar_init(&bars->drain2, 1);
    mbar_init(&bars->g_done[0], 1);
    mbar_init(&bars->g_done[1], 1);
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
  auto sK = [&](int ks) { return smem + (2 + ks) * C::kTileBytes; };
  auto sV = [&](int vs) { return smem + (2 + C::kKSt + vs) * C::kTileBytes; };
  BwdBars* bars = reinterpret_cast<BwdBars*>(smem + (2 + C::kKSt + C::kVSt) * C::kTileBytes);
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
  bwd_setup(bars, warp, 1);
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
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        const int ks = j % C::kKSt, vs = j % C::kVSt;
        if (!(ok = mbar_wait(&bars->k_empty[ks], ((j / C::kKSt) & 1) ^ 1, abort_flag, p.status))) break;
        mbar_arrive_expect_tx(&bars->k_full[ks], C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d_hint(&tm_k, &bars->k_full[ks], sK(ks) + pn * kPanelBytes, pn * 64, h, u.k_row0 + j * kBT, keep);
        k_issued = j + 1;
        if (!C::kJointKV && !(ok = mbar_wait(&bars->v_empty[vs], ((j / C::kVSt) & 1) ^ 1, abort_flag, p.status)))
          break;
        mbar_arrive_expect_tx(&bars->v_full[vs], C::kTileBytes);
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
          tma_load_3d_hint(&tm_v, &bars->v_full[vs], sV(vs) + pn * kPanelBytes, pn * 64, h, u.k_row0 + j * kBT, keep);
        v_issued = j + 1;
      }
      if (!ok) {  // the newest copy into each slot is the only one that can still be in flight
        drain_wait(&bars->fixed_full, 0);
        for (int j = max(0, k_issued - C::kKSt); j < k_issued; ++j) drain_wait(&bars->k_full[j % C::kKSt], (j / C::kKSt) & 1);
        for (int j = max(0, v_issued - C::kVSt); j < v_issued; ++j) drain_wait(&bars->v_full[j % C::kVSt], (j / C::kVSt) & 1);
      }
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp2) {
    // Block j: S = Q K_j^T into the S columns and dP = dO V_j^T into dP buffer j % 2 (N = 128, so
    // each MMA carries twice the work of a half block at the same issue cost), then, once the compute
    // warps have packed dS into that buffer, dQ += dS K_j.  S(j+1) is issued as soon as the compute
    // warps hold S(j) in registers; dP(j+2) goes into buffer j % 2 once dQ(j) no longer needs it, so
    // only S is issued between the blocks of the compute warps.  With two issuing threads the second
    // issues dQ (and reports its completion: g_done), so the two streams of MMAs are issued side by
    // side.
    constexpr int fmt = kFp16 ? 0 : 1;
    constexpr uint32_t idesc_s = instr_desc_f16(kBT, kBT, fmt, 0);
    constexpr uint32_t idesc_g = instr_desc_f16(kBT, D, fmt, 1);
    constexpr uint32_t col_acc = C::template kColAcc<false>;
    const uint64_t d_q = desc_kmajor(sQ), d_do = desc_kmajor(sDO);
    const uint64_t d_k = desc_kmajor(sK(0)), d_v = desc_kmajor(sV(0)), d_kn = desc_nmajor(sK(0));
    auto slot_off = [&](int slot) { return static_cast<uint64_t>((slot * C::kTileBytes) >> 4); };
    auto wait_k = [&](int jb) {
      return mbar_wait(&bars->k_full[jb % C::kKSt], (jb / C::kKSt) & 1, abort_flag, p.status);
    };
    auto wait_v = [&](int jb) {
      return mbar_wait(&bars->v_full[jb % C::kVSt], (jb / C::kVSt) & 1, abort_flag, p.status);
    };
    auto issue_dQ = [&](int j) {
      mma_tn<ds_col_dq>(tbase + col_acc, tbase + kColDP + 128 * (j & 1), d_kn + slot_off(j % C::kKSt), idesc_g,
                        j > 0);
    };
    if (lane == 0 && warp == kMmaWarp) {
      auto issue_S = [&](int jb) {
        mma_kk<D>(tbase + kColS, d_q, d_k + slot_off(jb % C::kKSt), idesc_s);
        // with two issuers this thread's share of releasing block jb's slots: S(jb), and dP(jb)
        // issued before it
        if (kIssuers == 2) mma_commit(&bars->k_empty[jb % C::kKSt]);
      };
      auto issue_dP = [&](int jb) {  // V(jb) is released once this product has completed
        mma_kk<D>(tbase + kColDP + 128 * (jb & 1), d_do, d_v + slot_off(jb % C::kVSt), idesc_s);
        if (!C::kJointKV) mma_commit(&bars->v_empty[jb % C::kVSt]);
      };
      bool ok = mbar_wait(&bars->fixed_full, 0, abort_flag, p.status) && wait_k(0) && wait_v(0);
      if (ok) {
        tc_fence_after();
        issue_dP(0);
        issue_S(0);
        mma_commit(&bars->s_full);
        if (n > 1 && (ok = wait_v(1))) {
          tc_fence_after();
          issue_dP(1);
        }
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n) {
          // the compute warps have S(j) in registers: S(j+1) may overwrite it
          if (!(ok = mbar_wait(&bars->s_read, j & 1, abort_flag, p.status) && wait_k(j + 1))) break;
          tc_fence_after();
          issue_S(j + 1);
          mma_commit(&bars->s_full);  // S(j+1) and dP(j+1)
        }
        if (kIssuers == 1) {
          if (!(ok = mbar_wait(&bars->p_full, j & 1, abort_flag, p.status))) break;
          tc_fence_after();
          issue_dQ(j);
          mma_commit(&bars->k_empty[j % C::kKSt]);  // K(j): S(j) and dQ(j) issued (and V(j) with joint rings)
        }
        if (j + 2 < n) {
          // dP(j+2) goes into buffer j % 2: after dQ(j) in this thread's order, or once the other
          // thread's dQ(j) has completed
          if (kIssuers == 2 && !(ok = mbar_wait(&bars->g_done[j & 1], (j >> 1) & 1, abort_flag, p.status))) break;
          if (!(ok = wait_v(j + 2))) break;
          tc_fence_after();
          issue_dP(j + 2);
        }
      }
      if (kIssuers == 1 && ok) mma_commit(&bars->o_done);
      mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    } else if (kIssuers == 2 && lane == 0 && warp == kMmaWarp2) {
      bool ok = true;
      for (int j = 0; ok && j < n; ++j) {
        if (!(ok = mbar_wait(&bars->p_full, j & 1, abort_flag, p.status))) break;
        tc_fence_after();
        issue_dQ(j);
        mma_commit(&bars->g_done[j & 1]);         // buffer j % 2 may take dP(j+2)
        mma_commit(&bars->k_empty[j % C::kKSt]);  // this thread's share of releasing K(j) (and V(j))
      }
      if (ok) mma_commit(&bars->o_done);
      mma_commit(&bars->drain2);
      drain_wait(&bars->drain2, 0);
    }
  } else {
    const int hc = warp >> 2;  // column half of every key block this warp works on
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
    const uint64_t sl2x2 = f2(sl2, sl2), nlse2x2 = f2(-lse2, -lse2), ndrx2 = f2(-dr, -dr);
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      if (!(ok = warp_wait(&bars->s_full, j & 1, abort_flag, p.status))) break;
      tc_fence_after();
      const bool masked = (j + 1) * kBT > tile_lim;
      const int lim = row_lim - j * kBT;
      // the half's 64 key columns in 16-column chunks; chunk c+1 is loaded while chunk c is computed
      const uint32_t cs = lane_base + kColS + 64 * hc, cd = lane_base + kColDP + 128 * (j & 1) + 64 * hc;
      uint32_t sb[2][16], db[2][16];
      tmem_ld16_async(cs, sb[0]);
      tmem_ld16_async(cd, db[0]);
      tmem_wait_ld_pair(sb[0], db[0]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int cur = c & 1;
        if (c + 1 < 4) {
          tmem_ld16_async(cs + 16 * (c + 1), sb[cur ^ 1]);
          tmem_ld16_async(cd + 16 * (c + 1), db[cur ^ 1]);
        }
        uint32_t pk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int c0 = 64 * hc + 16 * c + 2 * i;  // key column in the block
          // P = 2^(s scale log2e - LSE log2e), dS = P (dP - Drow), two columns per instruction
          float x0, x1;
          f2_split(f2_fma(f2_of(&sb[cur][2 * i]), sl2x2, nlse2x2), x0, x1);
          float p0 = ex2(x0), p1 = ex2(x1);
          if (masked) {
            if (c0 >= lim) p0 = 0.f;
            if (c0 + 1 >= lim) p1 = 0.f;
          }
          float d0, d1;
          f2_split(f2_mul(f2(p0, p1), f2_add(f2_of(&db[cur][2 * i]), ndrx2)), d0, d1);
          pk[i] = pack2<kFp16>(d0, d1);
        }
        tmem_st8(cd + 8 * c, pk);  // dS over dP columns this warp has already read (ds_col_dq)
        if (c + 1 < 4) {
          tmem_wait_ld_pair(sb[cur ^ 1], db[cur ^ 1]);
          if (c == 2) {  // all of this warp's S columns are in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->s_read);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok) ok = warp_wait(&bars->o_done, 0, abort_flag, p.status);
    if (ok) {
      tc_fence_after();
      const size_t row = static_cast<size_t>(u.q_row0 + min(qi, Lq - 1)) * p.H + h;
      // the two column halves of warps store the two halves of the row
      store_grad_row<D, kFp16, kOutF32>(p.g0, row * D, lane_base + C::template kColAcc<false>, p.scale, qi < Lq,
                                        p.status, p.g0_n, hc * D / 64, (hc + 1) * D / 64);
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
  float* sStat = reinterpret_cast<float*>(smem + (2 + 2 * C::kSt) * C::kTileBytes);  // [stage][-lse2 | -drow][128]
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
  bwd_setup(bars, warp, kIssuers);
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
      // the block's negated LSE (log2 units; -inf for rows without keys or past the end, so P = 0) and
      // negated Drow: all eight loads of a lane are independent and in flight together
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
        stat[lane + 32 * e] = (lv[e] != -INFINITY) ? -(lv[e] * kLog2e) : -INFINITY;
        stat[kBT + lane + 32 * e] = -dv[e];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->stat_full[st]);  // release: orders the warp's stores above
    }
    if (!ok && lane == 0) {
      drain_wait(&bars->fixed_full, 0);
      for (int jj = max(0, issued - C::kSt); jj < issued; ++jj) drain_wait(&bars->st_full[jj % C::kSt], (jj / C::kSt) & 1);
    }
  } else if (warp == kMmaWarp || warp == kMmaWarp2) {
    // Query block i (jj-th of the tile): S^T = K Q_i^T into the S columns and dP^T = V dO_i^T into a
    // dP buffer (N = 128); once the compute warps have packed dS^T and P^T into that buffer,
    // dV += P^T dO_i and dK += dS^T Q_i.  S^T(jj+1) is issued as soon as the compute warps hold
    // S^T(jj) in registers.  With two dP buffers (D = 64) dP^T(jj+2) follows the products of block
    // jj; with one (D = 128) dP^T(jj+1) does.  With two issuing threads the second issues dK (and
    // reports its completion: g_done) while the first issues S^T, dP^T and dV.
    constexpr int fmt = kFp16 ? 0 : 1;
    constexpr uint32_t idesc_s = instr_desc_f16(kBT, kBT, fmt, 0);
    constexpr uint32_t idesc_g = instr_desc_f16(kBT, D, fmt, 1);
    constexpr int kBufs = C::template kDPBufs<true>;
    constexpr uint32_t col_acc = C::template kColAcc<true>;
    const uint64_t d_k = desc_kmajor(sK), d_v = desc_kmajor(sV);
    const uint64_t d_q = desc_kmajor(sQ(0)), d_do = desc_kmajor(sDO(0));
    const uint64_t d_qn = desc_nmajor(sQ(0)), d_don = desc_nmajor(sDO(0));
    auto stage_off = [&](int st) { return static_cast<uint64_t>((st * C::kTileBytes) >> 4); };
    auto buf = [&](int jb) { return kColDP + 128 * (jb % kBufs); };
    // dP^T of block jb + kBufs goes out after block jb's products: it needs block jb + kBufs's stage
    // (kSt >= kBufs + 1 stages, so it is not block jb's own)
    static_assert(C::kSt >= kBufs + 1, "stages for the dP lookahead");
    if (lane == 0 && warp == kMmaWarp) {
      auto wait_stage = [&](int jb) {
        return mbar_wait(&bars->st_full[jb % C::kSt], (jb / C::kSt) & 1, abort_flag, p.status);
      };
      auto issue_S = [&](int jb) { mma_kk<D>(tbase + kColS, d_k, d_q + stage_off(jb % C::kSt), idesc_s); };
      auto issue_dP = [&](int jb) { mma_kk<D>(tbase + buf(jb), d_v, d_do + stage_off(jb % C::kSt), idesc_s); };
      bool ok = mbar_wait(&bars->fixed_full, 0, abort_flag, p.status) && wait_stage(0);
      if (ok) {
        tc_fence_after();
        issue_S(0);
        issue_dP(0);
        mma_commit(&bars->s_full);
        for (int jb = 1; ok && jb < kBufs && jb < n; ++jb) {  // the other buffers' first blocks
          if ((ok = wait_stage(jb))) {
            tc_fence_after();
            issue_dP(jb);
          }
        }
      }
      for (int jj = 0; ok && jj < n; ++jj) {
        const int st = jj % C::kSt;
        if (jj + 1 < n) {
          // the compute warps have S^T(jj) in registers: S^T(jj+1) may overwrite it (with two buffers
          // its stage was waited for when dP^T(jj+1) was issued)
          if (!(ok = mbar_wait(&bars->s_read, jj & 1, abort_flag, p.status))) break;
          if (kBufs == 1 && !(ok = wait_stage(jj + 1))) break;
          tc_fence_after();
          issue_S(jj + 1);
          if (kBufs > 1) mma_commit(&bars->s_full);  // S^T(jj+1) and dP^T(jj+1)
        }
        if (!(ok = mbar_wait(&bars->p_full, jj & 1, abort_flag, p.status))) break;
        tc_fence_after();
        if (kIssuers == 1) {
          // dV += P^T dO_i,  dK += dS^T Q_i  (P^T 8 columns after dS^T in every chunk)
          mma_tn2<ds_col_dkdv>(tbase + col_acc, tbase + buf(jj) + 8, d_don + stage_off(st), tbase + col_acc + D,
                               tbase + buf(jj), d_qn + stage_off(st), idesc_g, jj > 0);
        } else {
          mma_tn<ds_col_dkdv>(tbase + col_acc, tbase + buf(jj) + 8, d_don + stage_off(st), idesc_g, jj > 0);
        }
        mma_commit(&bars->st_empty[st]);  // this thread's products reading stage st are issued
        if (jj + kBufs < n) {
          // dP^T(jj+kBufs) goes into block jj's buffer: after its products in this thread's order, or
          // once the other thread's dK(jj) has completed
          if (kIssuers == 2 && !(ok = mbar_wait(&bars->g_done[jj % kBufs], (jj / kBufs) & 1, abort_flag, p.status)))
            break;
          if (!(ok = wait_stage(jj + kBufs))) break;
          tc_fence_after();
          issue_dP(jj + kBufs);
          if (kBufs == 1) mma_commit(&bars->s_full);  // S^T(jj+1) and dP^T(jj+1)
        }
      }
      if (ok) mma_commit(&bars->o_done);
      mma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    } else if (kIssuers == 2 && lane == 0 && warp == kMmaWarp2) {
      bool ok = true;
      for (int jj = 0; ok && jj < n; ++jj) {
        const int st = jj % C::kSt;
        if (!(ok = mbar_wait(&bars->p_full, jj & 1, abort_flag, p.status))) break;
        tc_fence_after();
        mma_tn<ds_col_dkdv>(tbase + col_acc + D, tbase + buf(jj), d_qn + stage_off(st), idesc_g, jj > 0);  // dK
        mma_commit(&bars->g_done[jj % kBufs]);  // block jj's buffer may take dP^T(jj + kBufs)
        mma_commit(&bars->st_empty[st]);        // this thread's share of releasing stage st
      }
      if (ok) mma_commit(&bars->o_done);
      mma_commit(&bars->drain2);
      drain_wait(&bars->drain2, 0);
    }
  } else {
    constexpr int kBufs = C::template kDPBufs<true>;
    const int hc = warp >> 2;  // column half of every query block this warp works on
    const int r = (warp & 3) * 32 + lane;
    const int kj = n0 + r;  // this thread's key
    const uint32_t lane_base = tbase + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2(sl2, sl2);
    bool ok = true;
    for (int jj = 0; jj < n; ++jj) {
      const int i = i_first + jj, st = jj % C::kSt;
      if (!(ok = warp_wait(&bars->s_full, jj & 1, abort_flag, p.status))) break;
      // the stage's LSE/Drow (this stage cannot be refilled before this block's P V products)
      if (!(ok = warp_wait(&bars->stat_full[st], (jj / C::kSt) & 1, abort_flag, p.status))) break;
      tc_fence_after();
      const float* stat = sStat + st * 2 * kBT;
      // key kj is visible to query q iff kj < prefix or q >= kj - diag (causal); the whole block is
      // visible iff its first query already sees the tile's last key; queries past the sequence end
      // have P = 0 through their +inf LSE
      const bool masked = p.causal && (i * kBT + diag < n0 + kBT - 1);
      const int q_lo = (kj < p.prefix) ? -kBT : kj - diag - i * kBT;  // columns c < q_lo are masked
      // the half's 64 query columns in 16-column chunks; chunk c+1 is loaded while chunk c is computed
      const uint32_t cs = lane_base + kColS + 64 * hc, cd = lane_base + kColDP + 128 * (jj % kBufs) + 64 * hc;
      uint32_t sb[2][16], db[2][16];
      tmem_ld16_async(cs, sb[0]);
      tmem_ld16_async(cd, db[0]);
      tmem_wait_ld_pair(sb[0], db[0]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int cur = c & 1;
        if (c + 1 < 4) {
          tmem_ld16_async(cs + 16 * (c + 1), sb[cur ^ 1]);
          tmem_ld16_async(cd + 16 * (c + 1), db[cur ^ 1]);
        }
        uint32_t pk[8], dk[8];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int c0 = 64 * hc + 16 * c + 4 * q4;  // query column in the block
          // the four queries' -LSE log2e and -Drow as pairs
          const ulonglong2 nl = *reinterpret_cast<const ulonglong2*>(stat + c0);
          const ulonglong2 nd = *reinterpret_cast<const ulonglong2*>(stat + kBT + c0);
          const uint64_t nlv[2] = {nl.x, nl.y}, ndv[2] = {nd.x, nd.y};
          float pv[4], dsv[4];
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            // P = 2^(s scale log2e - LSE log2e), dS = P (dP - Drow), two queries per instruction
            float x0, x1;
            f2_split(f2_fma(f2_of(&sb[cur][4 * q4 + e]), sl2x2, nlv[e / 2]), x0, x1);
            pv[e] = ex2(x0);
            pv[e + 1] = ex2(x1);
            if (masked) {
              if (c0 + e < q_lo) pv[e] = 0.f;
              if (c0 + e + 1 < q_lo) pv[e + 1] = 0.f;
            }
            f2_split(f2_mul(f2(pv[e], pv[e + 1]), f2_add(f2_of(&db[cur][4 * q4 + e]), ndv[e / 2])), dsv[e], dsv[e + 1]);
          }
          pk[2 * q4] = pack2<kFp16>(pv[0], pv[1]);
          pk[2 * q4 + 1] = pack2<kFp16>(pv[2], pv[3]);
          dk[2 * q4] = pack2<kFp16>(dsv[0], dsv[1]);
          dk[2 * q4 + 1] = pack2<kFp16>(dsv[2], dsv[3]);
        }
        // dS^T and P^T over the dP^T columns of this chunk, which this warp has read (ds_col_dkdv)
        tmem_st8(cd + 16 * c, dk);
        tmem_st8(cd + 16 * c + 8, pk);
        if (c + 1 < 4) {
          tmem_wait_ld_pair(sb[cur ^ 1], db[cur ^ 1]);
          if (c == 2) {  // all of this warp's S^T columns are in registers
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars->s_read);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->p_full);
    }
    if (ok) ok = warp_wait(&bars->o_done, 0, abort_flag, p.status);
    if (ok) {
      tc_fence_after();
      const size_t row = (static_cast<size_t>(u.k_row0 + min(kj, Lk - 1)) * p.H + h) * D;
      constexpr uint32_t col_acc = C::template kColAcc<true>;
      // warps of column half 0 store dV, those of half 1 dK
      if (hc == 0) store_grad_row<D, kFp16, kOutF32>(p.g1, row, lane_base + col_acc, 1.f, kj < Lk, p.status, p.g1_n);
      else store_grad_row<D, kFp16, kOutF32>(p.g0, row, lane_base + col_acc + D, p.scale, kj < Lk, p.status, p.g0_n);
    }
  }
  bwd_teardown(bars, warp, tbase);
}

template <int D, bool kFp16, bool kOutF32>
int launch_bwd_t(const BackwardArgs& a, const CUtensorMap (&m)[4], BwdParams p, cudaStream_t stream) {
  const int smem = BwdCfg<D>::kSmemBytes, smem_q = BwdCfg<D>::kDqSmemBytes;
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
    cudaError_t e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_q);
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
  kq<<<static_cast<unsigned>(pq.num_tiles * (varlen ? 1 : a.B) * a.H), kThreads, smem_q, stream>>>(m[0], m[1], m[2], m[3], pq);
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
