// fa_decode_sm100.cu -- single-token decode: split-KV partial attention + LSE combine.
//
// Decode attends one query per (batch, head) to the whole KV cache.  The work is a matrix-vector
// product (one multiply-add per loaded K or V element), bound by HBM bandwidth, so it runs on CUDA
// cores with wide streaming loads rather than on the tensor cores ("Was FlashAttention bei
// Transformer-Inference verändert": prefill and single-token decode expose different parallelism).
//
// Kernel 1 (split): CTA = (group of G query heads sharing one KV head, split, batch).  The split's
//   keys (of the batch item's valid cache length) are processed in chunks of kChunk: each K row
//   slice is loaded once and dotted with the G queries, all scores of a chunk go to shared memory,
//   then each head's chunk max updates its running max, its accumulator is rescaled and the value
//   rows (again loaded once for the G heads) are accumulated with p = 2^(s - m).  The CTA writes
//   each head's normalised partial output o_s and its natural-log LSE lse_s (fp32).  A split with
//   no keys writes o_s = 0, lse_s = -inf.
// Kernel 2 (combine): one warp per (batch, head) merges the splits: M = max_s lse_s,
//   w_s = exp(lse_s - M), O = sum_s w_s o_s / sum_s w_s, LSE = M + ln sum_s w_s -- the pairwise
//   merge of group statistics of "轻松读懂FlashAttention 上" ("Softmax求解重构") applied to all
//   splits at once; a query without any key (valid length 0) gets O = 0, LSE = -inf.
//
// Paged cache: K and V are pools of pages of 2^page_shift rows and a block table lists each batch
// item's pages in key order, so key j of batch item b is row table[b][j >> page_shift] *
// page_size + (j & (page_size - 1)) of the pool.  Both kernels read rows through that mapping;
// split ranges are then rounded to whole 64-key tiles, so no tile of the tensor-core kernel crosses
// a page, and each CTA checks the table entries of its range before it reads anything.
//
// Key-sharded decode (a cache too long for one GPU cut along the key axis): kernel 1 runs on one
// shard, seeing the shard's rows as keys [key_offset, key_offset + Nk) of the whole cache, and
// kernel 2 leaves that shard's fp32 (O, LSE).  The same combine kernel, with other strides, then
// merges the R shards' results gathered from all ranks (launch_decode_merge): the merge is
// associative, so combining splits first and shards second gives the softmax over all keys.
#include <algorithm>
#include <atomic>

#include "fa_internal.h"
#include "fa_prefill_common.cuh"  // bounded waits, TMA map builder
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kDecThreads = 128;
constexpr int kChunk = 256;
// A split covers at least this many keys: shorter caches use fewer splits (the rest exit at once),
// since a CTA's fixed costs (query load, reductions, partial writes) outweigh streaming a few keys.
constexpr int kMinSplitKeys = 512;
constexpr int kStatusPageTable = 12;  // FA_ERR_PAGE_TABLE

struct DecParams {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  float* ws_o;
  float* ws_lse;
  const int* seqlens_k;  // nullable; lengths of the whole cache
  int* status;
  int B, H, Nk, S;  // H: query heads; Nk: cache rows held here
  int Hkv, group;   // KV heads; query heads per KV head (H = Hkv * group)
  int key_offset;   // first key of the whole cache held here
  int Nk_total;     // keys of the whole cache
  float scale_log2;
  // paged cache (table != nullptr): k and v are pools of num_pages pages of 2^page_shift rows;
  // table[b * pages_per_seq + i] is the page holding keys [i << page_shift, (i + 1) << page_shift)
  const int* table;
  int pages_per_seq, page_shift, num_pages;
};

// Pool row of key j (counted from the first row held here) of batch item b: the contiguous cache
// row, or the row the block table maps it to (entries checked beforehand by page_range_ok).  The
// layout is a template parameter of the kernels, so the contiguous ones carry no table code.
template <bool kPaged>
__device__ __forceinline__ size_t key_row(const DecParams& p, int b, int j) {
  if constexpr (!kPaged) {
    return static_cast<size_t>(b) * p.Nk + j;
  } else {
    const int page = __ldg(p.table + static_cast<size_t>(b) * p.pages_per_seq + (j >> p.page_shift));
    return (static_cast<size_t>(page) << p.page_shift) + (j & ((1 << p.page_shift) - 1));
  }
}

// Split range [lo, hi) of keys: at least kMinSplitKeys keys per split; on a paged cache rounded up
// to whole 64-key tiles, so that every tile lies inside one page or covers whole pages.
template <bool kPaged>
__device__ __forceinline__ int split_keys(const DecParams& p, int len) {
  const int per = max((len + p.S - 1) / p.S, kMinSplitKeys);
  return kPaged ? (per + 63) & ~63 : per;
}

// True if every block-table entry covering keys [lo, hi) of batch item b names a pool page.
// Collective over the CTA (every thread must call it); a bad entry is reported as FA_ERR_PAGE_TABLE.
template <bool kPaged>
__device__ __forceinline__ bool page_range_ok(const DecParams& p, int b, int lo, int hi) {
  if (!kPaged || lo >= hi) return true;
  bool bad = false;
  for (int i = (lo >> p.page_shift) + static_cast<int>(threadIdx.x); i <= ((hi - 1) >> p.page_shift);
       i += blockDim.x) {
    const int page = __ldg(p.table + static_cast<size_t>(b) * p.pages_per_seq + i);
    bad |= (page < 0 || page >= p.num_pages);
  }
  bad = __syncthreads_or(bad) != 0;
  if (bad && threadIdx.x == 0) record_status(p.status, kStatusPageTable);
  return !bad;
}

// Elements of the buffers a decode kernel touches with plain loads and stores (debug index checks).
__device__ __forceinline__ long long q_elems(const DecParams& p, int D) { return static_cast<long long>(p.B) * p.H * D; }
__device__ __forceinline__ long long kv_elems(const DecParams& p, int D) {
  const long long rows = p.table ? static_cast<long long>(p.num_pages) << p.page_shift : static_cast<long long>(p.B) * p.Nk;
  return rows * p.Hkv * D;
}
__device__ __forceinline__ long long ws_o_elems(const DecParams& p, int D) {
  return static_cast<long long>(p.B) * p.H * p.S * D;
}
__device__ __forceinline__ long long ws_l_elems(const DecParams& p) { return static_cast<long long>(p.B) * p.H * p.S; }

// Partial results to merge: partial t of output row r (= b * H + h) has its normalised output at
// po + r * o_row + t * o_part (D floats) and its natural-log LSE at pl + r * l_row + t * l_part.
struct CombParams {
  const float* po;
  const float* pl;
  long long o_row, o_part, l_row, l_part;
  int T, rows;
  void* o;
  float* lse;
  long long po_n, pl_n;  // floats readable from po and from pl (bounds of the debug index checks)
  int* status;
};

template <bool kFp16>
__device__ __forceinline__ void load8_stream(const void* ptr, float (&f)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4*>(ptr));
  const float2 a = unpack2<kFp16>(u.x), b = unpack2<kFp16>(u.y);
  const float2 c = unpack2<kFp16>(u.z), d = unpack2<kFp16>(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <bool kFp16, int D, int G, bool kPaged>
__global__ void __launch_bounds__(kDecThreads, (G >= 4 ? 1 : 4)) decode_split_kernel(const DecParams p) {
  using T = uint16_t;
  constexpr int LPK = D / 8;       // lanes sharing one key row (16-byte slice each)
  constexpr int KPW = 32 / LPK;    // keys per warp per step
  constexpr int KPB = KPW * 4;     // keys per CTA per step
  constexpr int UNR = G >= 8 ? 2 : 4;  // independent row loads in flight per thread (registers)

  const int s = blockIdx.y, b = blockIdx.z;
  const int subs = p.group / G;  // CTAs per KV head
  const int hk = blockIdx.x / subs;
  const int hq0 = hk * p.group + (blockIdx.x % subs) * G;  // first of this CTA's G query heads
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = lane % LPK, kk = lane / LPK;

  int len = p.Nk_total;
  if (p.seqlens_k != nullptr) {
    len = __ldg(p.seqlens_k + b);
    if (len < 0 || len > p.Nk_total) {  // reported, and the batch item is treated as having no keys
      if (tid == 0 && s == 0 && blockIdx.x == 0) record_status(p.status, kStatusCuSeqlens);
      len = 0;
    }
  }
  len = min(max(len - p.key_offset, 0), p.Nk);  // valid keys among the rows held here
  const int per = split_keys<kPaged>(p, len);
  const int lo = min(len, s * per);
  int hi = min(len, lo + per);
  if (!page_range_ok<kPaged>(p, b, lo, hi)) hi = lo;  // a bad table entry: the range contributes nothing

  __shared__ float sc[G][kChunk];
  __shared__ float red_m[4][G];
  __shared__ float red_l[4][G];
  __shared__ float red_acc[4][G][D];

  auto ws_o = [&](int g) { return p.ws_o + ((static_cast<size_t>(b) * p.H + hq0 + g) * p.S + s) * D; };
  auto ws_l = [&](int g) { return p.ws_lse + (static_cast<size_t>(b) * p.H + hq0 + g) * p.S + s; };
  if (lo >= hi) {  // a split past the end of the valid cache: empty partials
#pragma unroll
    for (int g = 0; g < G; ++g) {
      for (int d = tid; d < D; d += kDecThreads)
        if (idx_ok(p.status, ws_o(g) + d - p.ws_o, 1, ws_o_elems(p, D))) ws_o(g)[d] = 0.f;
      if (tid == 0 && idx_ok(p.status, ws_l(g) - p.ws_lse, 1, ws_l_elems(p))) *ws_l(g) = -INFINITY;
    }
    return;
  }

  float qf[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const size_t qoff = (static_cast<size_t>(b) * p.H + hq0 + g) * D + c * 8;
    if (idx_ok(p.status, qoff, 8, q_elems(p, D))) {
      load8_stream<kFp16>(static_cast<const T*>(p.q) + qoff, qf[g]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[g][e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[g][e] *= p.scale_log2;  // scores come out in log2 units
  }

  const size_t rs = static_cast<size_t>(p.Hkv) * D;  // elements between consecutive cache rows
  // contiguous: the batch item's rows from here; paged: rows of the pool (through the table)
  const size_t b_off = kPaged ? 0 : static_cast<size_t>(b) * p.Nk * rs;
  const T* kb = static_cast<const T*>(p.k) + b_off + hk * D + c * 8;
  const T* vb = static_cast<const T*>(p.v) + b_off + hk * D + c * 8;
  // Element offset of key c0 + j of the current chunk: an affine function on a contiguous cache (the
  // compiler then keeps all UNR loads in flight); on a paged cache the pool row of every key of the
  // chunk is staged in shared memory once per chunk, so the key loop reads it with one shared load
  // (a table lookup in front of every key load cost two thirds of the bandwidth).
  __shared__ int s_row[kPaged ? kChunk : 1];
  auto row_off = [&](int c0, int j) -> size_t {
    if constexpr (kPaged) return static_cast<size_t>(s_row[j]) * rs;
    else return static_cast<size_t>(c0 + j) * rs;
  };

  float m_run[G], l_part[G], acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m_run[g] = -INFINITY;
    l_part[g] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
  }

  for (int c0 = lo; c0 < hi; c0 += kChunk) {
    const int n = min(kChunk, hi - c0);
    if constexpr (kPaged) {  // pool rows of the chunk's keys (their table entries were checked)
      for (int j = tid; j < n; j += kDecThreads) s_row[j] = static_cast<int>(key_row<true>(p, b, c0 + j));
      __syncthreads();
    }
    // scores of this chunk: each K row slice is loaded once for the G queries
    for (int j0 = warp * KPW; j0 < n; j0 += UNR * KPB) {
      float kf[UNR][8];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int j = j0 + u * KPB + kk;
        const size_t off = (kPaged && j >= n) ? 0 : row_off(c0, j);
        if (j < n && idx_ok(p.status, kb + off - static_cast<const T*>(p.k), 8, kv_elems(p, D))) {
          load8_stream<kFp16>(kb + off, kf[u]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) kf[u][e] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int j = j0 + u * KPB + kk;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float d = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) d = fmaf(qf[g][e], kf[u][e], d);
#pragma unroll
          for (int o = LPK / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
          if (j < n && c == 0) sc[g][j] = d;
        }
      }
    }
    __syncthreads();
    float m_new[G];
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float mx = -INFINITY;
      for (int j = tid; j < n; j += kDecThreads) mx = fmaxf(mx, sc[g][j]);
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (lane == 0) red_m[warp][g] = mx;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mx = fmaxf(fmaxf(red_m[0][g], red_m[1][g]), fmaxf(red_m[2][g], red_m[3][g]));
      m_new[g] = fmaxf(m_run[g], mx);
      const float alpha = ex2(m_run[g] - m_new[g]);  // 0 on the first chunk
      l_part[g] *= alpha;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] *= alpha;
    }
    // values of this chunk, each V row slice loaded once for the G heads
    for (int j0 = warp * KPW; j0 < n; j0 += UNR * KPB) {
      float vf[UNR][8];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int j = j0 + u * KPB + kk;
        const size_t off = (kPaged && j >= n) ? 0 : row_off(c0, j);
        if (j < n && idx_ok(p.status, vb + off - static_cast<const T*>(p.v), 8, kv_elems(p, D))) {
          load8_stream<kFp16>(vb + off, vf[u]);
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) vf[u][e] = 0.f;
        }
      }
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int j = j0 + u * KPB + kk;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pj = (j < n) ? ex2(sc[g][j] - m_new[g]) : 0.f;
          if (c == 0) l_part[g] += pj;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pj, vf[u][e], acc[g][e]);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g) m_run[g] = m_new[g];
    __syncthreads();  // sc and red_m are reused by the next chunk
  }

  // reduce over the key slots of a warp (lanes with the same dim slice), then over warps
#pragma unroll
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int o = LPK; o < 32; o <<= 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);
      l_part[g] += __shfl_xor_sync(0xffffffffu, l_part[g], o);
    }
    if (kk == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) red_acc[warp][g][c * 8 + e] = acc[g][e];
    }
    if (lane == 0) red_l[warp][g] = l_part[g];
  }
  __syncthreads();
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float l = red_l[0][g] + red_l[1][g] + red_l[2][g] + red_l[3][g];
    const float inv_l = 1.f / l;
    float* wo = ws_o(g);
    for (int d = tid; d < D; d += kDecThreads)
      if (idx_ok(p.status, wo + d - p.ws_o, 1, ws_o_elems(p, D)))
        wo[d] = (red_acc[0][g][d] + red_acc[1][g][d] + red_acc[2][g][d] + red_acc[3][g][d]) * inv_l;
    if (tid == 0 && idx_ok(p.status, ws_l(g) - p.ws_lse, 1, ws_l_elems(p))) *ws_l(g) = (m_run[g] + lg2(l)) * kLn2;
  }
}

// ------------------------------------------------------------------------------------------------
// Grouped decode on the tensor cores (G = 2..16 query heads per KV head).
//
// With G query heads sharing each K/V row, the split is a small matrix product: S = Q K^T with Q the
// G x D block of the group's queries, then O += P V.  On CUDA cores that costs G multiply-adds per
// loaded element plus a shuffle reduction per head, which leaves the grouped decode bound by
// instruction issue far below HBM bandwidth.  Here warp-level mma.sync m16n8k16 tiles take both
// products (the G heads are the M rows of a 16-row tile; rows >= G are zero), so a 16-key slice of
// K and V costs 2 * D/8 MMAs and D/4 ldmatrix per warp, and the kernel is bound by HBM again.
// (tcgen05 needs M >= 64 rows and a TMEM round trip per block; with at most 16 live rows the
// register-resident warp MMA is the better fit for this matrix-vector-like product.)
//
// CTA = (G heads of one KV head, split, batch): warp 4 streams 64-key K and V tiles of the split
// through a ring of kMmaStages shared-memory stages with TMA (box 64 columns x 1 head x 64 rows,
// 128-byte swizzle, no multicast); warps 0-3 each take 16 keys of every tile: S from ldmatrix'd K
// and Q fragments held in registers, an online softmax per head row in the log2 domain with lazy
// rescaling (O and l share a running max that is only raised when a block max exceeds it by more
// than 2^8, which keeps P <= 2^8 and is exact after the final division), P repacked in registers as
// the A operand, and O += P V from transposing ldmatrix of V.  The four warps' (m, l, O) are merged
// through shared memory at the end and the split's normalised partial and LSE are written as by
// decode_split_kernel, so the same combine follows.

constexpr int kMmaTileKeys = 64;
constexpr int kMmaThreads = 160;  // 4 MMA warps + 1 TMA warp
constexpr int kMmaProducerWarp = 4;
constexpr float kRescaleLog2 = 8.f;

template <int D>
struct MmaCfg {
  static constexpr int kPanelBytes = kMmaTileKeys * 128;     // 64 rows x 64 columns x 2 bytes
  static constexpr int kTileBytes = kPanelBytes * (D / 64);  // one K (or V) tile
  static constexpr int kStages = (D == 128) ? 3 : 5;         // two CTAs per SM
  static constexpr int kStageBytes = 2 * kTileBytes;         // K then V
  static constexpr int kBarOff = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;    // barriers + alignment slack
};

struct MmaBars {
  uint64_t full[8];
  uint64_t empty[8];
  int abort_flag;
};

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr)
               : "memory");
}

// D[16x8] += A[16x16] * B[16x8], fp32 accumulate; A and B of the same 16-bit type.
template <bool kFp16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (kFp16) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
                 "{%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// Byte offset of 16-bit element (row, col) in a tile of 64-column panels of kMmaTileKeys rows with
// the 128-byte swizzle TMA writes (16-byte chunk index XOR row % 8); col is a multiple of 8.
__device__ __forceinline__ uint32_t swz_off(int row, int col) {
  return static_cast<uint32_t>((col >> 6) * (kMmaTileKeys * 128) + row * 128 +
                               ((((col & 63) >> 3) ^ (row & 7)) << 4));
}

template <bool kFp16, int D, int G, bool kPaged>
__global__ void __launch_bounds__(kMmaThreads, 2)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_v,
                      const DecParams p) {
  using C = MmaCfg<D>;
  static_assert(G >= 2 && G <= 16, "2..16 heads per CTA");
  constexpr bool kHi = G > 8;  // rows 8..15 of the tile carry heads
  constexpr int KS = D / 16;   // k-steps of S = Q K^T
  constexpr int NT = D / 8;    // 8-column tiles of O

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  MmaBars* bars = reinterpret_cast<MmaBars*>(smem + C::kBarOff);

  const int s = blockIdx.y, b = blockIdx.z;
  const int subs = p.group / G;
  const int hk = blockIdx.x / subs;
  const int hq0 = hk * p.group + (blockIdx.x % subs) * G;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  int len = p.Nk_total;
  if (p.seqlens_k != nullptr) {
    len = __ldg(p.seqlens_k + b);
    if (len < 0 || len > p.Nk_total) {
      if (tid == 0 && s == 0 && blockIdx.x == 0) record_status(p.status, kStatusCuSeqlens);
      len = 0;
    }
  }
  len = min(max(len - p.key_offset, 0), p.Nk);
  const int per = split_keys<kPaged>(p, len);
  const int lo = min(len, s * per);
  int hi = min(len, lo + per);
  if (!page_range_ok<kPaged>(p, b, lo, hi)) hi = lo;  // a bad table entry: the range contributes nothing
  auto ws_o = [&](int g) { return p.ws_o + ((static_cast<size_t>(b) * p.H + hq0 + g) * p.S + s) * D; };
  auto ws_l = [&](int g) { return p.ws_lse + (static_cast<size_t>(b) * p.H + hq0 + g) * p.S + s; };
  if (lo >= hi) {  // uniform over the CTA: empty partials
    for (int i = tid; i < G * D; i += kMmaThreads)
      if (idx_ok(p.status, ws_o(i / D) + i % D - p.ws_o, 1, ws_o_elems(p, D))) ws_o(i / D)[i % D] = 0.f;
    if (tid < G && idx_ok(p.status, ws_l(tid) - p.ws_lse, 1, ws_l_elems(p))) *ws_l(tid) = -INFINITY;
    return;
  }
  const int n_tiles = (hi - lo + kMmaTileKeys - 1) / kMmaTileKeys;

  if (tid == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(&bars->full[i], 1);
      mbar_init(&bars->empty[i], 4);
    }
    bars->abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  volatile int* abort_flag = &bars->abort_flag;

  float m_fin[2] = {-INFINITY, -INFINITY}, l_fin[2] = {0.f, 0.f};
  float o[NT][4];

  if (warp == kMmaProducerWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tmap_k);
      tma_prefetch_desc(&tmap_v);
      int issued = 0;
      // a tile is loaded as boxes of `box` rows: one box on a contiguous cache, one box per page on
      // a paged cache with pages shorter than a tile (boxes past the valid keys are not loaded)
      const int box = kPaged ? min(kMmaTileKeys, 1 << p.page_shift) : kMmaTileKeys;
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % C::kStages;
        if (t >= C::kStages && !mbar_wait(&bars->empty[st], ((t / C::kStages) - 1) & 1, abort_flag, p.status))
          break;
        uint8_t* kdst = smem + st * C::kStageBytes;
        const int k0 = lo + t * kMmaTileKeys;
        const int boxes = min(kMmaTileKeys, hi - k0 + box - 1) / box;
        mbar_arrive_expect_tx(&bars->full[st], static_cast<uint32_t>(boxes * box * 128 * (D / 64) * 2));
        for (int i = 0; i < boxes; ++i) {
          const int row = static_cast<int>(key_row<kPaged>(p, b, k0 + i * box));
#pragma unroll
          for (int pn = 0; pn < D / 64; ++pn) {
            tma_load_3d(&tmap_k, &bars->full[st], kdst + pn * C::kPanelBytes + i * box * 128, pn * 64, hk, row);
            tma_load_3d(&tmap_v, &bars->full[st], kdst + C::kTileBytes + pn * C::kPanelBytes + i * box * 128, pn * 64,
                        hk, row);
          }
        }
        issued = t + 1;
      }
      if (*abort_flag) {  // let the copies already issued land before the stages are reused or freed
        for (int t = max(0, issued - C::kStages); t < issued; ++t)
          drain_wait(&bars->full[t % C::kStages], (t / C::kStages) & 1);
      }
    }
  } else {
    const int g = lane >> 2, tg = lane & 3;
    // Q fragments (A operand, rows = heads, scaled later): a0 (g, 2tg..), a1 (g+8, 2tg..),
    // a2 (g, 2tg+8..), a3 (g+8, 2tg+8..) of each 16-column step
    uint32_t qa[KS][4];
    {
      const uint32_t* q32 = static_cast<const uint32_t*>(p.q);
      const size_t qrow = (static_cast<size_t>(b) * p.H + hq0) * D;
      const bool q_in = idx_ok(p.status, qrow, static_cast<long long>(G) * D, q_elems(p, D));
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const int c = ks * 16 + 2 * tg;
        qa[ks][0] = (q_in && g < G) ? __ldg(q32 + (qrow + static_cast<size_t>(g) * D + c) / 2) : 0u;
        qa[ks][2] = (q_in && g < G) ? __ldg(q32 + (qrow + static_cast<size_t>(g) * D + c + 8) / 2) : 0u;
        qa[ks][1] = (q_in && kHi && g + 8 < G) ? __ldg(q32 + (qrow + static_cast<size_t>(g + 8) * D + c) / 2) : 0u;
        qa[ks][3] = (q_in && kHi && g + 8 < G) ? __ldg(q32 + (qrow + static_cast<size_t>(g + 8) * D + c + 8) / 2) : 0u;
      }
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    const float sl2 = p.scale_log2;
    const int mi = lane >> 3;  // which 8x8 matrix this lane addresses in ldmatrix.x4

    for (int t = 0; t < n_tiles; ++t) {
      const int st = t % C::kStages;
      if (!warp_wait(&bars->full[st], (t / C::kStages) & 1, abort_flag, p.status)) break;
      const uint32_t kb = smem_addr(smem + st * C::kStageBytes);
      const uint32_t vb = kb + C::kTileBytes;

      // S = Q K^T for this warp's 16 keys: n-tile 0 = keys 0..7, n-tile 1 = keys 8..15
      float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      {
        const int krow = warp * 16 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(kb + swz_off(krow, ks * 16 + (mi & 1) * 8), b0, b1, b2, b3);
          mma16816<kFp16>(sc[0], qa[ks], b0, b1);
          mma16816<kFp16>(sc[1], qa[ks], b2, b3);
        }
      }
      // keys of this thread: n-tile n, element e -> key warp*16 + 8n + 2tg + (e & 1); e < 2 row g,
      // e >= 2 row g + 8
      const int key0 = lo + t * kMmaTileKeys + warp * 16 + 2 * tg;
      const bool tail = (lo + (t + 1) * kMmaTileKeys > hi);
      if (tail) {
        // rows of the last tile past the valid keys hold whatever the cache (or a stale stage) holds
        // there; their P is 0, but 0 * NaN would still reach O, so this warp's V rows there are zeroed
        const int first_dead = hi - (lo + t * kMmaTileKeys + warp * 16);  // of this warp's 16 rows
        for (int i = lane; i < 16 * 8 * (D / 64); i += 32) {
          const int r = i / (8 * (D / 64)), pn = (i / 8) % (D / 64), ch = i % 8;
          if (r >= first_dead) {
            const uint32_t a = vb + pn * C::kPanelBytes + (warp * 16 + r) * 128 + ch * 16;
            asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(a), "r"(0u) : "memory");
          }
        }
        __syncwarp();
      }
      uint32_t pa[4];
#pragma unroll
      for (int r = 0; r < (kHi ? 2 : 1); ++r) {
        float x[4];
#pragma unroll
        for (int n = 0; n < 2; ++n) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            float v = sc[n][2 * r + e] * sl2;
            if (tail && key0 + 8 * n + e >= hi) v = -INFINITY;
            x[2 * n + e] = v;
          }
        }
        float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        if (mx > m_run[r] + kRescaleLog2 || (m_run[r] == -INFINITY && mx > -INFINITY)) {
          const float alpha = ex2(m_run[r] - mx);  // 0 while nothing was accumulated
          l_run[r] *= alpha;
#pragma unroll
          for (int j = 0; j < NT; ++j) {
            o[j][2 * r] *= alpha;
            o[j][2 * r + 1] *= alpha;
          }
          m_run[r] = mx;
        }
        float pv[4];
        if (m_run[r] == -INFINITY) {
          pv[0] = pv[1] = pv[2] = pv[3] = 0.f;
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) pv[i] = ex2(x[i] - m_run[r]);
        }
        l_run[r] += (pv[0] + pv[1]) + (pv[2] + pv[3]);
        // A operand of P V: a0/a2 hold row g (keys 2tg.. of n-tiles 0/1), a1/a3 row g + 8
        pa[r] = pack2<kFp16>(pv[0], pv[1]);
        pa[2 + r] = pack2<kFp16>(pv[2], pv[3]);
      }
      if constexpr (!kHi) {
        pa[1] = 0u;
        pa[3] = 0u;
      }
      // O += P V: ldmatrix.trans gives the B fragments of two 8-column tiles per call
      {
        const int vrow = warp * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int dt = 0; dt < NT / 2; ++dt) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vb + swz_off(vrow, dt * 16 + (mi >> 1) * 8), b0, b1, b2, b3);
          mma16816<kFp16>(o[2 * dt], pa, b0, b1);
          mma16816<kFp16>(o[2 * dt + 1], pa, b2, b3);
        }
      }
      // the zeroing stores above come before the next asynchronous (TMA) write into the stage
      if (tail) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->empty[st]);
    }
    // row sums over the quad (each lane summed its own keys)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
      l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
      m_fin[r] = m_run[r];
      l_fin[r] = l_run[r];
    }
  }
  __syncthreads();  // every stage consumed (or drained): the ring is free for the merge
  const bool ok = (*abort_flag == 0);

  // merge of the four MMA warps: red_o[w][h][d], red_m[w][h], red_l[w][h] over the stage memory
  float* red_o = reinterpret_cast<float*>(smem);
  float* red_m = red_o + 4 * G * D;
  float* red_l = red_m + 4 * G;
  if (ok && warp < 4) {
    const int g = lane >> 2, tg = lane & 3;
#pragma unroll
    for (int r = 0; r < (kHi ? 2 : 1); ++r) {
      const int h = g + 8 * r;
      if (h < G) {
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          red_o[(warp * G + h) * D + 8 * j + 2 * tg] = o[j][2 * r];
          red_o[(warp * G + h) * D + 8 * j + 2 * tg + 1] = o[j][2 * r + 1];
        }
        if (tg == 0) {
          red_m[warp * G + h] = m_fin[r];
          red_l[warp * G + h] = l_fin[r];
        }
      }
    }
  }
  __syncthreads();
  if (!ok) return;
  for (int i = tid; i < G * D; i += kMmaThreads) {
    const int h = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, red_m[w * G + h]);
    float l = 0.f, acc = 0.f;
    if (M > -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float e = ex2(red_m[w * G + h] - M);
        l += e * red_l[w * G + h];
        acc += e * red_o[(w * G + h) * D + d];
      }
    }
    if (idx_ok(p.status, ws_o(h) + d - p.ws_o, 1, ws_o_elems(p, D))) ws_o(h)[d] = (M > -INFINITY) ? acc / l : 0.f;
    if (d == 0 && idx_ok(p.status, ws_l(h) - p.ws_lse, 1, ws_l_elems(p)))
      *ws_l(h) = (M > -INFINITY) ? (M + lg2(l)) * kLn2 : -INFINITY;
  }
}

template <bool kFp16, int D, bool kOutF32>
__global__ void __launch_bounds__(128) decode_combine_kernel(const CombParams p) {
  constexpr int PER = D / 32;  // output elements per lane
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (bh >= p.rows) return;
  const float* wl = p.pl + static_cast<long long>(bh) * p.l_row;
  const float* wo = p.po + static_cast<long long>(bh) * p.o_row;
#ifdef FA_DEBUG
  // every partial this row reads must lie inside the partial buffers (warp-uniform)
  if (!idx_ok(p.status, wl - p.pl, static_cast<long long>(p.T - 1) * p.l_part + 1, p.pl_n) ||
      !idx_ok(p.status, wo - p.po, static_cast<long long>(p.T - 1) * p.o_part + D, p.po_n) ||
      !idx_ok(p.status, static_cast<long long>(bh) * D, D, static_cast<long long>(p.rows) * D))
    return;
#endif

  float mx = -INFINITY;
  for (int t = lane; t < p.T; t += 32) mx = fmaxf(mx, wl[t * p.l_part] * kLog2e);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  const bool empty = (mx == -INFINITY);  // no partial saw a key (warp-uniform)
  float wsum = 0.f;
  for (int t = lane; t < p.T; t += 32) wsum += ex2(wl[t * p.l_part] * kLog2e - mx);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  const float inv = empty ? 0.f : 1.f / wsum;

  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (int t = 0; t < p.T && !empty; ++t) {
    const float w = ex2(wl[t * p.l_part] * kLog2e - mx) * inv;
    const float* row = wo + t * p.o_part + lane * PER;
    if constexpr (PER == 4) {
      const float4 x = *reinterpret_cast<const float4*>(row);
      acc[0] = fmaf(w, x.x, acc[0]); acc[1] = fmaf(w, x.y, acc[1]);
      acc[2] = fmaf(w, x.z, acc[2]); acc[3] = fmaf(w, x.w, acc[3]);
    } else {
      const float2 x = *reinterpret_cast<const float2*>(row);
      acc[0] = fmaf(w, x.x, acc[0]); acc[1] = fmaf(w, x.y, acc[1]);
    }
  }
  const size_t obase = static_cast<size_t>(bh) * D + lane * PER;
  if constexpr (kOutF32) {
    float* out = static_cast<float*>(p.o) + obase;
    if constexpr (PER == 4) {
      *reinterpret_cast<float4*>(out) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    } else {
      *reinterpret_cast<float2*>(out) = make_float2(acc[0], acc[1]);
    }
  } else {
    uint32_t* out = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(p.o) + obase);
    if constexpr (PER == 4) {
      *reinterpret_cast<uint2*>(out) = make_uint2(pack2<kFp16>(acc[0], acc[1]), pack2<kFp16>(acc[2], acc[3]));
    } else {
      *out = pack2<kFp16>(acc[0], acc[1]);
    }
  }
  if (lane == 0) p.lse[bh] = empty ? -INFINITY : (mx + lg2(wsum)) * kLn2;
}

template <bool kFp16, int D, int G>
void launch_split(const DecodeArgs& a, const DecParams& p, cudaStream_t stream) {
  const dim3 grid(p.Hkv * (p.group / G), a.S, a.B);
  if (p.table)
    decode_split_kernel<kFp16, D, G, true><<<grid, kDecThreads, 0, stream>>>(p);
  else
    decode_split_kernel<kFp16, D, G, false><<<grid, kDecThreads, 0, stream>>>(p);
}

template <bool kFp16, int D>
void launch_combine(const CombParams& c, bool o_fp32, cudaStream_t stream) {
  const dim3 cgrid((c.rows + 3) / 4);
  if (o_fp32)
    decode_combine_kernel<kFp16, D, true><<<cgrid, 128, 0, stream>>>(c);
  else
    decode_combine_kernel<kFp16, D, false><<<cgrid, 128, 0, stream>>>(c);
}

template <bool kFp16, int D, int G>
int launch_mma(const DecodeArgs& a, const DecParams& p, cudaStream_t stream) {
  CUtensorMap mk, mv;
  const int rows = p.table ? (p.num_pages << p.page_shift) : a.B * a.Nk;
  const int box = p.table ? std::min(kMmaTileKeys, 1 << p.page_shift) : kMmaTileKeys;  // as the producer loads
  if (!make_tma_map(&mk, a.k, rows, p.Hkv, D, kFp16, box) || !make_tma_map(&mv, a.v, rows, p.Hkv, D, kFp16, box))
    return static_cast<int>(cudaErrorInvalidValue);
  auto kern = p.table ? decode_mma_kernel<kFp16, D, G, true> : decode_mma_kernel<kFp16, D, G, false>;
  // the shared-memory opt-in is a per-device (per-context) attribute of the function: set it once
  // (for both layouts' instantiations)
  static PerContext<int> configured;
  int unused = 0;
  const int ce = configured.get(&unused, [&](int*) {
    for (auto f : {decode_mma_kernel<kFp16, D, G, false>, decode_mma_kernel<kFp16, D, G, true>}) {
      const cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, MmaCfg<D>::kSmemBytes);
      if (e != cudaSuccess) return static_cast<int>(e);
    }
    return 0;
  });
  if (ce != 0) return ce;
  kern<<<dim3(p.Hkv * (p.group / G), a.S, a.B), kMmaThreads, MmaCfg<D>::kSmemBytes, stream>>>(mk, mv, p);
  return 0;
}

template <bool kFp16, int D>
int launch_decode_t(const DecodeArgs& a, const DecParams& p, cudaStream_t stream) {
  // Grouped heads: the tensor-core kernel with G = the largest of 16, 8, 4, 2 dividing the group
  // (the TMA maps index rows with 32-bit coordinates); one head per KV head: the CUDA-core kernel.
  const long long pool_rows = p.table ? static_cast<long long>(p.num_pages) << p.page_shift : static_cast<long long>(a.B) * a.Nk;
  const bool tma_rows_ok = pool_rows < (1LL << 31);
  int e = 0;
  if (tma_rows_ok && p.group % 16 == 0) e = launch_mma<kFp16, D, 16>(a, p, stream);
  else if (tma_rows_ok && p.group % 8 == 0) e = launch_mma<kFp16, D, 8>(a, p, stream);
  else if (tma_rows_ok && p.group % 4 == 0) e = launch_mma<kFp16, D, 4>(a, p, stream);
  else if (tma_rows_ok && p.group % 2 == 0) e = launch_mma<kFp16, D, 2>(a, p, stream);
  else if (p.group % 8 == 0) launch_split<kFp16, D, 8>(a, p, stream);
  else if (p.group % 4 == 0) launch_split<kFp16, D, 4>(a, p, stream);
  else if (p.group % 2 == 0) launch_split<kFp16, D, 2>(a, p, stream);
  else launch_split<kFp16, D, 1>(a, p, stream);
  if (e != 0) return e;
  CombParams c;
  c.po = p.ws_o;
  c.pl = p.ws_lse;
  c.o_row = static_cast<long long>(p.S) * D;
  c.o_part = D;
  c.l_row = p.S;
  c.l_part = 1;
  c.T = p.S;
  c.rows = a.B * a.H;
  c.o = p.o;
  c.lse = p.lse;
  c.po_n = static_cast<long long>(a.B) * a.H * p.S * D;
  c.pl_n = static_cast<long long>(a.B) * a.H * p.S;
  c.status = p.status;
  launch_combine<kFp16, D>(c, a.o_fp32, stream);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  DecParams p;
  p.q = a.q; p.k = a.k; p.v = a.v; p.o = a.o; p.lse = a.lse;
  p.ws_o = a.ws_o; p.ws_lse = a.ws_lse;
  p.seqlens_k = a.seqlens_k;
  p.status = a.status;
  p.B = a.B; p.H = a.H; p.Nk = a.Nk; p.S = a.S;
  p.Hkv = a.Hkv > 0 ? a.Hkv : a.H;
  p.group = a.H / p.Hkv;
  p.key_offset = a.key_offset;
  p.Nk_total = a.Nk_total > 0 ? a.Nk_total : a.Nk;
  p.scale_log2 = a.scale * kLog2e;
  p.table = a.block_table;
  p.pages_per_seq = a.pages_per_seq;
  p.page_shift = 0;
  while (a.block_table && (1 << p.page_shift) < a.page_size) ++p.page_shift;
  p.num_pages = a.num_pages;
  if (a.D == 64) return a.fp16 ? launch_decode_t<true, 64>(a, p, stream) : launch_decode_t<false, 64>(a, p, stream);
  return a.fp16 ? launch_decode_t<true, 128>(a, p, stream) : launch_decode_t<false, 128>(a, p, stream);
}

int launch_decode_merge(const MergeArgs& a, cudaStream_t stream) {
  CombParams c;
  const long long rows = static_cast<long long>(a.B) * a.H;
  c.po = a.parts;
  c.pl = a.parts + rows * a.D;
  c.o_row = a.D;
  c.o_part = a.part_floats;
  c.l_row = 1;
  c.l_part = a.part_floats;
  c.T = a.R;
  c.rows = static_cast<int>(rows);
  c.o = a.o;
  c.lse = a.lse;
  c.po_n = static_cast<long long>(a.R) * a.part_floats;
  c.pl_n = c.po_n - rows * a.D;
  c.status = a.status;
  if (a.D == 64) {
    if (a.o_fp16) launch_combine<true, 64>(c, a.o_fp32, stream);
    else launch_combine<false, 64>(c, a.o_fp32, stream);
  } else {
    if (a.o_fp16) launch_combine<true, 128>(c, a.o_fp32, stream);
    else launch_combine<false, 128>(c, a.o_fp32, stream);
  }
  return static_cast<int>(cudaGetLastError());
}

}  // namespace fa
