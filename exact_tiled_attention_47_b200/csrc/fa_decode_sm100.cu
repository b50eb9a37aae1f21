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
// Key-sharded decode (a cache too long for one GPU cut along the key axis): kernel 1 runs on one
// shard, seeing the shard's rows as keys [key_offset, key_offset + Nk) of the whole cache, and
// kernel 2 leaves that shard's fp32 (O, LSE).  The same combine kernel, with other strides, then
// merges the R shards' results gathered from all ranks (launch_decode_merge): the merge is
// associative, so combining splits first and shards second gives the softmax over all keys.
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kDecThreads = 128;
constexpr int kChunk = 256;
// A split covers at least this many keys: shorter caches use fewer splits (the rest exit at once),
// since a CTA's fixed costs (query load, reductions, partial writes) outweigh streaming a few keys.
constexpr int kMinSplitKeys = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

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
};

// Partial results to merge: partial t of output row r (= b * H + h) has its normalised output at
// po + r * o_row + t * o_part (D floats) and its natural-log LSE at pl + r * l_row + t * l_part.
struct CombParams {
  const float* po;
  const float* pl;
  long long o_row, o_part, l_row, l_part;
  int T, rows;
  void* o;
  float* lse;
};

template <bool kFp16>
__device__ __forceinline__ void load8_stream(const void* ptr, float (&f)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4*>(ptr));
  const float2 a = unpack2<kFp16>(u.x), b = unpack2<kFp16>(u.y);
  const float2 c = unpack2<kFp16>(u.z), d = unpack2<kFp16>(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <bool kFp16, int D, int G>
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
  const int per = max((len + p.S - 1) / p.S, kMinSplitKeys);
  const int lo = min(len, s * per);
  const int hi = min(len, lo + per);

  __shared__ float sc[G][kChunk];
  __shared__ float red_m[4][G];
  __shared__ float red_l[4][G];
  __shared__ float red_acc[4][G][D];

  auto ws_o = [&](int g) { return p.ws_o + ((static_cast<size_t>(b) * p.H + hq0 + g) * p.S + s) * D; };
  auto ws_l = [&](int g) { return p.ws_lse + (static_cast<size_t>(b) * p.H + hq0 + g) * p.S + s; };
  if (lo >= hi) {  // a split past the end of the valid cache: empty partials
#pragma unroll
    for (int g = 0; g < G; ++g) {
      for (int d = tid; d < D; d += kDecThreads) ws_o(g)[d] = 0.f;
      if (tid == 0) *ws_l(g) = -INFINITY;
    }
    return;
  }

  float qf[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    load8_stream<kFp16>(static_cast<const T*>(p.q) + (static_cast<size_t>(b) * p.H + hq0 + g) * D + c * 8, qf[g]);
#pragma unroll
    for (int e = 0; e < 8; ++e) qf[g][e] *= p.scale_log2;  // scores come out in log2 units
  }

  const size_t rs = static_cast<size_t>(p.Hkv) * D;  // elements between consecutive cache rows
  const T* kb = static_cast<const T*>(p.k) + static_cast<size_t>(b) * p.Nk * rs + hk * D + c * 8;
  const T* vb = static_cast<const T*>(p.v) + static_cast<size_t>(b) * p.Nk * rs + hk * D + c * 8;

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
    // scores of this chunk: each K row slice is loaded once for the G queries
    for (int j0 = warp * KPW; j0 < n; j0 += UNR * KPB) {
      float kf[UNR][8];
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        const int j = j0 + u * KPB + kk;
        if (j < n) {
          load8_stream<kFp16>(kb + static_cast<size_t>(c0 + j) * rs, kf[u]);
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
        if (j < n) {
          load8_stream<kFp16>(vb + static_cast<size_t>(c0 + j) * rs, vf[u]);
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
      wo[d] = (red_acc[0][g][d] + red_acc[1][g][d] + red_acc[2][g][d] + red_acc[3][g][d]) * inv_l;
    if (tid == 0) *ws_l(g) = (m_run[g] + lg2(l)) * kLn2;
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
  decode_split_kernel<kFp16, D, G><<<dim3(p.Hkv * (p.group / G), a.S, a.B), kDecThreads, 0, stream>>>(p);
}

template <bool kFp16, int D>
void launch_combine(const CombParams& c, bool o_fp32, cudaStream_t stream) {
  const dim3 cgrid((c.rows + 3) / 4);
  if (o_fp32)
    decode_combine_kernel<kFp16, D, true><<<cgrid, 128, 0, stream>>>(c);
  else
    decode_combine_kernel<kFp16, D, false><<<cgrid, 128, 0, stream>>>(c);
}

template <bool kFp16, int D>
int launch_decode_t(const DecodeArgs& a, const DecParams& p, cudaStream_t stream) {
  // query heads per CTA: the largest of 8, 4, 2, 1 that divides the group
  if (p.group % 8 == 0) launch_split<kFp16, D, 8>(a, p, stream);
  else if (p.group % 4 == 0) launch_split<kFp16, D, 4>(a, p, stream);
  else if (p.group % 2 == 0) launch_split<kFp16, D, 2>(a, p, stream);
  else launch_split<kFp16, D, 1>(a, p, stream);
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
