// fa_decode_sm100.cu -- single-token decode: split-KV partial attention + LSE combine.
//
// Decode attends one query per (batch, head) to the whole KV cache.  The work is a matrix-vector
// product (one multiply-add per loaded K or V element), bound by HBM bandwidth, so it runs on CUDA
// cores with wide streaming loads rather than on the tensor cores ("Was FlashAttention bei
// Transformer-Inference verändert": prefill and single-token decode expose different parallelism).
//
// Kernel 1 (split): CTA = (head, split, batch).  The split's keys are processed in chunks of
//   kChunk: all scores of a chunk go to shared memory, then the chunk max updates the running max,
//   the accumulator is rescaled and the value rows are accumulated with p = 2^(s - m).  The CTA
//   writes the split's normalised partial output o_s and its natural-log LSE lse_s (fp32).
// Kernel 2 (combine): one warp per (batch, head) merges the splits: M = max_s lse_s,
//   w_s = exp(lse_s - M), O = sum_s w_s o_s / sum_s w_s, LSE = M + ln sum_s w_s -- the pairwise
//   merge of group statistics of "轻松读懂FlashAttention 上" ("Softmax求解重构") applied to all
//   splits at once.
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

constexpr int kDecThreads = 128;
constexpr int kChunk = 256;
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
  int B, H, Nk, S;
  float scale_log2;
};

template <bool kFp16>
__device__ __forceinline__ void load8_stream(const void* ptr, float (&f)[8]) {
  const uint4 u = __ldcs(reinterpret_cast<const uint4*>(ptr));
  const float2 a = unpack2<kFp16>(u.x), b = unpack2<kFp16>(u.y);
  const float2 c = unpack2<kFp16>(u.z), d = unpack2<kFp16>(u.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <bool kFp16, int D>
__global__ void __launch_bounds__(kDecThreads) decode_split_kernel(const DecParams p) {
  using T = uint16_t;
  constexpr int LPK = D / 8;       // lanes sharing one key row (16-byte slice each)
  constexpr int KPW = 32 / LPK;    // keys per warp per step
  constexpr int KPB = KPW * 4;     // keys per CTA per step
  constexpr int UNR = 4;           // independent row loads in flight per thread

  const int h = blockIdx.x, s = blockIdx.y, b = blockIdx.z;
  const int per = (p.Nk + p.S - 1) / p.S;
  const int lo = min(p.Nk, s * per);
  const int hi = min(p.Nk, lo + per);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = lane % LPK, kk = lane / LPK;

  __shared__ float sc[kChunk];
  __shared__ float red_m[4];
  __shared__ float red_l[4];
  __shared__ float red_acc[4][D];

  const size_t bh = static_cast<size_t>(b) * p.H + h;
  float* wo = p.ws_o + (bh * p.S + s) * D;
  float* wl = p.ws_lse + bh * p.S + s;
  if (lo >= hi) {  // a split past the end of the cache: empty partial
    for (int d = tid; d < D; d += kDecThreads) wo[d] = 0.f;
    if (tid == 0) *wl = -INFINITY;
    return;
  }

  float qf[8];
  load8_stream<kFp16>(static_cast<const T*>(p.q) + bh * D + c * 8, qf);
#pragma unroll
  for (int e = 0; e < 8; ++e) qf[e] *= p.scale_log2;  // scores come out in log2 units

  const size_t rs = static_cast<size_t>(p.H) * D;  // elements between consecutive cache rows
  const T* kb = static_cast<const T*>(p.k) + static_cast<size_t>(b) * p.Nk * rs + h * D + c * 8;
  const T* vb = static_cast<const T*>(p.v) + static_cast<size_t>(b) * p.Nk * rs + h * D + c * 8;

  float m_run = -INFINITY, l_part = 0.f;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;

  for (int c0 = lo; c0 < hi; c0 += kChunk) {
    const int n = min(kChunk, hi - c0);
    // scores of this chunk
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
        float d = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) d = fmaf(qf[e], kf[u][e], d);
#pragma unroll
        for (int o = LPK / 2; o >= 1; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        const int j = j0 + u * KPB + kk;
        if (j < n && c == 0) sc[j] = d;
      }
    }
    __syncthreads();
    float mx = -INFINITY;
    for (int j = tid; j < n; j += kDecThreads) mx = fmaxf(mx, sc[j]);
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red_m[warp] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(red_m[0], red_m[1]), fmaxf(red_m[2], red_m[3]));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = ex2(m_run - m_new);  // 0 on the first chunk
    l_part *= alpha;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= alpha;
    // values of this chunk
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
        const float pj = (j < n) ? ex2(sc[j] - m_new) : 0.f;
        if (c == 0) l_part += pj;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(pj, vf[u][e], acc[e]);
      }
    }
    m_run = m_new;
    __syncthreads();  // sc and red_m are reused by the next chunk
  }

  // reduce over the key slots of a warp (lanes with the same dim slice), then over warps
#pragma unroll
  for (int o = LPK; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    l_part += __shfl_xor_sync(0xffffffffu, l_part, o);
  }
  if (kk == 0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red_acc[warp][c * 8 + e] = acc[e];
  }
  if (lane == 0) red_l[warp] = l_part;
  __syncthreads();
  const float l = red_l[0] + red_l[1] + red_l[2] + red_l[3];
  const float inv_l = 1.f / l;
  for (int d = tid; d < D; d += kDecThreads)
    wo[d] = (red_acc[0][d] + red_acc[1][d] + red_acc[2][d] + red_acc[3][d]) * inv_l;
  if (tid == 0) *wl = (m_run + lg2(l)) * kLn2;
}

template <bool kFp16, int D, bool kOutF32>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecParams p) {
  constexpr int PER = D / 32;  // output elements per lane
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * 4 + (threadIdx.x >> 5);
  if (bh >= p.B * p.H) return;
  const float* wl = p.ws_lse + static_cast<size_t>(bh) * p.S;
  const float* wo = p.ws_o + static_cast<size_t>(bh) * p.S * D;

  float mx = -INFINITY;
  for (int s = lane; s < p.S; s += 32) mx = fmaxf(mx, wl[s] * kLog2e);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float wsum = 0.f;
  for (int s = lane; s < p.S; s += 32) wsum += ex2(wl[s] * kLog2e - mx);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, o);
  const float inv = 1.f / wsum;

  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  for (int s = 0; s < p.S; ++s) {
    const float w = ex2(wl[s] * kLog2e - mx) * inv;
    const float* row = wo + static_cast<size_t>(s) * D + lane * PER;
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
  if (lane == 0) p.lse[bh] = (mx + lg2(wsum)) * kLn2;
}

template <bool kFp16, int D>
int launch_decode_t(const DecodeArgs& a, const DecParams& p, cudaStream_t stream) {
  decode_split_kernel<kFp16, D><<<dim3(a.H, a.S, a.B), kDecThreads, 0, stream>>>(p);
  const int nbh = a.B * a.H;
  const dim3 cgrid((nbh + 3) / 4);
  if (a.o_fp32)
    decode_combine_kernel<kFp16, D, true><<<cgrid, 128, 0, stream>>>(p);
  else
    decode_combine_kernel<kFp16, D, false><<<cgrid, 128, 0, stream>>>(p);
  return static_cast<int>(cudaGetLastError());
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  DecParams p;
  p.q = a.q; p.k = a.k; p.v = a.v; p.o = a.o; p.lse = a.lse;
  p.ws_o = a.ws_o; p.ws_lse = a.ws_lse;
  p.B = a.B; p.H = a.H; p.Nk = a.Nk; p.S = a.S;
  p.scale_log2 = a.scale * kLog2e;
  if (a.D == 64) return a.fp16 ? launch_decode_t<true, 64>(a, p, stream) : launch_decode_t<false, 64>(a, p, stream);
  return a.fp16 ? launch_decode_t<true, 128>(a, p, stream) : launch_decode_t<false, 128>(a, p, stream);
}

}  // namespace fa
