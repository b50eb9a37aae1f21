// fa_api.cu -- the extern "C" boundary of libfa_sm100.so (declared in include/fa.h).
//
// Argument checks run on the host before anything is enqueued, in a fixed order: null pointers,
// element types, head dimension, shapes and scale, alignment, workspace, then the device.  Kernels
// report failures they detect (a bounded wait that ran out, an inconsistent cu_seqlens) through a
// per-device status word read by fa_device_status().
#include <cuda.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "fa_internal.h"

namespace fa {
namespace {

__device__ int g_status_word = 0;

constexpr int kMaxDevices = 64;
int g_device_ok[kMaxDevices];      // 0 unknown, 1 sm_100, -1 other
std::mutex g_mu;
PerContext<int*> g_status_ptr;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

}  // namespace

unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
    cudaGetLastError();
  });
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// FA_OK if the current device is an sm_100 part, else FA_ERR_DEVICE.
int check_device(int* dev_out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return FA_ERR_DEVICE;
  }
  *dev_out = dev;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_device_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_DEVICE;
    }
    g_device_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_device_ok[dev] == 1 ? FA_OK : FA_ERR_DEVICE;
}

int* device_status_ptr() {
  int* out = nullptr;
  const int e = g_status_ptr.get(&out, [](int** v) {
    void* p = nullptr;
    const cudaError_t r = cudaGetSymbolAddress(&p, g_status_word);
    if (r != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return static_cast<int>(r != cudaSuccess ? r : cudaErrorInvalidSymbol);
    }
    *v = static_cast<int*>(p);
    return 0;
  });
  return e == 0 ? out : nullptr;
}

}  // namespace fa

extern "C" {

int fa_abi_version(void) { return 1; }

int fa_build_flags(void) {
#ifdef FA_DEBUG
  return FA_BUILD_DEBUG;
#else
  return 0;
#endif
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_NULL: return "a required pointer is NULL";
    case FA_ERR_DTYPE: return "unsupported element type (inputs must be bf16 or fp16; output the input type or fp32)";
    case FA_ERR_HEADDIM: return "unsupported head dimension (must be 64 or 128)";
    case FA_ERR_SHAPE: return "invalid shape, split count or scale";
    case FA_ERR_ALIGN: return "a tensor pointer is misaligned (16 bytes; lse 4 bytes)";
    case FA_ERR_CU_SEQLENS: return "sequence lengths out of range (cu_seqlens must be non-decreasing within the packed extent, seqlens_k within [0, Nk])";
    case FA_ERR_WORKSPACE: return "decode workspace missing or too small";
    case FA_ERR_DEVICE: return "no usable sm_100 (B200) CUDA device";
    case FA_ERR_LAUNCH: return "CUDA launch or driver call failed";
    case FA_ERR_TIMEOUT: return "a bounded wait inside a kernel ran out";
    case FA_ERR_BOUNDS: return "an index check of the debug build caught an access outside its buffer";
    case FA_ERR_PAGE_TABLE: return "a block-table entry of the paged cache names no page of the pool";
    default: return "unknown status";
  }
}

}  // extern "C"

namespace {

int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk, int D,
             float scale, int causal, int prefix, const int* cu_seqlens, fa_stream_t stream, int in_dtype,
             int o_dtype) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  if (in_dtype != FA_BF16 && in_dtype != FA_FP16) return FA_ERR_DTYPE;
  if (o_dtype != in_dtype && o_dtype != FA_FP32) return FA_ERR_DTYPE;
  if (D != 64 && D != 128) return FA_ERR_HEADDIM;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || H > 65535) return FA_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_SHAPE;
  if (prefix < 0) return FA_ERR_SHAPE;
  if (cu_seqlens) {
    if (Nq != Nk) return FA_ERR_SHAPE;  // self-attention: one packed extent for Q and K/V
    if (static_cast<int64_t>(Nq) / 128 + B > INT32_MAX) return FA_ERR_SHAPE;
  } else {
    if (B > 65535 || Nq > (1 << 24) || Nk > (1 << 24)) return FA_ERR_SHAPE;
    if (static_cast<int64_t>(B) * Nq >= INT32_MAX || static_cast<int64_t>(B) * Nk >= INT32_MAX)
      return FA_ERR_SHAPE;
  }
  if (!fa::aligned(q, 16) || !fa::aligned(k, 16) || !fa::aligned(v, 16) || !fa::aligned(o, 16) || !fa::aligned(lse, 4))
    return FA_ERR_ALIGN;
  if (cu_seqlens && !fa::aligned(cu_seqlens, 4)) return FA_ERR_ALIGN;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  int* status = fa::device_status_ptr();
  if (!status) return FA_ERR_LAUNCH;
  fa::PrefillArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.cu_seqlens = cu_seqlens;
  a.status = status;
  a.B = B;
  a.H = H;
  a.Nq = Nq;
  a.Nk = Nk;
  a.D = D;
  a.scale = scale;
  a.causal = causal != 0;
  a.prefix = prefix;
  a.fp16 = in_dtype == FA_FP16;
  a.o_fp32 = o_dtype == FA_FP32;
  const int e = fa::launch_prefill(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != 0) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq, int Nk,
           int D, float scale, int causal, const int* cu_seqlens, fa_stream_t stream, int in_dtype,
           int o_dtype) {
  return fwd_impl(q, k, v, o, lse, B, H, Nq, Nk, D, scale, causal, 0, cu_seqlens, stream, in_dtype, o_dtype);
}

int fa_fwd_prefix(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                  int Nk, int D, float scale, int prefix_len, const int* cu_seqlens, fa_stream_t stream,
                  int in_dtype, int o_dtype) {
  return fwd_impl(q, k, v, o, lse, B, H, Nq, Nk, D, scale, 1, prefix_len, cu_seqlens, stream, in_dtype,
                  o_dtype);
}

size_t fa_decode_workspace_bytes(int B, int H, int D, int num_splits) {
  if (B < 1 || H < 1 || num_splits < 1 || (D != 64 && D != 128)) return 0;
  const size_t n = static_cast<size_t>(num_splits) * B * H;
  const size_t bytes = n * D * sizeof(float) + n * sizeof(float);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

}  // extern "C"

namespace {

// Argument checks of every split-KV decode entry point, in the boundary's fixed order.  The
// workspace is either the caller's (ws != nullptr required, at least ws_bytes, 16-byte aligned) or
// the library's fixed scratch array (fixed_ws: only its capacity ws_bytes is checked).
int decode_check(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse, int B, int H,
                 int Hkv, int Nk, int D, float scale, int num_splits, const int* seqlens_k, const void* ws,
                 size_t ws_bytes, bool fixed_ws, int in_dtype, int o_dtype, int key_offset, int Nk_total) {
  if (!q || !k_cache || !v_cache || !o || !lse) return FA_ERR_NULL;
  if (in_dtype != FA_BF16 && in_dtype != FA_FP16) return FA_ERR_DTYPE;
  if (o_dtype != in_dtype && o_dtype != FA_FP32) return FA_ERR_DTYPE;
  if (D != 64 && D != 128) return FA_ERR_HEADDIM;
  if (B < 1 || H < 1 || Nk < 1 || B > 65535 || H > 65535) return FA_ERR_SHAPE;
  if (Hkv < 1 || H % Hkv != 0) return FA_ERR_SHAPE;
  if (key_offset < 0 || static_cast<int64_t>(key_offset) + Nk > Nk_total) return FA_ERR_SHAPE;
  if (num_splits < 1 || num_splits > 128) return FA_ERR_SHAPE;
  if (static_cast<int64_t>(B) * H > (static_cast<int64_t>(1) << 28)) return FA_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_SHAPE;
  if (!fa::aligned(q, 16) || !fa::aligned(k_cache, 16) || !fa::aligned(v_cache, 16) || !fa::aligned(o, 16) || !fa::aligned(lse, 4))
    return FA_ERR_ALIGN;
  if ((!fixed_ws && !ws) || ws_bytes < fa_decode_workspace_bytes(B, H, D, num_splits)) return FA_ERR_WORKSPACE;
  if (!fixed_ws && !fa::aligned(ws, 16)) return FA_ERR_ALIGN;
  if (seqlens_k && !fa::aligned(seqlens_k, 4)) return FA_ERR_ALIGN;
  return FA_OK;
}

}  // namespace

namespace fa {

int decode_checked_launch(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse, int B,
                          int H, int Hkv, int Nk, int D, float scale, int num_splits, const int* seqlens_k,
                          void* ws, int in_dtype, int o_dtype, int key_offset, int Nk_total, cudaStream_t stream,
                          const int* block_table, int pages_per_seq, int page_size, int num_pages) {
  int* status = fa::device_status_ptr();
  if (!status) return FA_ERR_LAUNCH;
  fa::DecodeArgs a;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.o = o;
  a.lse = lse;
  const size_t n = static_cast<size_t>(num_splits) * B * H;
  a.ws_o = static_cast<float*>(ws);
  a.ws_lse = static_cast<float*>(ws) + n * D;
  a.status = status;
  a.B = B;
  a.H = H;
  a.Nk = Nk;
  a.D = D;
  a.S = num_splits;
  a.scale = scale;
  a.fp16 = in_dtype == FA_FP16;
  a.o_fp32 = o_dtype == FA_FP32;
  a.Hkv = Hkv;
  a.seqlens_k = seqlens_k;
  a.key_offset = key_offset;
  a.Nk_total = Nk_total;
  a.block_table = block_table;
  a.pages_per_seq = pages_per_seq;
  a.page_size = page_size;
  a.num_pages = num_pages;
  const int e = fa::launch_decode(a, stream);
  if (e != 0) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

int decode_check_fixed(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse, int B, int H,
                       int Nk, int D, float scale, int num_splits, size_t capacity, int in_dtype, int o_dtype) {
  return decode_check(q, k_cache, v_cache, o, lse, B, H, H, Nk, D, scale, num_splits, nullptr, nullptr, capacity,
                      true, in_dtype, o_dtype, 0, Nk);
}

}  // namespace fa

namespace {

int decode_impl(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse, int B, int H,
                int Hkv, int Nk, int D, float scale, int num_splits, const int* seqlens_k, void* workspace,
                size_t workspace_bytes, fa_stream_t stream, int in_dtype, int o_dtype, int key_offset = 0,
                int Nk_total = 0) {
  if (Nk_total == 0) Nk_total = Nk;
  if (const int st = decode_check(q, k_cache, v_cache, o, lse, B, H, Hkv, Nk, D, scale, num_splits, seqlens_k,
                                  workspace, workspace_bytes, false, in_dtype, o_dtype, key_offset, Nk_total))
    return st;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  return fa::decode_checked_launch(q, k_cache, v_cache, o, lse, B, H, Hkv, Nk, D, scale, num_splits, seqlens_k,
                                   workspace, in_dtype, o_dtype, key_offset, Nk_total,
                                   reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int fa_decode_splitkv(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse, int B,
                      int H, int Nk, int D, float scale, int num_splits, void* workspace,
                      size_t workspace_bytes, fa_stream_t stream, int in_dtype, int o_dtype) {
  return decode_impl(q, k_cache, v_cache, o, lse, B, H, H, Nk, D, scale, num_splits, nullptr, workspace,
                     workspace_bytes, stream, in_dtype, o_dtype);
}

int fa_decode_splitkv_gqa(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse, int B,
                          int Hq, int Hkv, int Nk, int D, float scale, int num_splits, const int* seqlens_k,
                          void* workspace, size_t workspace_bytes, fa_stream_t stream, int in_dtype,
                          int o_dtype) {
  return decode_impl(q, k_cache, v_cache, o, lse, B, Hq, Hkv, Nk, D, scale, num_splits, seqlens_k, workspace,
                     workspace_bytes, stream, in_dtype, o_dtype);
}

int fa_decode_splitkv_paged(const void* q, const void* k_pages, const void* v_pages, const int* block_table,
                            void* o, float* lse, int B, int Hq, int Hkv, int num_pages, int page_size,
                            int pages_per_seq, int D, float scale, int num_splits, const int* seqlens_k,
                            void* workspace, size_t workspace_bytes, fa_stream_t stream, int in_dtype,
                            int o_dtype) {
  if (!block_table) return FA_ERR_NULL;
  // page size: a power of two from 16 rows (whole 16-key boxes; 64-key tiles cover whole pages);
  // pool rows, cache capacity and table size within 32-bit indices
  if (page_size < 16 || page_size > (1 << 16) || (page_size & (page_size - 1)) != 0) return FA_ERR_SHAPE;
  if (num_pages < 1 || pages_per_seq < 1 || B < 1) return FA_ERR_SHAPE;
  if (static_cast<int64_t>(num_pages) * page_size >= (static_cast<int64_t>(1) << 31) ||
      static_cast<int64_t>(pages_per_seq) * page_size >= (static_cast<int64_t>(1) << 31) ||
      static_cast<int64_t>(B) * pages_per_seq >= (static_cast<int64_t>(1) << 31))
    return FA_ERR_SHAPE;
  const int Nk = pages_per_seq * page_size;
  if (const int st = decode_check(q, k_pages, v_pages, o, lse, B, Hq, Hkv, Nk, D, scale, num_splits, seqlens_k,
                                  workspace, workspace_bytes, false, in_dtype, o_dtype, 0, Nk))
    return st;
  if (!fa::aligned(block_table, 4)) return FA_ERR_ALIGN;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  return fa::decode_checked_launch(q, k_pages, v_pages, o, lse, B, Hq, Hkv, Nk, D, scale, num_splits, seqlens_k,
                                   workspace, in_dtype, o_dtype, 0, Nk, reinterpret_cast<cudaStream_t>(stream),
                                   block_table, pages_per_seq, page_size, num_pages);
}

size_t fa_decode_part_bytes(int B, int H, int D) {
  if (B < 1 || H < 1 || (D != 64 && D != 128)) return 0;
  const size_t bytes = static_cast<size_t>(B) * H * (D + 1) * sizeof(float);
  return (bytes + 15) & ~static_cast<size_t>(15);
}

int fa_decode_splitkv_shard(const void* q, const void* k_shard, const void* v_shard, float* part, int B,
                            int Hq, int Hkv, int Nk_shard, int key_offset, int Nk_total, int D, float scale,
                            int num_splits, const int* seqlens_k, void* workspace, size_t workspace_bytes,
                            fa_stream_t stream, int in_dtype) {
  if (!part) return FA_ERR_NULL;
  if (Nk_total < 1) return FA_ERR_SHAPE;
  float* lse = (B >= 1 && Hq >= 1 && (D == 64 || D == 128)) ? part + static_cast<size_t>(B) * Hq * D : part;
  return decode_impl(q, k_shard, v_shard, part, lse, B, Hq, Hkv, Nk_shard, D, scale, num_splits, seqlens_k,
                     workspace, workspace_bytes, stream, in_dtype, FA_FP32, key_offset, Nk_total);
}

int fa_decode_merge(const float* parts, int R, int B, int H, int D, void* o, float* lse, fa_stream_t stream,
                    int o_dtype) {
  if (!parts || !o || !lse) return FA_ERR_NULL;
  if (o_dtype != FA_BF16 && o_dtype != FA_FP16 && o_dtype != FA_FP32) return FA_ERR_DTYPE;
  if (D != 64 && D != 128) return FA_ERR_HEADDIM;
  if (R < 1 || R > 65536 || B < 1 || H < 1 || B > 65535 || H > 65535) return FA_ERR_SHAPE;
  if (static_cast<int64_t>(B) * H > (static_cast<int64_t>(1) << 28)) return FA_ERR_SHAPE;
  if (!fa::aligned(parts, 16) || !fa::aligned(o, 16) || !fa::aligned(lse, 4)) return FA_ERR_ALIGN;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  fa::MergeArgs a;
  a.parts = parts;
  a.part_floats = static_cast<long long>(fa_decode_part_bytes(B, H, D) / sizeof(float));
  a.R = R;
  a.B = B;
  a.H = H;
  a.D = D;
  a.o = o;
  a.lse = lse;
  a.o_fp16 = o_dtype == FA_FP16;
  a.o_fp32 = o_dtype == FA_FP32;
  a.status = fa::device_status_ptr();
  if (!a.status) return FA_ERR_LAUNCH;
  if (fa::launch_decode_merge(a, reinterpret_cast<cudaStream_t>(stream)) != 0) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

int fa_device_status(int* status_out, int clear) {
  if (!status_out) return FA_ERR_NULL;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  int* p = fa::device_status_ptr();
  if (!p) return FA_ERR_LAUNCH;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  *status_out = v;
  if (clear) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) {
      cudaGetLastError();
      return FA_ERR_LAUNCH;
    }
  }
  return FA_OK;
}

size_t fa_bwd_workspace_bytes(int B, int H, int Nq) {
  if (B < 1 || H < 1 || Nq < 1) return 0;
  const size_t bytes = static_cast<size_t>(B) * H * Nq * sizeof(float);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

int fa_bwd_masked(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, int B, int H, int Nq, int Nk, int D, float scale, int causal,
                  int prefix_len, const int* cu_seqlens, void* workspace, size_t workspace_bytes, fa_stream_t stream,
                  int in_dtype, int grad_dtype) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_NULL;
  if (in_dtype != FA_BF16 && in_dtype != FA_FP16) return FA_ERR_DTYPE;
  if (grad_dtype != in_dtype && grad_dtype != FA_FP32) return FA_ERR_DTYPE;
  if (D != 64 && D != 128) return FA_ERR_HEADDIM;
  if (B < 1 || H < 1 || Nq < 1 || Nk < 1 || B > 65535 || H > 65535) return FA_ERR_SHAPE;
  if (prefix_len < 0) return FA_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_SHAPE;
  if (cu_seqlens) {
    if (Nq != Nk) return FA_ERR_SHAPE;  // self-attention: one packed extent for Q and K/V
    if (static_cast<int64_t>(Nq) / 128 + B > INT32_MAX / 2) return FA_ERR_SHAPE;
    if (static_cast<int64_t>(H) * (Nq / 128 + B) >= INT32_MAX) return FA_ERR_SHAPE;
  } else {
    if (Nq > (1 << 24) || Nk > (1 << 24)) return FA_ERR_SHAPE;
    if (static_cast<int64_t>(B) * Nq >= INT32_MAX || static_cast<int64_t>(B) * Nk >= INT32_MAX) return FA_ERR_SHAPE;
    if (static_cast<int64_t>(B) * H * ((std::max(Nq, Nk) + 127) / 128) >= INT32_MAX) return FA_ERR_SHAPE;
  }
  if (!fa::aligned(q, 16) || !fa::aligned(k, 16) || !fa::aligned(v, 16) || !fa::aligned(o, 16) ||
      !fa::aligned(dout, 16) || !fa::aligned(dq, 16) || !fa::aligned(dk, 16) || !fa::aligned(dv, 16) ||
      !fa::aligned(lse, 4))
    return FA_ERR_ALIGN;
  if (cu_seqlens && !fa::aligned(cu_seqlens, 4)) return FA_ERR_ALIGN;
  // Drow: one float per query row, [B, H, Nq] dense or [H, total] varlen
  const size_t ws_need = cu_seqlens ? fa_bwd_workspace_bytes(1, H, Nq) : fa_bwd_workspace_bytes(B, H, Nq);
  if (!workspace || workspace_bytes < ws_need) return FA_ERR_WORKSPACE;
  if (!fa::aligned(workspace, 16)) return FA_ERR_ALIGN;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  int* status = fa::device_status_ptr();
  if (!status) return FA_ERR_LAUNCH;
  fa::BackwardArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dout = dout;
  a.lse = lse;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.drow = static_cast<float*>(workspace);
  a.status = status;
  a.cu_seqlens = cu_seqlens;
  a.B = B;
  a.H = H;
  a.Nq = Nq;
  a.Nk = Nk;
  a.D = D;
  a.scale = scale;
  a.causal = (causal != 0 || prefix_len > 0) ? 1 : 0;
  a.prefix = prefix_len;
  a.fp16 = in_dtype == FA_FP16;
  a.g_fp32 = grad_dtype == FA_FP32;
  const int e = fa::launch_backward(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != 0) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
           void* dk, void* dv, int B, int H, int Nq, int Nk, int D, float scale, int causal, void* workspace,
           size_t workspace_bytes, fa_stream_t stream, int in_dtype, int grad_dtype) {
  return fa_bwd_masked(q, k, v, o, dout, lse, dq, dk, dv, B, H, Nq, Nk, D, scale, causal, 0, nullptr, workspace,
                       workspace_bytes, stream, in_dtype, grad_dtype);
}

}  // extern "C"
