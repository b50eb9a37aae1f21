// fa_noalloc.cu -- split-KV decode for callers that cannot allocate device memory.
//
// fa_decode_splitkv needs a caller-provided workspace for the per-split partial results.  Some
// callers cannot obtain one at call time (an engine that reserves all of its device memory at start
// and forbids later allocation, a plugin whose host framework owns the allocator, or code that must
// not pay for cudaMalloc, which can synchronise the device).  fa_decode_splitkv_noalloc runs the
// same two kernels with their partials placed in a fixed array that lives in this file:
//   * FA_NOALLOC_SCRATCH_BYTES (32 MiB) per GPU, reserved when this library's code is first used on
//     that GPU and held until the process exits;
//   * problems needing more scratch than that are rejected with FA_ERR_WORKSPACE before any launch;
//   * the first call on a device looks up the array's device address with that device current
//     (cudaGetSymbolAddress) and caches it; make that first call before any stream capture;
//   * all calls on a device share the one array, which keeps whatever the last call left in it.
//     Nothing needs clearing -- the split kernel writes every partial that the combine kernel of the
//     same call reads -- but two calls whose kernels overlap on the GPU (different streams without
//     ordering between them) race on the array and may return wrong results.
// No cudaMalloc, cudaFree or other allocating routine is called here.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "fa_internal.h"

namespace fa {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on device `dev` (the current device).  In host code the
// array's name is only a host-side stand-in, so the address must come from the runtime.
int noalloc_scratch(int dev, void** out) {
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return FA_ERR_LAUNCH;
    }
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" int fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o,
                                         float* lse, int B, int H, int Nk, int D, float scale, int num_splits,
                                         fa_stream_t stream, int in_dtype, int o_dtype) {
  if (!q || !k_cache || !v_cache || !o || !lse) return FA_ERR_NULL;
  if (in_dtype != FA_BF16 && in_dtype != FA_FP16) return FA_ERR_DTYPE;
  if (o_dtype != in_dtype && o_dtype != FA_FP32) return FA_ERR_DTYPE;
  if (D != 64 && D != 128) return FA_ERR_HEADDIM;
  if (B < 1 || H < 1 || Nk < 1 || B > 65535 || H > 65535) return FA_ERR_SHAPE;
  if (num_splits < 1 || num_splits > 128) return FA_ERR_SHAPE;
  if (static_cast<int64_t>(B) * H > (static_cast<int64_t>(1) << 28)) return FA_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return FA_ERR_SHAPE;
  if (!fa::aligned(q, 16) || !fa::aligned(k_cache, 16) || !fa::aligned(v_cache, 16) || !fa::aligned(o, 16) ||
      !fa::aligned(lse, 4))
    return FA_ERR_ALIGN;
  if (fa_decode_workspace_bytes(B, H, D, num_splits) > FA_NOALLOC_SCRATCH_BYTES) return FA_ERR_WORKSPACE;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  int* status = fa::device_status_ptr();
  if (!status) return FA_ERR_LAUNCH;
  void* scratch = nullptr;
  if (const int st = fa::noalloc_scratch(dev, &scratch)) return st;
  fa::DecodeArgs a;
  a.q = q;
  a.k = k_cache;
  a.v = v_cache;
  a.o = o;
  a.lse = lse;
  const size_t n = static_cast<size_t>(num_splits) * B * H;
  a.ws_o = static_cast<float*>(scratch);
  a.ws_lse = static_cast<float*>(scratch) + n * D;
  a.status = status;
  a.B = B;
  a.H = H;
  a.Nk = Nk;
  a.D = D;
  a.S = num_splits;
  a.scale = scale;
  a.fp16 = in_dtype == FA_FP16;
  a.o_fp32 = o_dtype == FA_FP32;
  const int e = fa::launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != 0) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}
