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
//     (cudaGetSymbolAddress) and caches it for the device's CUDA context (a later context, after a
//     device reset, looks it up again); make that first call before any stream capture;
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

// Device address of the scratch array on the current device.  In host code the array's name is only
// a host-side stand-in, so the address comes from the runtime, looked up once per device and CUDA
// context (again after the context was destroyed and recreated, e.g. by cudaDeviceReset).
PerContext<void*> g_noalloc_addr;

int noalloc_scratch(void** out) {
  const int e = g_noalloc_addr.get(out, [](void** v) {
    void* p = nullptr;
    const cudaError_t r = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (r != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return static_cast<int>(r != cudaSuccess ? r : cudaErrorInvalidSymbol);
    }
    *v = p;
    return 0;
  });
  return e == 0 ? FA_OK : FA_ERR_LAUNCH;
}

}  // namespace
}  // namespace fa

extern "C" int fa_decode_splitkv_noalloc(const void* q, const void* k_cache, const void* v_cache, void* o,
                                         float* lse, int B, int H, int Nk, int D, float scale, int num_splits,
                                         fa_stream_t stream, int in_dtype, int o_dtype) {
  // the same checks as fa_decode_splitkv, with the fixed array's capacity in place of a workspace
  if (const int st = fa::decode_check_fixed(q, k_cache, v_cache, o, lse, B, H, Nk, D, scale, num_splits,
                                            FA_NOALLOC_SCRATCH_BYTES, in_dtype, o_dtype))
    return st;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  void* scratch = nullptr;
  if (const int st = fa::noalloc_scratch(&scratch)) return st;
  return fa::decode_checked_launch(q, k_cache, v_cache, o, lse, B, H, H, Nk, D, scale, num_splits, nullptr, scratch,
                                   in_dtype, o_dtype, 0, Nk, reinterpret_cast<cudaStream_t>(stream));
}
