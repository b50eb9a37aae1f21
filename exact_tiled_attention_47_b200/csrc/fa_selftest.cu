// fa_selftest.cu -- a check that a kernel's bounded wait ends with an error status instead of a hang.
//
// Every mbarrier wait in the library's kernels is bounded (fa_ptx.cuh, mbar_wait: one second of
// global time without progress raises the CTA's abort flag, records FA_ERR_TIMEOUT in the device
// status word and returns false).  fa_selftest_wait_timeout runs that very wait on a barrier that
// nothing ever arrives on, in a one-thread kernel, so that a caller (and the test suite) can see the
// path end with FA_ERR_TIMEOUT in fa_device_status() and the CUDA context still usable.  It traps,
// faults and spins without limit nowhere.
#include "../../include/fa.h"
#include "fa_internal.h"
#include "fa_ptx.cuh"

namespace fa {
namespace {

__global__ void __launch_bounds__(32, 1) selftest_wait_kernel(int* status, int* waited_out) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  mbar_fence_init();
  abort_flag = 0;
  const uint64_t t0 = global_timer_ns();
  const bool ok = mbar_wait(&bar, 0, &abort_flag, status);  // no arrival ever comes
  const uint64_t t1 = global_timer_ns();
  *waited_out = ok ? -1 : static_cast<int>((t1 - t0) / 1000000ull);  // milliseconds waited
}

}  // namespace
}  // namespace fa

extern "C" int fa_selftest_wait_timeout(int* waited_ms, fa_stream_t stream) {
  if (!waited_ms) return FA_ERR_NULL;
  int dev = -1;
  if (const int st = fa::check_device(&dev)) return st;
  int* status = fa::device_status_ptr();
  if (!status) return FA_ERR_LAUNCH;
  int* d_out = nullptr;
  // the result travels through the status word; the wait time through a pinned host word
  if (cudaHostAlloc(reinterpret_cast<void**>(&d_out), sizeof(int), cudaHostAllocMapped) != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  *d_out = 0;
  int* dev_view = nullptr;
  if (cudaHostGetDevicePointer(reinterpret_cast<void**>(&dev_view), d_out, 0) != cudaSuccess) {
    cudaFreeHost(d_out);
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  fa::selftest_wait_kernel<<<1, 32, 0, s>>>(status, dev_view);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  *waited_ms = *d_out;
  cudaFreeHost(d_out);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FA_ERR_LAUNCH;
  }
  return FA_OK;
}
