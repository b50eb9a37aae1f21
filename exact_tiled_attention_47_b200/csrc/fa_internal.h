// fa_internal.h -- launchers shared between the C-ABI layer (fa_api.cu) and the kernel files.
// Arguments reaching these functions have already been validated.
#pragma once
#include <cstddef>
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

namespace fa {

struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const int* cu_seqlens;  // nullptr = dense mode
  int* status;            // device status word
  int B, H, Nq, Nk, D;
  float scale;
  int causal;
  int prefix;  // causal only: keys [0, prefix) are visible to every query (0 = plain causal)
  int fp16;    // input type: 1 = fp16, 0 = bf16
  int o_fp32;  // output type: 1 = fp32, 0 = input type
};

struct DecodeArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  float* ws_o;    // [B, H, S, D]
  float* ws_lse;  // [B, H, S]
  int* status;
  int B, H, Nk, D, S;  // H: query heads
  float scale;
  int fp16;
  int o_fp32;
  int Hkv = 0;                     // KV heads (0: same as H); H is a multiple of it
  const int* seqlens_k = nullptr;  // device int32[B]: valid cache length per batch item (nullptr: Nk)
  // The cache may be one key shard of a longer cache: its rows are the keys [key_offset,
  // key_offset + Nk) of a cache of Nk_total keys (0: Nk), and seqlens_k counts keys of the whole cache.
  int key_offset = 0;
  int Nk_total = 0;
  // Paged cache (block_table != nullptr): k and v are pools of num_pages pages of page_size rows (a
  // power of two); block_table[b * pages_per_seq + i] is the page holding keys
  // [i * page_size, (i + 1) * page_size) of batch item b, and Nk = pages_per_seq * page_size.
  const int* block_table = nullptr;
  int pages_per_seq = 0, page_size = 0, num_pages = 0;
};

// Merge of R partial decode results (one per key shard) laid out as R packed blocks of part_floats
// floats: block r holds O_r [B, H, D] then LSE_r [B, H].
struct MergeArgs {
  const float* parts;
  long long part_floats;
  int R, B, H, D;
  void* o;
  float* lse;
  int o_fp16;  // 16-bit output: fp16 (1) or bf16 (0); ignored with o_fp32
  int o_fp32;
  int* status = nullptr;  // device status word (debug index checks)
};

struct BackwardArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o;     // forward output, input type
  const void* dout;  // upstream gradient, input type
  const float* lse;  // forward LSE [B, H, Nq]
  void* dq;
  void* dk;
  void* dv;
  float* drow;  // workspace: [B, H, Nq] fp32 ([H, total] varlen)
  int* status;
  const int* cu_seqlens = nullptr;  // packed varlen (Nq = Nk = total); nullptr = dense
  int B, H, Nq, Nk, D;
  float scale;
  int causal;
  int prefix = 0;  // causal only: keys [0, prefix) are visible to every query
  int fp16;    // input type: 1 = fp16, 0 = bf16
  int g_fp32;  // gradient type: 1 = fp32, 0 = input type
};

// Return a cudaError_t-compatible code (0 = success).
int launch_prefill(const PrefillArgs& a, cudaStream_t stream);
int launch_decode(const DecodeArgs& a, cudaStream_t stream);
int launch_decode_merge(const MergeArgs& a, cudaStream_t stream);
int launch_backward(const BackwardArgs& a, cudaStream_t stream);

// Split-KV decode after its arguments passed the boundary's checks and the device check: launches
// the split and combine kernels with the per-split partials in ws.  Returns an fa_status.
int decode_checked_launch(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse, int B,
                          int H, int Hkv, int Nk, int D, float scale, int num_splits, const int* seqlens_k,
                          void* ws, int in_dtype, int o_dtype, int key_offset, int Nk_total, cudaStream_t stream,
                          const int* block_table = nullptr, int pages_per_seq = 0, int page_size = 0,
                          int num_pages = 0);
// The boundary's decode argument checks for a workspace of fixed capacity (no caller pointer).
int decode_check_fixed(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse, int B, int H,
                       int Nk, int D, float scale, int num_splits, size_t capacity, int in_dtype, int o_dtype);

int* device_status_ptr();  // address of this device's status word (nullptr on failure)
int check_device(int* dev_out);  // FA_OK if the current device is sm_100, else FA_ERR_DEVICE
bool aligned(const void* p, uintptr_t a);

// Unique id of the calling thread's current CUDA context (0 if none is current or the driver cannot
// say).  Contexts are never given the id of an earlier one, so a cached per-device value tagged
// with it is known to be stale once the device's context was destroyed and recreated (for example
// by cudaDeviceReset).
unsigned long long current_context_id();

// A value set up once per device and CUDA context (a symbol's device address, a function attribute
// that was raised): make(&v) runs on the first use in a context and again whenever the current
// context's id differs from the one recorded, and its error is returned without being cached.
template <class T>
class PerContext {
 public:
  template <class F>
  int get(T* out, F&& make) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSlots) {
      cudaGetLastError();
      return static_cast<int>(cudaErrorInvalidDevice);
    }
    std::lock_guard<std::mutex> lk(mu_);
    const unsigned long long id = current_context_id();
    if (ok_[dev] && id != 0 && id == ctx_[dev]) {
      *out = val_[dev];
      return 0;
    }
    T v{};
    const int e = make(&v);
    if (e != 0) return e;
    val_[dev] = v;
    ctx_[dev] = current_context_id();  // make() has initialised the context if it was not yet
    ok_[dev] = true;
    *out = v;
    return 0;
  }

 private:
  static constexpr int kSlots = 64;
  std::mutex mu_;
  T val_[kSlots]{};
  unsigned long long ctx_[kSlots]{};
  bool ok_[kSlots]{};
};

}  // namespace fa
