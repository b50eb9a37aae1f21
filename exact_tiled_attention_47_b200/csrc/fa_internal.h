// fa_internal.h -- launchers shared between the C-ABI layer (fa_api.cu) and the kernel files.
// Arguments reaching these functions have already been validated.
#pragma once
#include <cstddef>
#include <cstdint>
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
  float* drow;  // workspace: [B, H, Nq] fp32
  int* status;
  int B, H, Nq, Nk, D;
  float scale;
  int causal;
  int fp16;    // input type: 1 = fp16, 0 = bf16
  int g_fp32;  // gradient type: 1 = fp32, 0 = input type
};

// Return a cudaError_t-compatible code (0 = success).
int launch_prefill(const PrefillArgs& a, cudaStream_t stream);
int launch_decode(const DecodeArgs& a, cudaStream_t stream);
int launch_decode_merge(const MergeArgs& a, cudaStream_t stream);
int launch_backward(const BackwardArgs& a, cudaStream_t stream);

int* device_status_ptr();  // address of this device's status word (nullptr on failure)
int check_device(int* dev_out);  // FA_OK if the current device is sm_100, else FA_ERR_DEVICE
bool aligned(const void* p, uintptr_t a);

}  // namespace fa
