/* c_abi_check.c -- calls libfa_sm100.so through include/fa.h from plain C99: no CUDA headers, no
 * C++ and no torch.  Checks the version query, the status strings, argument validation (which comes
 * before any device access, so fake pointers are never dereferenced) and, with the argument
 * "nodevice", the answer on a machine without a B200.  Exit status 0 when every check holds. */
#include <stdio.h>
#include <string.h>

#include "fa.h"

#define A ((void*)0x100000) /* 16-byte aligned, never dereferenced */
#define AF ((float*)0x100000)

static int fails = 0;
#define CHECK(cond)                                                  \
  do {                                                               \
    if (!(cond)) {                                                   \
      printf("FAIL %s:%d: %s\n", __FILE__, __LINE__, #cond);         \
      ++fails;                                                       \
    }                                                                \
  } while (0)

int main(int argc, char** argv) {
  const int no_device = argc > 1 && strcmp(argv[1], "nodevice") == 0;
  int code, st = -1;

  CHECK(fa_abi_version() == 1);
  CHECK(fa_build_flags() == 0 || fa_build_flags() == FA_BUILD_DEBUG);
  for (code = FA_OK; code <= FA_ERR_PAGE_TABLE; ++code) CHECK(strcmp(fa_status_string(code), "unknown status") != 0);
  CHECK(strcmp(fa_status_string(FA_OK), fa_status_string(FA_ERR_NULL)) != 0);
  CHECK(strcmp(fa_status_string(-1), "unknown status") == 0);

  /* validation, in the documented order, before the device check */
  CHECK(fa_fwd(NULL, A, A, A, AF, 1, 1, 128, 128, 64, 0.125f, 0, NULL, NULL, FA_BF16, FA_BF16) == FA_ERR_NULL);
  CHECK(fa_fwd(A, A, A, A, AF, 1, 1, 128, 128, 64, 0.125f, 0, NULL, NULL, FA_FP32, FA_FP32) == FA_ERR_DTYPE);
  CHECK(fa_fwd(A, A, A, A, AF, 1, 1, 128, 128, 80, 0.125f, 0, NULL, NULL, FA_BF16, FA_BF16) == FA_ERR_HEADDIM);
  CHECK(fa_fwd(A, A, A, A, AF, 1, 1, 128, 128, 64, -1.0f, 0, NULL, NULL, FA_BF16, FA_BF16) == FA_ERR_SHAPE);
  CHECK(fa_fwd((char*)A + 2, A, A, A, AF, 1, 1, 128, 128, 64, 0.125f, 0, NULL, NULL, FA_BF16, FA_BF16) ==
        FA_ERR_ALIGN);
  CHECK(fa_decode_workspace_bytes(64, 32, 128, 16) >= (size_t)16 * 64 * 32 * 129 * 4);
  CHECK(fa_decode_workspace_bytes(64, 32, 96, 16) == 0);
  CHECK(fa_decode_part_bytes(3, 1, 64) == 784);
  CHECK(fa_decode_merge(AF, 0, 2, 8, 128, A, AF, NULL, FA_BF16) == FA_ERR_SHAPE);
  CHECK(fa_decode_splitkv_shard(A, A, A, AF, 2, 8, 2, 64, 65, 128, 128, 0.1f, 4, NULL, A, 1 << 20, NULL, FA_BF16) ==
        FA_ERR_SHAPE);
  CHECK(fa_decode_splitkv_paged(A, A, A, NULL, A, AF, 2, 8, 2, 32, 64, 4, 128, 0.1f, 4, NULL, A, 1 << 20, NULL,
                                FA_BF16, FA_BF16) == FA_ERR_NULL);
  CHECK(fa_decode_splitkv_paged(A, A, A, (const int*)A, A, AF, 2, 8, 2, 32, 48, 4, 128, 0.1f, 4, NULL, A, 1 << 20,
                                NULL, FA_BF16, FA_BF16) == FA_ERR_SHAPE);
  CHECK(fa_device_status(NULL, 0) == FA_ERR_NULL);

  if (no_device) { /* every argument valid: only the device check fails, nothing is launched */
    CHECK(fa_fwd(A, A, A, A, AF, 1, 1, 128, 128, 64, 0.125f, 1, NULL, NULL, FA_BF16, FA_FP32) == FA_ERR_DEVICE);
    CHECK(fa_decode_merge(AF, 2, 2, 8, 128, A, AF, NULL, FA_FP32) == FA_ERR_DEVICE);
    CHECK(fa_decode_splitkv_paged(A, A, A, (const int*)A, A, AF, 2, 8, 2, 32, 16, 4, 128, 0.1f, 4, NULL, A, 1 << 20,
                                  NULL, FA_BF16, FA_FP32) == FA_ERR_DEVICE);
    CHECK(fa_device_status(&st, 0) == FA_ERR_DEVICE);
  }
  printf(fails ? "c_abi_check: %d failure(s)\n" : "c_abi_check: ok\n", fails);
  return fails != 0;
}
