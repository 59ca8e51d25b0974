/* A plain C99 caller of the library: compiles against include/awq.h alone and
 * exercises the host-side checks of the entry points, none of which reaches
 * the GPU (every call below is rejected, or has no work, before any CUDA
 * call). Exit status 0 when every result is the documented one. */
#include <stdio.h>
#include <stdint.h>

#include "awq.h"

static int failures = 0;

static void expect(const char* what, awq_status_t got, awq_status_t want) {
  if (got != want) {
    fprintf(stderr, "%s: got %d (%s), want %d\n", what, (int)got, awq_status_string(got), (int)want);
    ++failures;
  }
}

int main(void) {
  /* fake device addresses: 16-byte aligned and misaligned; never dereferenced */
  const void* A = (const void*)(uintptr_t)0x10000;
  const void* MIS = (const void*)(uintptr_t)0x10002;
  awq_qconfig_t asym = {128, 1, 0};
  awq_qconfig_t g64 = {64, 1, 0};
  awq_qconfig_t packed = {128, 1, AWQ_FLAG_PACKED_ZEROS};
  size_t bytes = 7;

  if (awq_abi_version() != AWQ_ABI_VERSION) {
    fprintf(stderr, "ABI version %d, header %d\n", awq_abi_version(), AWQ_ABI_VERSION);
    ++failures;
  }
  expect("gemv: null x", awq_gemv(NULL, A, A, A, 1, 64, 256, asym, (uint16_t*)A, NULL, 0, NULL), AWQ_ERR_NULL);
  expect("gemv: M = 17", awq_gemv(A, A, A, A, 17, 64, 256, asym, (uint16_t*)A, NULL, 0, NULL), AWQ_ERR_SHAPE);
  expect("gemv: group 64", awq_gemv(A, A, A, A, 1, 64, 256, g64, (uint16_t*)A, NULL, 0, NULL),
         AWQ_ERR_UNSUPPORTED);
  expect("gemv: misaligned x", awq_gemv(MIS, A, A, A, 1, 64, 256, asym, (uint16_t*)A, NULL, 0, NULL),
         AWQ_ERR_ALIGN);
  expect("gemv: empty", awq_gemv(A, A, A, A, 1, 0, 256, asym, (uint16_t*)A, NULL, 0, NULL), AWQ_OK);
  expect("gemm: packed zeros, no workspace for their fp16 copy",
         awq_gemm(A, A, A, A, 32, 64, 256, packed, (uint16_t*)A, NULL, 0, NULL), AWQ_ERR_WORKSPACE);
  expect("gemm: empty batch", awq_gemm(A, A, A, A, 0, 64, 256, asym, (uint16_t*)A, NULL, 0, NULL), AWQ_OK);
  expect("quantize: K % 128", awq_pseudo_quantize_pack(A, 8, 100, asym, (int32_t*)A, (uint16_t*)A,
                                                       (uint16_t*)A, NULL), AWQ_ERR_SHAPE);
  expect("dequant: null W_out", awq_dequant(A, A, A, 8, 256, asym, NULL, NULL), AWQ_ERR_NULL);
  expect("pack zeros: N % 8", awq_pack_zeros(A, 2, 12, (int32_t*)A, NULL), AWQ_ERR_SHAPE);
  expect("unpack zeros: empty", awq_unpack_zeros(A, 0, 16, (uint16_t*)A, NULL), AWQ_OK);
  expect("workspace: null out", awq_workspace_bytes(1, 64, 256, asym, NULL), AWQ_ERR_NULL);
  expect("workspace: empty", awq_workspace_bytes(1, 0, 256, asym, &bytes), AWQ_OK);
  if (bytes != 0) {
    fprintf(stderr, "workspace bytes for an empty product: %zu\n", bytes);
    ++failures;
  }
  expect("noalloc: N % 8", awq_gemv_noalloc(A, A, A, A, 1, 60, 256, asym, (uint16_t*)A, NULL), AWQ_ERR_SHAPE);
  if (awq_status_string((awq_status_t)99) == NULL) ++failures;
  if (failures == 0) printf("abi_check: ok\n");
  return failures == 0 ? 0 : 1;
}
