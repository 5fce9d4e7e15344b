/* The C example shown in README.md: one forward call through the C ABI with
 * a workspace from cudaMalloc.  tests/test_abi_cpu.py compiles it against
 * include/sage_b200.h and links it with the library. */
#include <cuda_runtime.h>
#include "sage_b200.h"

int attend(const void* q, const void* k, const void* v, void* out, int B, int N, int H, int D,
           cudaStream_t stream) {
  const int64_t sh = D, sn = (int64_t)H * D, sb = (int64_t)N * H * D;  /* element strides */
  sage_view_bf16 vq = {q, sb, sn, sh}, vk = {k, sb, sn, sh}, vv = {v, sb, sn, sh};
  size_t bytes = 0;
  void* ws = NULL;
  int rc = sage_workspace_bytes(SAGE_OP_ATTN_FWD, B, N, H, D, &bytes);
  if (rc != SAGE_OK) return rc;
  if (cudaMalloc(&ws, bytes) != cudaSuccess) return SAGE_ERR_CUDA;  /* 256-byte aligned */
  rc = sage_attn_fwd(vq, vk, vv, out, sb, sn, sh, B, N, H, D, 0.0f /* 1/sqrt(D) */, ws, bytes, stream);
  if (rc == SAGE_OK) rc = sage_read_device_status(ws, stream);  /* waits for the stream */
  cudaFree(ws);
  return rc;  /* SAGE_OK, or see sage_strerror(rc) */
}
