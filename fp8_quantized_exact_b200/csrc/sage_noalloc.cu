// sage_attn_fwd_noalloc: the whole attention path for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is not allowed or not
// available to it, for example inside a region that must not allocate (a
// real-time or capture-sensitive section), inside a host framework whose
// device memory is wholly owned by its own arena, or a plug-in that is
// handed tensors but no allocator.  Such a caller cannot provide the
// workspace that sage_attn_fwd asks for.
//
// What it does: the scratch that sage_attn_fwd keeps in its workspace (the
// quantised Q/K/V, their scales, the K mean, the per-chunk partial sums and
// the status word) lives in one fixed array compiled into this library.
// Every GPU that loads the library keeps that array until the process
// exits.  The caller still passes the inputs and the output.
#include <mutex>

#include "sage_common.cuh"

namespace {

// The fixed scratch area (device memory of every device that loads the
// library).  Its host-side name is only a handle: the device address comes
// from cudaGetSymbolAddress, taken once per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SAGE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call made with that device current).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return SAGE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return SAGE_OK;
}

}  // namespace

extern "C" SAGE_API int sage_attn_fwd_noalloc(sage_view_bf16 q, sage_view_bf16 k,
                                              sage_view_bf16 v, void* out, int64_t out_stride_b,
                                              int64_t out_stride_n, int64_t out_stride_h, int B,
                                              int N, int H, int D, float sm_scale, void* stream) {
  size_t need = 0;
  int rc = sage_workspace_bytes(SAGE_OP_ATTN_FWD, B, N, H, D, &need);
  if (rc != SAGE_OK) return rc;
  if (B == 0 || N == 0 || H == 0) return SAGE_OK;
  if (need > (size_t)SAGE_NOALLOC_SCRATCH_BYTES) return SAGE_ERR_WORKSPACE;  // problem too large
  void* scratch = nullptr;
  if ((rc = scratch_address(&scratch)) != SAGE_OK) return rc;
  // The same kernels as sage_attn_fwd, with the fixed array as workspace.
  // sage_attn_fwd clears the status word; every other byte it reads there
  // it has written earlier in the same call.
  return sage_attn_fwd(q, k, v, out, out_stride_b, out_stride_n, out_stride_h, B, N, H, D,
                       sm_scale, scratch, (size_t)SAGE_NOALLOC_SCRATCH_BYTES, stream);
}

// The status word at the start of the fixed array (sage_attn_fwd clears it
// at the start of each call and the kernels record their errors there).
extern "C" SAGE_API int sage_noalloc_read_status(void* stream) {
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != SAGE_OK) return rc;
  return sage_read_device_status(scratch, stream);
}
