// C ABI of the library: argument checks, workspace carving, launches.
// See include/sage_b200.h for the contract of every entry point.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "sage_common.cuh"

using namespace sage;

namespace {

constexpr size_t kAlign = 1024;
constexpr int kMaxGridYZ = 65535;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Process-wide settings; entry points may be called from several threads.
std::atomic<int> g_mainloop{SAGE_MAINLOOP_DEFAULT};
std::once_flag g_mainloop_env_once;            // SAGE_MAINLOOP is read once
std::atomic<int> g_stall_tile{-1};             // test hook (sage_debug_set_stall)
std::atomic<long long> g_wait_limit{kDefaultWaitLimit};

// Prepass implementations.  SAGE_PREPASS=separate|stream, read once, picks
// one for every call (a measurement and test hook); without it each entry
// point uses its own default.
enum PrepassImpl { kPrepSeparate = 0, kPrepStream = 1 };
std::once_flag g_prepass_env_once;
int g_prepass_env = -1;
void read_prepass_env() {
  const char* e = getenv("SAGE_PREPASS");
  if (!e) return;
  if (!strcmp(e, "separate")) g_prepass_env = kPrepSeparate;
  else if (!strcmp(e, "stream")) g_prepass_env = kPrepStream;
}
int prepass_impl(int dflt) {
  std::call_once(g_prepass_env_once, read_prepass_env);
  return g_prepass_env >= 0 ? g_prepass_env : dflt;
}

struct Dims {
  int B, N, H, D, Nq, Nk, G32, T64;
};

Dims make_dims(int B, int N, int H, int D) {
  Dims d{B, N, H, D, 0, 0, 0, 0};
  d.Nq = ceil_div(N, kQTile) * kQTile;
  d.T64 = ceil_div(N, kKTile);
  d.Nk = d.T64 * kKTile;
  d.G32 = ceil_div(N, kQGroup);
  return d;
}

int check_dims(int B, int N, int H, int D) {
  if (B < 0 || N < 0 || H < 0 || D < 0) return SAGE_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SAGE_ERR_UNSUPPORTED;
  // H and B are the y and z extents of the kernels' grids
  if (B > kMaxGridYZ || H > kMaxGridYZ) return SAGE_ERR_UNSUPPORTED;
  // keep every flat index inside int range assumptions of the kernels
  if ((int64_t)B * H > (1 << 30) || N > (1 << 28)) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

bool empty(int B, int N, int H) { return B == 0 || N == 0 || H == 0; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_view(const sage_view_bf16& v) {
  if (!v.data) return SAGE_ERR_INVALID_ARG;
  if (v.stride_b < 0 || v.stride_n < 0 || v.stride_h < 0) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(v.data) || (v.stride_b | v.stride_n | v.stride_h) & 7) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

int check_out(const void* out, int64_t sb, int64_t sn, int64_t sh) {
  if (!out) return SAGE_ERR_INVALID_ARG;
  if (sb < 0 || sn < 0 || sh < 0) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(out) || (sb | sn | sh) & 7) return SAGE_ERR_UNSUPPORTED;
  return SAGE_OK;
}

// Byte offsets of every region of a workspace.
struct Layout {
  size_t status = 0;
  size_t q8 = 0, q_scale = 0, k8 = 0, k_scale = 0, k_mean = 0, v8 = 0, v_scale = 0;
  size_t k_part = 0, v_amax = 0, sync = 0;
  size_t total = 0;
};

Layout plan(int op, const Dims& d) {
  Layout L;
  size_t off = align_up(SAGE_STATUS_BYTES);
  const size_t bh = (size_t)d.B * d.H;
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  if (op == SAGE_OP_ATTN_FWD) {
    L.q8 = take(bh * d.Nq * d.D);
    L.q_scale = take(bh * d.G32 * sizeof(float));
    L.k8 = take(bh * d.Nk * d.D);
    L.k_scale = take(bh * d.T64 * sizeof(float));
    L.k_mean = take(bh * d.D * sizeof(float));
    L.v8 = take(bh * d.D * d.Nk);
    L.v_scale = take(bh * d.D * sizeof(float));
  }
  const bool all3 = op == SAGE_OP_ATTN_FWD || op == SAGE_OP_QUANT_QKV;
  if (all3 || op == SAGE_OP_QUANT_QK) L.k_part = take(bh * d.T64 * d.D * sizeof(double));
  if (all3 || op == SAGE_OP_QUANT_V) L.v_amax = take(bh * d.D * sizeof(float));
  if (all3) L.sync = take(prepass_sync_bytes(d.B, d.H, d.D));  // single-launch prepasses
  L.total = off;
  return L;
}

int check_ws(void* ws, size_t bytes, size_t need) {
  if (!ws) return SAGE_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SAGE_ERR_WORKSPACE;
  if (bytes < need) return SAGE_ERR_WORKSPACE;
  return SAGE_OK;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

FusedOut fused_out(void* ws, const Layout& L, int8_t* q8, float* qs, int8_t* k8, float* ks, float* km,
                   uint8_t* v8, float* vs, void* status) {
  FusedOut o;
  o.q8 = q8; o.q_scale = qs; o.k8 = k8; o.k_scale = ks; o.k_mean = km; o.v8 = v8; o.v_scale = vs;
  o.k_part = at<double>(ws, L.k_part);
  o.sync = at<void>(ws, L.sync);
  o.status = static_cast<DeviceStatus*>(status);
  o.wait_limit = g_wait_limit.load();
  o.stall_unit = g_stall_tile.load();
  return o;
}

// The three prepasses on checked arguments into the given outputs, by the
// implementation `impl` (a PrepassImpl, unless SAGE_PREPASS overrides it).
// Both give the same bytes.
int prepass_all(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, int B, int N, int H,
                int D, int8_t* q8, float* qs, int8_t* k8, float* ks, float* km, uint8_t* v8, float* vs,
                void* ws, const Layout& L, void* status, int impl, cudaStream_t s) {
  int rc;
  impl = prepass_impl(impl);
  if (impl == kPrepStream)
    return launch_prepass_stream(q, k, v, B, N, H, D, fused_out(ws, L, q8, qs, k8, ks, km, v8, vs, status), s);
  if ((rc = launch_prepass_qk(q, k, B, N, H, D, q8, qs, k8, ks, km, at<double>(ws, L.k_part), s))) return rc;
  return launch_prepass_v(v, B, N, H, D, v8, vs, at<float>(ws, L.v_amax), s);
}

// The streaming single launch below about the L2 size of Q, K and V, where
// the six separate launches' fixed cost dominates; the separate kernels
// above it, where they stream faster (measured on B200: 0.016 against
// 0.060 ms at B1 N256 H2 D128, 0.24 against 0.18 ms at B2 N8192 H32 D128).
int default_prepass(int B, int N, int H, int D) {
  const double bytes = 3.0 * B * H * (double)N * D * 2.0;
  return bytes < (double)(128u << 20) ? kPrepStream : kPrepSeparate;
}

int clear_status(void* ws, cudaStream_t s) {
  return cudaMemsetAsync(ws, 0, sizeof(DeviceStatus), s) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

float log2_scale(float sm_scale, int D) {
  if (!(sm_scale > 0.0f)) sm_scale = (float)(1.0 / sqrt((double)D));
  return (float)((double)sm_scale * 1.4426950408889634074);
}

// The SAGE_MAINLOOP environment variable picks the mainloop until the first
// sage_set_mainloop call, which always wins.
void read_mainloop_env() {
  const char* e = getenv("SAGE_MAINLOOP");
  if (!e) return;
  if (!strcmp(e, "tcgen05")) g_mainloop.store(SAGE_MAINLOOP_TCGEN05);
  else if (!strcmp(e, "mma_sync") || !strcmp(e, "mmasync")) g_mainloop.store(SAGE_MAINLOOP_MMA_SYNC);
  else if (!strcmp(e, "tcgen05_f32")) g_mainloop.store(SAGE_MAINLOOP_TCGEN05_F32);
}

int resolved_mainloop() {
  std::call_once(g_mainloop_env_once, read_mainloop_env);
  const int m = g_mainloop.load();
  if (m == SAGE_MAINLOOP_DEFAULT) return tc_available() ? SAGE_MAINLOOP_TCGEN05 : SAGE_MAINLOOP_MMA_SYNC;
  return m;
}

AttnParams make_params(const Dims& d, const int8_t* q8, const float* qs, const int8_t* k8,
                       const float* ks, const uint8_t* v8, const float* vs, void* out,
                       int64_t osb, int64_t osn, int64_t osh, float sm_scale, void* status) {
  AttnParams p;
  p.q8 = q8; p.q_scale = qs; p.k8 = k8; p.k_scale = ks; p.v8 = v8; p.v_scale = vs;
  p.out = static_cast<uint16_t*>(out);
  p.os_b = osb; p.os_n = osn; p.os_h = osh;
  p.B = d.B; p.N = d.N; p.H = d.H; p.D = d.D;
  p.Nq = d.Nq; p.Nk = d.Nk; p.G32 = d.G32; p.T64 = d.T64;
  p.sl2 = log2_scale(sm_scale, d.D);
  p.status = static_cast<DeviceStatus*>(status);
  p.wait_limit = g_wait_limit.load();
  p.stall_tile = g_stall_tile.load();
  p.dbg_qt = p.dbg_h = p.dbg_b = 0;
  p.dbg_tile = -1;
  p.dbg_out = nullptr;
  return p;
}

int run_mainloop(const AttnParams& p, cudaStream_t s) {
  switch (resolved_mainloop()) {
    case SAGE_MAINLOOP_TCGEN05: return launch_attn_tc(p, s);
    case SAGE_MAINLOOP_TCGEN05_F32: return launch_attn_tc_f32(p, s);
    default: return launch_attn_mma(p, s);
  }
}


// Copy the heads [h0, h1) of a [B, N, H, D] BF16 view between two buffers
// laid out with the same element strides: per batch, one 2D copy whose rows
// are the tokens when those heads are adjacent within a token's row, else
// one 2D copy per head.
int copy_heads(void* dst, const void* src, int64_t sb, int64_t sn, int64_t sh, int B, int N, int D,
               int h0, int h1, cudaMemcpyKind kind, cudaStream_t s) {
  const bool merged = sh == D && sn >= (int64_t)(h1 - h0) * D;
  const int step = merged ? h1 - h0 : 1;
  for (int b = 0; b < B; ++b)
    for (int h = h0; h < h1; h += step) {
      const size_t off = (size_t)((int64_t)b * sb + (int64_t)h * sh) * 2;
      const size_t width = (size_t)step * D * 2;
      const size_t pitch = N > 1 ? (size_t)sn * 2 : width;
      if (cudaMemcpy2DAsync(static_cast<char*>(dst) + off, pitch, static_cast<const char*>(src) + off, pitch,
                            width, (size_t)N, kind, s) != cudaSuccess)
        return SAGE_ERR_CUDA;
    }
  return SAGE_OK;
}

// Pinned (page-locked or registered) host memory, and device-accessible memory.
int pointer_type(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return (int)a.type;
}
bool host_pinned(const void* p) { return pointer_type(p) == (int)cudaMemoryTypeHost; }
bool device_memory(const void* p) {
  const int t = pointer_type(p);
  return t == (int)cudaMemoryTypeDevice || t == (int)cudaMemoryTypeManaged;
}

// The path of sage_attn_fwd on checked arguments, its buffers carved from
// `workspace`; device errors go to the status word at `status` (which the
// callers clear).
int fwd_body(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, void* out,
             int64_t out_stride_b, int64_t out_stride_n, int64_t out_stride_h, int B, int N, int H, int D,
             float sm_scale, void* workspace, void* status, int prepass, cudaStream_t s) {
  int rc;
  const Dims d = make_dims(B, N, H, D);
  const Layout L = plan(SAGE_OP_ATTN_FWD, d);
  int8_t* q8 = at<int8_t>(workspace, L.q8);
  float* qs = at<float>(workspace, L.q_scale);
  int8_t* k8 = at<int8_t>(workspace, L.k8);
  float* ks = at<float>(workspace, L.k_scale);
  float* km = at<float>(workspace, L.k_mean);
  uint8_t* v8 = at<uint8_t>(workspace, L.v8);
  float* vs = at<float>(workspace, L.v_scale);
  if ((rc = prepass_all(q, k, v, B, N, H, D, q8, qs, k8, ks, km, v8, vs, workspace, L, status, prepass, s)))
    return rc;
  return run_mainloop(make_params(d, q8, qs, k8, ks, v8, vs, out, out_stride_b, out_stride_n,
                                  out_stride_h, sm_scale, status),
                      s);
}

// Head counts of the chunks of sage_attn_fwd_host: 2, 2, then `hc` heads at
// a time, and 2 at the end.  The first copy-in and the last copy-out overlap
// nothing, so they are kept small; but not one head, whose rows (one head's
// D elements per token) the copy engines move at half the rate of two heads'
// (measured on B200: 26 against 52 GB/s for 256- and 512-byte rows).  Two
// heads copy in faster than they compute, so the ramp never starves the
// compute stream.
std::vector<int> host_chunks(int H, int hc) {
  std::vector<int> sizes;
  const int tail = (H >= 6 && hc >= 2) ? 2 : 0;
  int rem = H - tail;
  for (int x : {2, 2}) {
    if (rem <= 0) break;
    const int c = std::min(std::min(x, hc), rem);
    sizes.push_back(c);
    rem -= c;
  }
  while (rem > 0) {
    const int c = std::min(hc, rem);
    sizes.push_back(c);
    rem -= c;
  }
  if (tail) sizes.push_back(tail);
  return sizes;
}
}  // namespace

extern "C" {

int sage_workspace_bytes(int op, int B, int N, int H, int D, size_t* bytes) {
  if (!bytes || op < SAGE_OP_QUANT_QK || op > SAGE_OP_ATTN_FWD_HOST) return SAGE_ERR_INVALID_ARG;
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (op == SAGE_OP_ATTN_FWD_HOST)  // two chunk workspaces of H heads
    *bytes = 2 * align_up(plan(SAGE_OP_ATTN_FWD, make_dims(B, N, H, D)).total);
  else
    *bytes = plan(op, make_dims(B, N, H, D)).total;
  return SAGE_OK;
}

int sage_fwd_workspace_layout(int B, int N, int H, int D, sage_fwd_layout* out) {
  if (!out) return SAGE_ERR_INVALID_ARG;
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  Layout L = plan(SAGE_OP_ATTN_FWD, make_dims(B, N, H, D));
  out->q_i8 = L.q8; out->q_scale = L.q_scale; out->k_i8 = L.k8; out->k_scale = L.k_scale;
  out->k_mean = L.k_mean; out->v_fp8 = L.v8; out->v_scale = L.v_scale; out->total = L.total;
  return SAGE_OK;
}

int sage_quant_qk(sage_view_bf16 q, sage_view_bf16 k, int B, int N, int H, int D, int8_t* q_i8,
                  float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean, void* workspace,
                  size_t workspace_bytes, void* stream) {
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return SAGE_OK;
  if ((rc = check_view(q)) || (rc = check_view(k))) return rc;
  if (!q_i8 || !q_scale || !k_i8 || !k_scale || !k_mean) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(q_scale) || !aligned16(k_scale) ||
      !aligned16(k_mean))
    return SAGE_ERR_UNSUPPORTED;
  const Dims d = make_dims(B, N, H, D);
  const Layout L = plan(SAGE_OP_QUANT_QK, d);
  if ((rc = check_ws(workspace, workspace_bytes, L.total))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(workspace, s))) return rc;
  return launch_prepass_qk(q, k, B, N, H, D, q_i8, q_scale, k_i8, k_scale, k_mean,
                           at<double>(workspace, L.k_part), s);
}

int sage_norm_rope_quant_qk(sage_view_bf16 q, sage_view_bf16 k, const void* wq, const void* wk, const float* cos_t,
                            const float* sin_t, float eps, int B, int N, int H, int D, int8_t* q_i8, float* q_scale,
                            int8_t* k_i8, float* k_scale, float* k_mean, void* workspace, size_t workspace_bytes,
                            void* stream) {
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return SAGE_OK;
  if ((rc = check_view(q)) || (rc = check_view(k))) return rc;
  if (!wq || !wk || !cos_t || !sin_t || !q_i8 || !q_scale || !k_i8 || !k_scale || !k_mean) return SAGE_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(wq) || !aligned16(wk) || !aligned16(cos_t) || !aligned16(sin_t) || !aligned16(q_i8) ||
      !aligned16(k_i8) || !aligned16(q_scale) || !aligned16(k_scale) || !aligned16(k_mean))
    return SAGE_ERR_UNSUPPORTED;
  const Dims d = make_dims(B, N, H, D);
  const Layout L = plan(SAGE_OP_QUANT_QK, d);
  if ((rc = check_ws(workspace, workspace_bytes, L.total))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(workspace, s))) return rc;
  NormRopeIn in{static_cast<const uint16_t*>(wq), static_cast<const uint16_t*>(wk), cos_t, sin_t, eps};
  return launch_norm_rope_qk(in, q, k, B, N, H, D, q_i8, q_scale, k_i8, k_scale, k_mean,
                             at<double>(workspace, L.k_part), s);
}

int sage_quant_v(sage_view_bf16 v, int B, int N, int H, int D, uint8_t* v_fp8, float* v_scale,
                 void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return SAGE_OK;
  if ((rc = check_view(v))) return rc;
  if (!v_fp8 || !v_scale) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(v_fp8) || !aligned16(v_scale)) return SAGE_ERR_UNSUPPORTED;
  const Dims d = make_dims(B, N, H, D);
  const Layout L = plan(SAGE_OP_QUANT_V, d);
  if ((rc = check_ws(workspace, workspace_bytes, L.total))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(workspace, s))) return rc;
  return launch_prepass_v(v, B, N, H, D, v_fp8, v_scale, at<float>(workspace, L.v_amax), s);
}

int sage_quant_qkv(sage_view_bf16 q, sage_view_bf16 k, sage_view_bf16 v, int B, int N, int H, int D,
                   int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean,
                   uint8_t* v_fp8, float* v_scale, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return SAGE_OK;
  if ((rc = check_view(q)) || (rc = check_view(k)) || (rc = check_view(v))) return rc;
  if (!q_i8 || !q_scale || !k_i8 || !k_scale || !k_mean || !v_fp8 || !v_scale) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(q_scale) || !aligned16(k_scale) ||
      !aligned16(k_mean) || !aligned16(v_fp8) || !aligned16(v_scale))
    return SAGE_ERR_UNSUPPORTED;
  const Dims d = make_dims(B, N, H, D);
  const Layout L = plan(SAGE_OP_QUANT_QKV, d);
  if ((rc = check_ws(workspace, workspace_bytes, L.total))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(workspace, s))) return rc;
  return prepass_all(q, k, v, B, N, H, D, q_i8, q_scale, k_i8, k_scale, k_mean, v_fp8, v_scale, workspace, L,
                     workspace, kPrepStream, s);
}

int sage_attn_fwd_prepass_kernels(int B, int N, int H, int D) {
  const int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return 0;
  return prepass_impl(default_prepass(B, N, H, D)) == kPrepStream ? 1 : 6;
}

int sage_quant_qkv_kernels(int B, int N, int H, int D) {
  const int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return 0;
  return 1;
}

int sage_attn_from_quant(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                         const float* k_scale, const uint8_t* v_fp8, const float* v_scale,
                         void* out, int64_t out_stride_b, int64_t out_stride_n,
                         int64_t out_stride_h, int B, int N, int H, int D, float sm_scale,
                         void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return SAGE_OK;
  if (!q_i8 || !q_scale || !k_i8 || !k_scale || !v_fp8 || !v_scale) return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(v_fp8) || !aligned16(q_scale) ||
      !aligned16(k_scale) || !aligned16(v_scale))
    return SAGE_ERR_UNSUPPORTED;
  if ((rc = check_out(out, out_stride_b, out_stride_n, out_stride_h))) return rc;
  const Dims d = make_dims(B, N, H, D);
  if ((rc = check_ws(workspace, workspace_bytes, plan(SAGE_OP_ATTN_FROM_QUANT, d).total))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(workspace, s))) return rc;
  return run_mainloop(make_params(d, q_i8, q_scale, k_i8, k_scale, v_fp8, v_scale, out,
                                  out_stride_b, out_stride_n, out_stride_h, sm_scale, workspace),
                      s);
}

int sage_attn_fwd(sage_view_bf16 q, sage_view_bf16 k, sage_view_bf16 v, void* out,
                  int64_t out_stride_b, int64_t out_stride_n, int64_t out_stride_h, int B, int N,
                  int H, int D, float sm_scale, void* workspace, size_t workspace_bytes,
                  void* stream) {
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return SAGE_OK;
  if ((rc = check_view(q)) || (rc = check_view(k)) || (rc = check_view(v))) return rc;
  if ((rc = check_out(out, out_stride_b, out_stride_n, out_stride_h))) return rc;
  const Layout L = plan(SAGE_OP_ATTN_FWD, make_dims(B, N, H, D));
  if ((rc = check_ws(workspace, workspace_bytes, L.total))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(workspace, s))) return rc;
  return fwd_body(q, k, v, out, out_stride_b, out_stride_n, out_stride_h, B, N, H, D, sm_scale, workspace,
                  workspace, default_prepass(B, N, H, D), s);
}

int sage_attn_fwd_host(sage_view_bf16 q_host, sage_view_bf16 k_host, sage_view_bf16 v_host,
                       sage_view_bf16 q_dev, sage_view_bf16 k_dev, sage_view_bf16 v_dev, void* out_host,
                       void* out_dev, int64_t out_stride_b, int64_t out_stride_n, int64_t out_stride_h, int B,
                       int N, int H, int D, float sm_scale, int heads_per_chunk, void* workspace,
                       size_t workspace_bytes, void* stream, void* stream_alt, void* stream_in, void* stream_out,
                       void* event_in, void* event_compute, void* event_out) {
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return SAGE_OK;
  if ((rc = check_view(q_dev)) || (rc = check_view(k_dev)) || (rc = check_view(v_dev))) return rc;
  if ((rc = check_out(out_dev, out_stride_b, out_stride_n, out_stride_h))) return rc;
  const sage_view_bf16* hv[3] = {&q_host, &k_host, &v_host};
  const sage_view_bf16* dv[3] = {&q_dev, &k_dev, &v_dev};
  for (int i = 0; i < 3; ++i) {
    if (!hv[i]->data) return SAGE_ERR_INVALID_ARG;
    if (hv[i]->stride_b != dv[i]->stride_b || hv[i]->stride_n != dv[i]->stride_n ||
        hv[i]->stride_h != dv[i]->stride_h)
      return SAGE_ERR_INVALID_ARG;
    if (N > 1 && dv[i]->stride_n < D) return SAGE_ERR_UNSUPPORTED;
  }
  if (!out_host || !event_in || !event_compute || !event_out) return SAGE_ERR_INVALID_ARG;
  if (N > 1 && out_stride_n < D) return SAGE_ERR_UNSUPPORTED;
  const int hc = heads_per_chunk > 0 ? (heads_per_chunk < H ? heads_per_chunk : H) : (H < 4 ? H : 4);
  // with a second compute stream the chunks alternate between two workspaces
  const size_t per_chunk = align_up(plan(SAGE_OP_ATTN_FWD, make_dims(B, N, hc, D)).total);
  const int n_ws = stream_alt ? 2 : 1;
  if ((rc = check_ws(workspace, workspace_bytes, per_chunk * n_ws))) return rc;
  for (int i = 0; i < 3; ++i)
    if (!host_pinned(hv[i]->data) || !device_memory(dv[i]->data)) return SAGE_ERR_INVALID_ARG;
  if (!host_pinned(out_host) || !device_memory(out_dev)) return SAGE_ERR_INVALID_ARG;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaStream_t s_alt = static_cast<cudaStream_t>(stream_alt);
  cudaStream_t s_in = static_cast<cudaStream_t>(stream_in);
  cudaStream_t s_out = static_cast<cudaStream_t>(stream_out);
  cudaEvent_t e_in = static_cast<cudaEvent_t>(event_in);
  cudaEvent_t e_comp = static_cast<cudaEvent_t>(event_compute);
  cudaEvent_t e_out = static_cast<cudaEvent_t>(event_out);
  // Each cudaStreamWaitEvent below is enqueued before the next record of the
  // same event, so it waits for the record just before it; three events serve
  // every chunk.
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  if ((rc = clear_status(workspace, s))) return rc;
  // the caller's earlier work on `stream` (users of the device buffers) first
  if (!ok(cudaEventRecord(e_in, s)) || !ok(cudaStreamWaitEvent(s_in, e_in, 0)) ||
      !ok(cudaStreamWaitEvent(s_out, e_in, 0)) || (s_alt && !ok(cudaStreamWaitEvent(s_alt, e_in, 0))))
    return SAGE_ERR_CUDA;
  const std::vector<int> chunks = host_chunks(H, hc);
  int h0 = 0;
  for (size_t j = 0; j < chunks.size(); h0 += chunks[j], ++j) {
    const int h1 = h0 + chunks[j];
    // even chunks on `stream` with the first workspace, odd ones on the
    // second stream with the second: a chunk's start overlaps the last wave
    // of the chunk before
    const bool alt = s_alt && (j & 1);
    cudaStream_t sc = alt ? s_alt : s;
    void* wsc = static_cast<char*>(workspace) + (alt ? per_chunk : 0);
    for (int i = 0; i < 3; ++i)
      if ((rc = copy_heads(const_cast<void*>(dv[i]->data), hv[i]->data, dv[i]->stride_b, dv[i]->stride_n,
                           dv[i]->stride_h, B, N, D, h0, h1, cudaMemcpyHostToDevice, s_in)))
        return rc;
    if (!ok(cudaEventRecord(e_in, s_in)) || !ok(cudaStreamWaitEvent(sc, e_in, 0))) return SAGE_ERR_CUDA;
    sage_view_bf16 cv[3];
    for (int i = 0; i < 3; ++i) {
      cv[i] = *dv[i];
      cv[i].data = static_cast<const uint16_t*>(dv[i]->data) + (int64_t)h0 * dv[i]->stride_h;
    }
    void* co = static_cast<uint16_t*>(out_dev) + (int64_t)h0 * out_stride_h;
    // the chunk's prepass by the rule of sage_attn_fwd (a chunk of a few
    // heads is small enough for the single launch up to long sequences;
    // measured on B200 with host buffers: 47.99 against 48.10 ms at B1
    // N37810 H56 D128 in chunks of four heads, 0.071 against 0.099 ms at B1
    // N256 H2 D128)
    if ((rc = fwd_body(cv[0], cv[1], cv[2], co, out_stride_b, out_stride_n, out_stride_h, B, N, h1 - h0, D,
                       sm_scale, wsc, workspace, default_prepass(B, N, h1 - h0, D), sc)))
      return rc;
    if (!ok(cudaEventRecord(e_comp, sc)) || !ok(cudaStreamWaitEvent(s_out, e_comp, 0))) return SAGE_ERR_CUDA;
    if ((rc = copy_heads(out_host, out_dev, out_stride_b, out_stride_n, out_stride_h, B, N, D, h0, h1,
                         cudaMemcpyDeviceToHost, s_out)))
      return rc;
  }
  // the caller's stream completes after the last copy-out, which follows every
  // chunk's compute (each copy-out waited for its chunk)
  if (!ok(cudaEventRecord(e_out, s_out)) || !ok(cudaStreamWaitEvent(s, e_out, 0))) return SAGE_ERR_CUDA;
  return SAGE_OK;
}

int sage_read_device_status(const void* workspace, void* stream) {
  if (!workspace) return SAGE_ERR_INVALID_ARG;
  DeviceStatus st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&st, workspace, sizeof(st), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return SAGE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return SAGE_ERR_CUDA;
  return st.code;
}

const char* sage_strerror(int code) {
  switch (code) {
    case SAGE_OK: return "success";
    case SAGE_ERR_INVALID_ARG: return "invalid argument (null pointer, negative size or stride)";
    case SAGE_ERR_UNSUPPORTED: return "unsupported (head dim not 64/128, or a misaligned pointer or stride)";
    case SAGE_ERR_WORKSPACE: return "workspace missing, not 256-byte aligned, or too small";
    case SAGE_ERR_CUDA: return "a CUDA launch or runtime call failed";
    case SAGE_ERR_TIMEOUT: return "a bounded device wait ran out (kernel abandoned its work)";
    case SAGE_ERR_DEVICE: return "a kernel flagged an inconsistent device state";
    default: return "unknown status code";
  }
}

int sage_set_mainloop(int which) {
  if (which < SAGE_MAINLOOP_DEFAULT || which > SAGE_MAINLOOP_TCGEN05_F32) return SAGE_ERR_UNSUPPORTED;
  std::call_once(g_mainloop_env_once, read_mainloop_env);
  g_mainloop.store(which);
  return SAGE_OK;
}

int sage_get_mainloop(void) { return resolved_mainloop(); }

int sage_debug_prepass_list(int B, int N, int H, int D, int grid, int* lag, long long n_items, int* items) {
  const int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  if (empty(B, N, H)) return n_items == 0 ? SAGE_OK : SAGE_ERR_INVALID_ARG;
  if (!items) return SAGE_ERR_INVALID_ARG;
  return prepass_stream_list(B, N, H, grid, lag, n_items, items);
}

int sage_debug_set_stall(int k_tile, long long wait_limit_cycles) {
  g_stall_tile.store(k_tile < 0 ? -1 : k_tile);
  g_wait_limit.store(wait_limit_cycles > 0 ? wait_limit_cycles : kDefaultWaitLimit);
  return SAGE_OK;
}

int sage_debug_qk_s32(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8, const float* k_scale,
                      const uint8_t* v_fp8, const float* v_scale, int B, int N, int H, int D, int b, int h,
                      int q_tile, int k_tile, int32_t* s_out, void* workspace, size_t workspace_bytes,
                      void* stream) {
  int rc = check_dims(B, N, H, D);
  if (rc) return rc;
  const Dims d = make_dims(B, N, H, D);
  if (!q_i8 || !q_scale || !k_i8 || !k_scale || !v_fp8 || !v_scale || !s_out || empty(B, N, H))
    return SAGE_ERR_INVALID_ARG;
  if (b < 0 || b >= B || h < 0 || h >= H || q_tile < 0 || q_tile >= d.Nq / kQTile || k_tile < 0 ||
      k_tile >= d.T64)
    return SAGE_ERR_INVALID_ARG;
  if (!aligned16(q_i8) || !aligned16(k_i8) || !aligned16(v_fp8) || !aligned16(q_scale) || !aligned16(k_scale) ||
      !aligned16(v_scale) || !aligned16(s_out))
    return SAGE_ERR_UNSUPPORTED;
  if ((rc = check_ws(workspace, workspace_bytes, plan(SAGE_OP_DEBUG_QK, d).total))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((rc = clear_status(workspace, s))) return rc;
  AttnParams p = make_params(d, q_i8, q_scale, k_i8, k_scale, v_fp8, v_scale, nullptr, 0, 0, 0, 0.0f, workspace);
  switch (resolved_mainloop()) {
    case SAGE_MAINLOOP_TCGEN05:
    case SAGE_MAINLOOP_TCGEN05_F32:
      // one CTA of the mainloop itself, which copies the scores it reads
      p.dbg_qt = q_tile;
      p.dbg_h = h;
      p.dbg_b = b;
      p.dbg_tile = k_tile;
      p.dbg_out = s_out;
      return run_mainloop(p, s);
    default:
      return launch_debug_qk_mma(p, b, h, q_tile, k_tile, s_out, s);
  }
}

}  // extern "C"
