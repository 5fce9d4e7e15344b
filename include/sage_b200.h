/*
 * sage_b200.h — C ABI of the B200 (sm_100a) quantized attention library.
 *
 * The library computes SageAttention-2-style non-causal attention:
 * INT8 Q K^T on tensor cores, an FP32 online softmax, FP8-E4M3 P V with an
 * FP16 per-K32 instantaneous buffer added in order into an FP32 output
 * accumulator, then 1/d normalisation, the V scale and a BF16 store.
 *
 * The operation is the one described in "Sage2 Blackwell Mainloop"
 * (section "Existing Contract") and "State-Ownership Architecture
 * Decision" (sections "Non-Negotiable Dataflow", the exact handoff record
 * and "Interface And Future Ulysses Layout").  Where those pages leave a
 * step open, this library takes the readings below:
 *   - K mean: FP64 sum per (b,h,d), sequential in 64-token chunks, chunk
 *     partials added in chunk order, km = float(sum / N).
 *   - Q: 32 consecutive rows per scale; K (after subtracting km): 64 rows per
 *     scale; both symmetric, scale = amax/127, byte = rint_even(x*(127/amax)).
 *   - V: one scale per (b,h,d) over all tokens, scale = amax/448,
 *     byte = E4M3 (OCP "FN", satfinite, round-to-nearest-even) of x*(448/amax).
 *   - scores s = float(S) * fl32(fl32(q_scale*k_scale) * fl32(sm_scale*log2 e)),
 *     base-2 exponentials, denominator summed from FP32 p before FP8.
 *   - PV: keys 0-31 and 32-63 of each 64-key tile are two FP16 buffers, each
 *     added into the FP32 accumulator in that order.
 *   - out = bf16(fl32(fl32(RO * fl32(1/d)) * v_scale[d])).
 *
 * Conventions shared by every entry point:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device and
 *     are owned by the caller, except the pinned host buffers that
 *     sage_attn_fwd_host copies from and to.  The library allocates nothing,
 *     frees nothing and does not synchronise the host (except
 *     sage_read_device_status).  Work is enqueued on `stream` (a
 *     cudaStream_t; NULL = legacy default stream), and on the further
 *     streams the caller passes to sage_attn_fwd_host.
 *   - Shapes: B (batch), N (tokens), H (heads), D (head dim, 64 or 128).
 *     B, N or H equal to 0 is an empty problem: SAGE_OK, nothing launched.
 *     Limits (SAGE_ERR_UNSUPPORTED beyond them): B <= 65535 and H <= 65535
 *     (grid extents), B*H <= 2^30, N <= 2^28.
 *   - BF16 views carry element strides (b, n, h); d has unit stride.  The
 *     base address and every stride must be 16-byte aligned (strides a
 *     multiple of 8 elements); three views may alias one fused projection
 *     buffer.  No input copy or transpose is made.
 *   - Return codes are synchronous argument / launch checks.  Faults found
 *     on the device (a bounded wait that ran out) are written to the status
 *     block at the start of the workspace; read them with
 *     sage_read_device_status.
 *   - Outputs are fully overwritten, padding included.
 *   - Launch order: the last prepass kernel of sage_quant_qkv, sage_quant_v
 *     and sage_attn_fwd lets the next kernel of the stream start early if
 *     that kernel was launched as a programmatic dependent (CUDA's
 *     programmatic stream serialization).  The library's mainloop is: it
 *     waits (griddepcontrol.wait) for the prepass grid to complete before it
 *     reads any quantised tensor.  A caller's own kernel launched that way
 *     after a prepass call must wait in the same way before it reads them.
 *
 * Quantised buffer layouts (all 16-byte aligned, written by the prepasses):
 *   Nq = ceil(N/128)*128, Nk = ceil(N/64)*64, G32 = ceil(N/32), T64 = Nk/64
 *   q_i8    int8   [B][H][Nq][D]   rows >= N are zero
 *   q_scale float  [B][H][G32]
 *   k_i8    int8   [B][H][Nk][D]   smoothed (K - k_mean); rows >= N zero
 *   k_scale float  [B][H][T64]
 *   k_mean  float  [B][H][D]
 *   v_fp8   uint8  [B][H][D][Nk]   E4M3, transposed (tokens contiguous);
 *                                  tokens >= N zero
 *   v_scale float  [B][H][D]
 */
#ifndef SAGE_B200_H
#define SAGE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAGE_API __attribute__((visibility("default")))
#else
#define SAGE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

enum sage_status_code {
  SAGE_OK = 0,
  SAGE_ERR_INVALID_ARG = 1,  /* null pointer, negative size, bad stride */
  SAGE_ERR_UNSUPPORTED = 2,  /* D not in {64, 128}; misaligned base or stride;
                                a size beyond the limits below */
  SAGE_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small */
  SAGE_ERR_CUDA = 4,         /* a CUDA launch or runtime call failed */
  SAGE_ERR_TIMEOUT = 5,      /* device status: a bounded wait ran out */
  SAGE_ERR_DEVICE = 6        /* device status: a kernel flagged bad state */
};

/* Which call a workspace is sized for. */
enum sage_op {
  SAGE_OP_QUANT_QK = 0,
  SAGE_OP_QUANT_V = 1,
  SAGE_OP_ATTN_FWD = 2,
  SAGE_OP_ATTN_FROM_QUANT = 3,
  SAGE_OP_DEBUG_QK = 4,
  SAGE_OP_QUANT_QKV = 5,
  SAGE_OP_ATTN_FWD_HOST = 6  /* sage_attn_fwd_host with chunks of H heads and
                                two compute streams (two chunk workspaces) */
};

/* Mainloop implementations.  DEFAULT, TCGEN05 and MMA_SYNC compute the
 * exact contract (same numerics, chosen by measurement).  TCGEN05_F32 is the
 * fast variant the pages leave to a future backend with its own contract
 * ("Vortex Exact", section "Scope"): same quantised inputs, INT8 QK^T and
 * E4M3 probabilities, but the PV products accumulate in FP32 in TMEM across
 * all tiles (no FP16 buffer per K32 slice) and the running maximum used for
 * the probabilities is raised only when a tile's maximum exceeds it by more
 * than 8 (log2 units), with the accumulator rescaled only then.  Its output
 * is held to a quality gate (cosine similarity to FP64 attention, distance
 * to the exact path), not to the oracle bit for bit.  It is never chosen by
 * DEFAULT. */
enum sage_mainloop {
  SAGE_MAINLOOP_DEFAULT = 0,     /* the fastest validated exact variant */
  SAGE_MAINLOOP_TCGEN05 = 1,     /* tcgen05 MMAs with TMEM accumulators, TMA */
  SAGE_MAINLOOP_MMA_SYNC = 2,    /* warp-level mma.sync */
  SAGE_MAINLOOP_TCGEN05_F32 = 3  /* quality-gated fast variant (see above) */
};

/* Bytes at the start of every workspace that hold the device status word. */
#define SAGE_STATUS_BYTES 256

/* A strided BF16 [B, N, H, D] view (element strides; unit stride over d). */
typedef struct sage_view_bf16 {
  const void* data;
  int64_t stride_b, stride_n, stride_h;
} sage_view_bf16;

/* Workspace size for one call `op` on a (B, N, H, D) problem.
 * Returns SAGE_OK and writes *bytes, or SAGE_ERR_INVALID_ARG. */
SAGE_API int sage_workspace_bytes(int op, int B, int N, int H, int D, size_t* bytes);

/* Prepasses for Q and K: K channel mean (FP64, reading above), K smoothing
 * and per-64-row INT8 K, per-32-row INT8 Q.  Defined by "Sage2 Blackwell
 * Mainloop", sections "Decision" (K mean/smoothing, Q quantization, K
 * subtract-mean quantization) and "Existing Contract".
 * Outputs use the layouts above.  Workspace: sage_workspace_bytes(
 * SAGE_OP_QUANT_QK, ...) bytes, 256-byte aligned. */
SAGE_API int sage_quant_qk(sage_view_bf16 q, sage_view_bf16 k, int B, int N, int H, int D,
                  int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean,
                  void* workspace, size_t workspace_bytes, void* stream);

/* Q/K producer with RMSNorm and split-half RoPE in front of the quantisation
 * (the fused strided-NHD producer of "Sage2 Blackwell Mainloop", section
 * "Completed P1 And P2"): per (b, n, h) row x of D values,
 *   ss = FP32 sum of fl32(x_d*x_d) in channel order,
 *   r  = fl32(1 / fl32(sqrt(fl32(fl32(ss/D) + eps)))),
 *   y_d = bf16(fl32(bf16(fl32(x_d*r)) * w_d)),
 *   z_j = bf16(fl32(fl32(y_j*c) - fl32(y_{j+D/2}*s))),
 *   z_{j+D/2} = bf16(fl32(fl32(y_{j+D/2}*c) + fl32(y_j*s))),  c, s = cos/sin[n][j];
 * then z goes through exactly the rules of sage_quant_qk (same outputs and
 * layouts).  wq, wk: BF16 [D]; cos_t, sin_t: FP32 [N][D/2] row-major; all
 * 16-byte aligned; eps >= 0.  The normalised rows are not stored.
 * Workspace: sage_workspace_bytes(SAGE_OP_QUANT_QK, ...). */
SAGE_API int sage_norm_rope_quant_qk(sage_view_bf16 q, sage_view_bf16 k, const void* wq, const void* wk,
                            const float* cos_t, const float* sin_t, float eps, int B, int N, int H, int D,
                            int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean,
                            void* workspace, size_t workspace_bytes, void* stream);

/* Prepass for V: per-channel amax over all tokens, scale, E4M3 bytes stored
 * transposed.  Defined by "Sage2 Blackwell Mainloop", section "Decision"
 * (V transpose/pad/permute, V scale/FP8 quantization) and section
 * "Completed P1 And P2" (one owned direct-NHD V producer).
 * Workspace: sage_workspace_bytes(SAGE_OP_QUANT_V, ...). */
SAGE_API int sage_quant_v(sage_view_bf16 v, int B, int N, int H, int D, uint8_t* v_fp8, float* v_scale,
                 void* workspace, size_t workspace_bytes, void* stream);

/* All three prepasses: the outputs of sage_quant_qk and sage_quant_v, bit
 * for bit (same K sum, same rounding), in one kernel launch (after a memset
 * of its scratch) in which K and V are read from HBM about once (the pages'
 * producer fusions, "Sage2 Blackwell Mainloop", section "Completed P1 And
 * P2").
 *   - The work is a list of 64-token tiles of one head: K statistics, V
 *     statistics, Q codes, then, a few heads later in the list, the K and V
 *     codes of the head.  Persistent CTAs take the tiles in list order, so
 *     a head's codes re-read its K and V while they are still in L2.
 *   - The K mean: each channel's FP64 sum is taken from an accumulator that
 *     the tiles add to atomically when every partial sum of the channel is
 *     exact in FP64 (a bound on the channel's exponent range, checked per
 *     channel), and from the chunk partials in chunk order otherwise; both
 *     give the chunk-order sum of the definition.
 *   - A head's code tiles wait (bounded) until all of its statistics tiles
 *     are counted in; a wait that runs out leaves SAGE_ERR_TIMEOUT in the
 *     status word, and the kernel then returns.
 *   - Any shape the separate kernels take.  On one B200 it is faster than
 *     the six separate launches up to about 128 MB of Q, K and V (0.016
 *     against 0.060 ms at B1 N256 H2 D128) and slower above (0.77 against
 *     0.59 ms at B1 N37810 H56 D128); sage_attn_fwd picks by that size.
 * Workspace: sage_workspace_bytes(SAGE_OP_QUANT_QKV, ...), 256-byte
 * aligned; concurrent calls need separate workspaces. */
SAGE_API int sage_quant_qkv(sage_view_bf16 q, sage_view_bf16 k, sage_view_bf16 v, int B, int N, int H, int D,
                   int8_t* q_i8, float* q_scale, int8_t* k_i8, float* k_scale, float* k_mean,
                   uint8_t* v_fp8, float* v_scale, void* workspace, size_t workspace_bytes, void* stream);

/* Kernel launches that sage_quant_qkv makes for this shape: 1 (0 for an
 * empty shape); a negative SAGE_ERR_* for a shape the library refuses.  No
 * counterpart in the pages (launch accounting). */
SAGE_API int sage_quant_qkv_kernels(int B, int N, int H, int D);

/* Prepass kernel launches that sage_attn_fwd makes for this shape: 1 (the
 * single launch of sage_quant_qkv, below about 128 MiB of Q, K and V) or 6
 * (the separate kernels of sage_quant_qk and sage_quant_v); 0 for an empty
 * shape; a negative SAGE_ERR_* for a shape the library refuses.  The
 * SAGE_PREPASS environment variable ("separate" or "stream", read once)
 * overrides the choice for every call.  No counterpart in the pages (launch
 * accounting). */
SAGE_API int sage_attn_fwd_prepass_kernels(int B, int N, int H, int D);

/* Fused mainloop on quantised inputs: every 64-key tile in increasing order,
 * INT8 QK^T, score scaling, online softmax, E4M3 P, two K32 FP16 PV buffers
 * added into FP32, then 1/d, V scale and the BF16 store to `out`
 * ([B, N, H, D] with element strides out_stride_*; unit stride over d).
 * Defined by "State-Ownership Architecture Decision", section
 * "Non-Negotiable Dataflow" and the exact handoff record.
 * sm_scale <= 0 selects 1/sqrt(D).
 * Workspace: sage_workspace_bytes(SAGE_OP_ATTN_FROM_QUANT, ...). */
SAGE_API int sage_attn_from_quant(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8,
                         const float* k_scale, const uint8_t* v_fp8, const float* v_scale,
                         void* out, int64_t out_stride_b, int64_t out_stride_n,
                         int64_t out_stride_h, int B, int N, int H, int D, float sm_scale,
                         void* workspace, size_t workspace_bytes, void* stream);

/* The whole path: the three prepasses (below about 128 MB of Q, K and V the
 * single launch of sage_quant_qkv, above it the separate kernels of
 * sage_quant_qk and sage_quant_v, whichever is faster there; the same bytes
 * either way; quantised tensors kept in the workspace) then the fused
 * mainloop.  Workspace: sage_workspace_bytes(SAGE_OP_ATTN_FWD, ...) bytes,
 * 256-byte aligned. */
SAGE_API int sage_attn_fwd(sage_view_bf16 q, sage_view_bf16 k, sage_view_bf16 v, void* out,
                  int64_t out_stride_b, int64_t out_stride_n, int64_t out_stride_h, int B, int N,
                  int H, int D, float sm_scale, void* workspace, size_t workspace_bytes,
                  void* stream);

/* sage_attn_fwd from and to host memory, with the copies overlapped with the
 * computation (no counterpart in the pages: a packaging of the same path for
 * callers whose tensors live on the host).  Every (b, h) head is independent
 * (per-head K mean and V scale; "Sage2 Blackwell Mainloop", section
 * "Decision"), so the heads are processed in chunks: chunk j's Q/K/V heads
 * are copied host -> device on `stream_in`, the path of sage_attn_fwd runs on
 * them on a compute stream, and their output is copied device -> host on
 * `stream_out`; the copy-in of chunk j+1 and the copy-out of chunk j-1
 * overlap the compute of chunk j.  The chunks hold 2, 2 heads, then
 * `heads_per_chunk` (<= 0 selects 4) at a time, and 2 at the end, so that
 * the first copy-in and the last copy-out, which overlap nothing, are small
 * (not one head: the copy engines move one head's 256-byte rows at half the
 * rate of wider ones).  With `stream_alt` non-NULL the chunks alternate between
 * `stream` and `stream_alt` (each with its own half of the workspace), so
 * that a chunk's first launches fill the SMs that the previous chunk's last
 * wave leaves idle.  The bytes written are those of sage_attn_fwd on the
 * whole problem.
 *   q_host, k_host, v_host  host views ([B, N, H, D] BF16, unit stride over
 *                           d) in pinned memory (cudaHostAlloc or
 *                           cudaHostRegister); they may alias one buffer.
 *   q_dev, k_dev, v_dev     device views with the same strides, which
 *                           receive the inputs (aliasing as the host views
 *                           do); each needs stride_n >= D when N > 1.
 *   out_host, out_dev       BF16 [B, N, H, D] outputs with the strides
 *                           out_stride_* (pinned host memory; device memory).
 *   workspace               sage_workspace_bytes(SAGE_OP_ATTN_FWD_HOST, B,
 *                           N, min(H, heads_per_chunk), D) bytes (half of
 *                           that suffices without `stream_alt`), 256-byte
 *                           aligned; its status word covers all chunks.
 *   stream, stream_alt,     streams of the current device (`stream` is the
 *   stream_in, stream_out   caller's: the call starts after its earlier work
 *                           and its later work starts after the last
 *                           copy-out; `stream_alt` may be NULL).
 *   event_in, event_compute,
 *   event_out               three events created by the caller (timing
 *                           disabled is best), recorded and waited on in
 *                           turn; they must not be in use elsewhere until
 *                           `stream` has passed this call.
 * Returns SAGE_ERR_INVALID_ARG when a host buffer is not pinned or a device
 * buffer is not device memory, or when host and device strides differ;
 * otherwise as sage_attn_fwd.  Everything is enqueued asynchronously; the
 * host output is complete once `stream` has completed the call. */
SAGE_API int sage_attn_fwd_host(sage_view_bf16 q_host, sage_view_bf16 k_host, sage_view_bf16 v_host,
                       sage_view_bf16 q_dev, sage_view_bf16 k_dev, sage_view_bf16 v_dev, void* out_host,
                       void* out_dev, int64_t out_stride_b, int64_t out_stride_n, int64_t out_stride_h, int B,
                       int N, int H, int D, float sm_scale, int heads_per_chunk, void* workspace,
                       size_t workspace_bytes, void* stream, void* stream_alt, void* stream_in, void* stream_out,
                       void* event_in, void* event_compute, void* event_out);

/* Where the quantised tensors of sage_attn_fwd live inside its workspace
 * (byte offsets from the workspace base, layouts above). */
typedef struct sage_fwd_layout {
  size_t q_i8, q_scale, k_i8, k_scale, k_mean, v_fp8, v_scale, total;
} sage_fwd_layout;
SAGE_API int sage_fwd_workspace_layout(int B, int N, int H, int D, sage_fwd_layout* layout);

/* Synchronises `stream`, then returns the device status word stored at the
 * start of `workspace` (SAGE_OK, SAGE_ERR_TIMEOUT, SAGE_ERR_DEVICE) or
 * SAGE_ERR_CUDA if the copy fails.  The word is cleared by each call that
 * uses the workspace. */
SAGE_API int sage_read_device_status(const void* workspace, void* stream);

/* Static English text for a return code. */
SAGE_API const char* sage_strerror(int code);

/* Select the mainloop used by sage_attn_fwd / sage_attn_from_quant for the
 * calling process.  Returns SAGE_ERR_UNSUPPORTED for an unknown value.
 * Until the first call, the environment variable SAGE_MAINLOOP ("tcgen05",
 * "mma_sync" or "tcgen05_f32", read once) may pick it.  Safe to call from
 * several threads; a launch uses the value current when it is enqueued. */
SAGE_API int sage_set_mainloop(int which);
SAGE_API int sage_get_mainloop(void);

/* Test export for failure detection.  From the next call on, the tcgen05
 * mainloop's producer withholds K/V tile `k_tile` of every CTA (< 0: none),
 * and every bounded device wait gives up after `wait_limit_cycles` SM clock
 * cycles (<= 0: the default, about one second).  In the single-launch
 * prepass (sage_quant_qkv, and sage_attn_fwd where it uses it) the first K
 * statistics tile of head unit b*H + h == k_tile is never counted in
 * instead (wait site 45).  A withheld tile makes the
 * waits run out: the kernel records SAGE_ERR_TIMEOUT in the status word,
 * abandons the work, frees its tensor memory and returns, leaving the
 * context usable.  Process-wide; call with (-1, 0) to restore. */
SAGE_API int sage_debug_set_stall(int k_tile, long long wait_limit_cycles);

/* Test export, host only (no device is touched): the work list of the
 * single-launch prepass (sage_quant_qkv) for this shape and `grid` CTAs.
 * Writes n_items = 5 * B * H * ceil(N/128) * 2 triples (kind, head unit
 * b*H + h, 64-token tile) to `items` in list order, kind 0 K statistics,
 * 1 V statistics, 2 Q codes, 3 K codes, 4 V codes, and the lag in heads to
 * `lag` (may be NULL).  The kernel's bounded waits all end because each
 * tile appears once and every head's statistics come before its codes; a
 * test checks both here.  SAGE_ERR_INVALID_ARG for a wrong n_items, grid <= 0
 * or a NULL `items`. */
SAGE_API int sage_debug_prepass_list(int B, int N, int H, int D, int grid, int* lag, long long n_items, int* items);

/* Size of the fixed device array behind sage_attn_fwd_noalloc (64 MiB). */
#define SAGE_NOALLOC_SCRATCH_BYTES (64u << 20)

/* sage_attn_fwd for callers that cannot allocate device memory (no
 * counterpart in the pages: it is a packaging of the same path).  Some
 * callers have no way to obtain a workspace: they run where cudaMalloc is
 * not allowed, or inside a framework that owns all device memory, or are
 * handed tensors but no allocator.  This entry point takes the same
 * arguments as sage_attn_fwd minus the workspace and uses instead one fixed
 * array of SAGE_NOALLOC_SCRATCH_BYTES compiled into the library, which every
 * GPU that loads the library keeps until the process exits.  It allocates
 * and frees nothing.
 *   - Problems whose sage_workspace_bytes(SAGE_OP_ATTN_FWD, ...) exceeds
 *     SAGE_NOALLOC_SCRATCH_BYTES are rejected with SAGE_ERR_WORKSPACE before
 *     anything is launched (B*H*N*D of roughly 20 million or fewer fits).
 *   - The first call on a device looks up the array's device address on
 *     that device (the device must be current); make that first call before
 *     any stream capture.
 *   - All calls share the one array and it keeps the last call's contents;
 *     each call rewrites every byte it reads.  Calls whose work can overlap
 *     on the GPU (different streams, or different host threads on one
 *     device) race on the array and must be serialised by the caller. */
SAGE_API int sage_attn_fwd_noalloc(sage_view_bf16 q, sage_view_bf16 k, sage_view_bf16 v,
                                   void* out, int64_t out_stride_b, int64_t out_stride_n,
                                   int64_t out_stride_h, int B, int N, int H, int D,
                                   float sm_scale, void* stream);

/* The device status of the last sage_attn_fwd_noalloc call on the current
 * device (no counterpart in the pages: it reads the status word that the
 * fixed array holds in place of a workspace's).  A caller of the no-alloc
 * entry point has no workspace to pass to sage_read_device_status; this call
 * does the same for the array: it waits for `stream` (the host blocks until
 * the work queued there is done) and returns SAGE_OK or the code a kernel
 * recorded, e.g. SAGE_ERR_TIMEOUT when a bounded wait ran out and the output
 * was left partly written.  SAGE_ERR_CUDA if the copy or the wait fails.  The
 * word belongs to whichever call last cleared it: read it before the next
 * no-alloc call on the device. */
SAGE_API int sage_noalloc_read_status(void* stream);

/* Test export: the int32 Q K^T scores of query tile q_tile (128 rows) and
 * key tile k_tile (64 keys) of head (b, h), written to s_out[128][64]
 * (device, row-major, natural key order).  The operation is the per-tile
 * INT8 QK^T of "State-Ownership Architecture Decision", section
 * "Non-Negotiable Dataflow".
 *   - With a tcgen05 mainloop selected, the scores come from the mainloop
 *     itself: one CTA of it runs for (b, h, q_tile) over all key tiles, with
 *     the same TMA ring, descriptors and 128-key MMAs as a forward call, and
 *     copies the tile's scores as its softmax owners read them from tensor
 *     memory.  It stores no attention output.
 *   - With the mma.sync mainloop, a one-tile kernel runs that mainloop's
 *     fragment code for the QK product.
 * The quantised tensors are those sage_quant_qk / sage_quant_v produce (the
 * scales and V are read by the mainloop run).  workspace: at least
 * sage_workspace_bytes(SAGE_OP_DEBUG_QK, ...).  Errors as for
 * sage_attn_from_quant, and SAGE_ERR_INVALID_ARG for an out-of-range
 * (b, h, q_tile, k_tile). */
SAGE_API int sage_debug_qk_s32(const int8_t* q_i8, const float* q_scale, const int8_t* k_i8, const float* k_scale,
                               const uint8_t* v_fp8, const float* v_scale, int B, int N, int H, int D, int b, int h,
                               int q_tile, int k_tile, int32_t* s_out, void* workspace, size_t workspace_bytes,
                               void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SAGE_B200_H */
