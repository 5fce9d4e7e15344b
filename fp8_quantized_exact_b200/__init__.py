"""Python binding of the B200 quantized-attention C ABI (``include/sage_b200.h``).

Argument marshalling only: every step of the path runs in the CUDA kernels
of ``libsage_b200.so``.  PyTorch supplies device memory and streams.  The
functions keep the C names; tensors are passed where the C ABI takes device
pointers, and a non-zero return code raises :class:`SageError`.

There is no CPU fallback: if the shared library is missing or cannot be
loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_build", "libsage_b200.so")

SAGE_OK = 0
SAGE_ERR_INVALID_ARG = 1
SAGE_ERR_UNSUPPORTED = 2
SAGE_ERR_WORKSPACE = 3
SAGE_ERR_CUDA = 4
SAGE_ERR_TIMEOUT = 5
SAGE_ERR_DEVICE = 6

SAGE_OP_QUANT_QK = 0
SAGE_OP_QUANT_V = 1
SAGE_OP_ATTN_FWD = 2
SAGE_OP_ATTN_FROM_QUANT = 3
SAGE_OP_DEBUG_QK = 4
SAGE_OP_QUANT_QKV = 5
SAGE_OP_ATTN_FWD_HOST = 6

SAGE_MAINLOOP_DEFAULT = 0
SAGE_MAINLOOP_TCGEN05 = 1
SAGE_MAINLOOP_MMA_SYNC = 2
SAGE_MAINLOOP_TCGEN05_F32 = 3  # quality-gated fast variant, not the exact contract

SAGE_STATUS_BYTES = 256

# every symbol the header declares (the CPU test checks the exports)
EXPORTS = ("sage_workspace_bytes", "sage_quant_qk", "sage_quant_v", "sage_quant_qkv", "sage_quant_qkv_kernels",
           "sage_attn_fwd_prepass_kernels",
           "sage_norm_rope_quant_qk",
           "sage_attn_from_quant",
           "sage_attn_fwd", "sage_fwd_workspace_layout", "sage_read_device_status",
           "sage_strerror", "sage_set_mainloop", "sage_get_mainloop", "sage_debug_qk_s32",
           "sage_attn_fwd_noalloc", "sage_noalloc_read_status", "sage_debug_set_stall", "sage_attn_fwd_host",
           "sage_debug_prepass_list")
SAGE_NOALLOC_SCRATCH_BYTES = 64 << 20


class SageError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {sage_strerror(code)} (code {code})")


class sage_view_bf16(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("stride_b", ctypes.c_int64),
                ("stride_n", ctypes.c_int64), ("stride_h", ctypes.c_int64)]


class sage_fwd_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("q_i8", "q_scale", "k_i8", "k_scale", "k_mean", "v_fp8", "v_scale", "total")]


_lib = None


def lib():
    """Load libsage_b200.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        P, I, L64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        V = sage_view_bf16
        sig = {
            "sage_workspace_bytes": [I, I, I, I, I, ctypes.POINTER(SZ)],
            "sage_quant_qk": [V, V, I, I, I, I, P, P, P, P, P, P, SZ, P],
            "sage_quant_v": [V, I, I, I, I, P, P, P, SZ, P],
            "sage_quant_qkv": [V, V, V, I, I, I, I, P, P, P, P, P, P, P, P, SZ, P],
            "sage_quant_qkv_kernels": [I, I, I, I],
            "sage_attn_fwd_prepass_kernels": [I, I, I, I],
            "sage_norm_rope_quant_qk": [V, V, P, P, P, P, ctypes.c_float, I, I, I, I, P, P, P, P, P, P, SZ, P],
            "sage_attn_from_quant": [P, P, P, P, P, P, P, L64, L64, L64, I, I, I, I,
                                     ctypes.c_float, P, SZ, P],
            "sage_attn_fwd": [V, V, V, P, L64, L64, L64, I, I, I, I, ctypes.c_float, P, SZ, P],
            "sage_fwd_workspace_layout": [I, I, I, I, ctypes.POINTER(sage_fwd_layout)],
            "sage_read_device_status": [P, P],
            "sage_strerror": [I],
            "sage_set_mainloop": [I],
            "sage_get_mainloop": [],
            "sage_debug_qk_s32": [P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, P, SZ, P],
            "sage_attn_fwd_noalloc": [V, V, V, P, L64, L64, L64, I, I, I, I, ctypes.c_float, P],
            "sage_noalloc_read_status": [P],
            "sage_debug_set_stall": [I, ctypes.c_longlong],
            "sage_debug_prepass_list": [I, I, I, I, I, P, ctypes.c_longlong, P],
            "sage_attn_fwd_host": [V, V, V, V, V, V, P, P, L64, L64, L64, I, I, I, I, ctypes.c_float, I, P, SZ,
                                   P, P, P, P, P, P, P],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_char_p if name == "sage_strerror" else ctypes.c_int
        _lib = L
    return _lib


def sage_strerror(code: int) -> str:
    try:
        return lib().sage_strerror(int(code)).decode()
    except Exception:  # the library itself is missing
        return f"error {code}"


def _check(rc: int, what: str):
    if rc != SAGE_OK:
        raise SageError(rc, what)


def _stream(stream):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _view(t) -> sage_view_bf16:
    import torch
    if t.dtype != torch.bfloat16 or t.dim() != 4 or t.stride(3) != 1 or not t.is_cuda:
        raise ValueError("expected a CUDA bfloat16 [B, N, H, D] view with unit stride over D")
    return sage_view_bf16(t.data_ptr(), t.stride(0), t.stride(1), t.stride(2))


# ----------------------------------------------------------- C entry points
def sage_workspace_bytes(op: int, B: int, N: int, H: int, D: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().sage_workspace_bytes(op, B, N, H, D, ctypes.byref(n)), "sage_workspace_bytes")
    return n.value


def sage_fwd_workspace_layout(B: int, N: int, H: int, D: int) -> dict:
    lay = sage_fwd_layout()
    _check(lib().sage_fwd_workspace_layout(B, N, H, D, ctypes.byref(lay)), "sage_fwd_workspace_layout")
    return {f: getattr(lay, f) for f, _ in sage_fwd_layout._fields_}


def sage_quant_qk(q, k, q_i8, q_scale, k_i8, k_scale, k_mean, workspace, stream=None):
    B, N, H, D = q.shape
    _check(lib().sage_quant_qk(_view(q), _view(k), B, N, H, D, _ptr(q_i8), _ptr(q_scale),
                               _ptr(k_i8), _ptr(k_scale), _ptr(k_mean), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream)),
           "sage_quant_qk")


def sage_quant_qkv(q, k, v, q_i8, q_scale, k_i8, k_scale, k_mean, v_fp8, v_scale, workspace, stream=None):
    B, N, H, D = q.shape
    _check(lib().sage_quant_qkv(_view(q), _view(k), _view(v), B, N, H, D, _ptr(q_i8), _ptr(q_scale),
                                _ptr(k_i8), _ptr(k_scale), _ptr(k_mean), _ptr(v_fp8), _ptr(v_scale),
                                _ptr(workspace), workspace.numel() * workspace.element_size(),
                                _stream(stream)),
           "sage_quant_qkv")


def sage_attn_fwd_prepass_kernels(B, N, H, D):
    """Prepass kernel launches of sage_attn_fwd for this shape (1: the single
    launch, 6: the separate kernels; 0 for an empty shape)."""
    n = lib().sage_attn_fwd_prepass_kernels(B, N, H, D)
    if n < 0:
        _check(n, "sage_attn_fwd_prepass_kernels")
    return n


def sage_quant_qkv_kernels(B, N, H, D):
    """Kernel launches of sage_quant_qkv for this shape (1; 0 for an empty shape)."""
    n = lib().sage_quant_qkv_kernels(B, N, H, D)
    if n < 0:
        _check(n, "sage_quant_qkv_kernels")
    return n


def sage_norm_rope_quant_qk(q, k, wq, wk, cos_t, sin_t, eps, q_i8, q_scale, k_i8, k_scale, k_mean, workspace,
                            stream=None):
    B, N, H, D = q.shape
    _check(lib().sage_norm_rope_quant_qk(_view(q), _view(k), _ptr(wq), _ptr(wk), _ptr(cos_t), _ptr(sin_t),
                                         float(eps), B, N, H, D, _ptr(q_i8), _ptr(q_scale), _ptr(k_i8),
                                         _ptr(k_scale), _ptr(k_mean), _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(stream)),
           "sage_norm_rope_quant_qk")


def sage_quant_v(v, v_fp8, v_scale, workspace, stream=None):
    B, N, H, D = v.shape
    _check(lib().sage_quant_v(_view(v), B, N, H, D, _ptr(v_fp8), _ptr(v_scale), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream)),
           "sage_quant_v")


def sage_attn_from_quant(q_i8, q_scale, k_i8, k_scale, v_fp8, v_scale, out, sm_scale, workspace,
                         stream=None):
    B, N, H, D = out.shape
    _check(lib().sage_attn_from_quant(_ptr(q_i8), _ptr(q_scale), _ptr(k_i8), _ptr(k_scale),
                                      _ptr(v_fp8), _ptr(v_scale), _ptr(out), out.stride(0),
                                      out.stride(1), out.stride(2), B, N, H, D, float(sm_scale),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _stream(stream)),
           "sage_attn_from_quant")


def sage_attn_fwd(q, k, v, out, sm_scale, workspace, stream=None):
    B, N, H, D = q.shape
    if out.stride(3) != 1 or tuple(out.shape) != (B, N, H, D):
        raise ValueError("out must be [B, N, H, D] with unit stride over D")
    _check(lib().sage_attn_fwd(_view(q), _view(k), _view(v), _ptr(out), out.stride(0),
                               out.stride(1), out.stride(2), B, N, H, D, float(sm_scale),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream)),
           "sage_attn_fwd")


def sage_attn_fwd_noalloc(q, k, v, out, sm_scale, stream=None):
    """sage_attn_fwd without a workspace, for callers that cannot allocate
    device memory: the scratch is a fixed array inside the library (see the
    header for the size limit and the rule that overlapping calls race)."""
    B, N, H, D = q.shape
    if out.stride(3) != 1 or tuple(out.shape) != (B, N, H, D):
        raise ValueError("out must be [B, N, H, D] with unit stride over D")
    _check(lib().sage_attn_fwd_noalloc(_view(q), _view(k), _view(v), _ptr(out), out.stride(0),
                                       out.stride(1), out.stride(2), B, N, H, D, float(sm_scale),
                                       _stream(stream)),
           "sage_attn_fwd_noalloc")


def sage_noalloc_read_status(stream=None) -> int:
    """Wait for the stream and return the status code of the last no-alloc
    call on the current device (SAGE_OK, SAGE_ERR_TIMEOUT, ...)."""
    return int(lib().sage_noalloc_read_status(_stream(stream)))


def _host_view(t) -> sage_view_bf16:
    import torch
    if t.dtype != torch.bfloat16 or t.dim() != 4 or t.stride(3) != 1 or t.is_cuda or not t.is_pinned():
        raise ValueError("expected a pinned host bfloat16 [B, N, H, D] view with unit stride over D")
    return sage_view_bf16(t.data_ptr(), t.stride(0), t.stride(1), t.stride(2))


_aux = {}


def _aux_streams(device):
    """A second compute stream, two copy streams and three events per device,
    created once; each event is recorded once here so that it exists before
    its handle is passed on."""
    import torch
    key = torch.device(device).index
    if key not in _aux:
        with torch.cuda.device(key):
            s_alt, s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
            evs = [torch.cuda.Event() for _ in range(3)]
            for e in evs:
                e.record()
        _aux[key] = (s_alt, s_in, s_out, evs)
    return _aux[key]


def sage_attn_fwd_host(q_host, k_host, v_host, q_dev, k_dev, v_dev, out_host, out_dev, sm_scale, workspace,
                       heads_per_chunk=4, stream=None, two_streams=True):
    """sage_attn_fwd from pinned host tensors to a pinned host output, the
    copies of each chunk of heads overlapped with the compute of the previous
    one (see the header).  The device tensors receive the inputs and the
    output; they must have the host tensors' strides.  The workspace is
    workspace(SAGE_OP_ATTN_FWD_HOST, B, N, min(H, heads_per_chunk), D)."""
    B, N, H, D = q_dev.shape
    for t in (out_host, out_dev):
        if t.stride(3) != 1 or tuple(t.shape) != (B, N, H, D):
            raise ValueError("outputs must be [B, N, H, D] with unit stride over D")
    if out_host.stride() != out_dev.stride():
        raise ValueError("host and device outputs must have the same strides")
    if out_dev.dtype != out_host.dtype or not out_dev.is_cuda or not out_host.is_pinned():
        raise ValueError("out_dev must be a CUDA tensor and out_host a pinned host tensor of the same dtype")
    s_alt, s_in, s_out, evs = _aux_streams(q_dev.device)
    _check(lib().sage_attn_fwd_host(_host_view(q_host), _host_view(k_host), _host_view(v_host), _view(q_dev),
                                    _view(k_dev), _view(v_dev), ctypes.c_void_p(out_host.data_ptr()), _ptr(out_dev),
                                    out_dev.stride(0), out_dev.stride(1), out_dev.stride(2), B, N, H, D,
                                    float(sm_scale), int(heads_per_chunk), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream),
                                    ctypes.c_void_p(s_alt.cuda_stream if two_streams else None),
                                    ctypes.c_void_p(s_in.cuda_stream), ctypes.c_void_p(s_out.cuda_stream),
                                    *[ctypes.c_void_p(e.cuda_event) for e in evs]),
           "sage_attn_fwd_host")


def sage_read_device_status(workspace, stream=None) -> int:
    return lib().sage_read_device_status(_ptr(workspace), _stream(stream))


def sage_set_mainloop(which: int):
    _check(lib().sage_set_mainloop(int(which)), "sage_set_mainloop")


def sage_get_mainloop() -> int:
    return lib().sage_get_mainloop()


def sage_debug_set_stall(k_tile: int, wait_limit_cycles: int = 0):
    _check(lib().sage_debug_set_stall(int(k_tile), int(wait_limit_cycles)), "sage_debug_set_stall")


def sage_debug_prepass_list(B: int, N: int, H: int, D: int, grid: int):
    """The single-launch prepass's work list on the host: (lag, int32 array of
    (kind, head unit, 64-token tile) rows in list order)."""
    import numpy as np
    n = 5 * B * H * (-(-N // 128)) * 2
    items = np.zeros((n, 3), dtype=np.int32)
    lag = ctypes.c_int(0)
    _check(lib().sage_debug_prepass_list(B, N, H, D, grid, ctypes.byref(lag), n, items.ctypes.data),
           "sage_debug_prepass_list")
    return lag.value, items


def sage_debug_qk_s32(q_i8, q_scale, k_i8, k_scale, v_fp8, v_scale, B, N, H, D, b, h, q_tile, k_tile, s_out,
                      workspace, stream=None):
    _check(lib().sage_debug_qk_s32(_ptr(q_i8), _ptr(q_scale), _ptr(k_i8), _ptr(k_scale), _ptr(v_fp8),
                                   _ptr(v_scale), B, N, H, D, b, h, q_tile, k_tile, _ptr(s_out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
           "sage_debug_qk_s32")


# ------------------------------------------------------- tensor conveniences
def quant_shapes(B: int, N: int, H: int, D: int) -> dict:
    """Shapes of the quantised buffers (layouts of include/sage_b200.h)."""
    Nq = -(-N // 128) * 128
    T64 = -(-N // 64)
    Nk = T64 * 64
    G32 = -(-N // 32)
    return {"q_i8": (B, H, Nq, D), "q_scale": (B, H, G32), "k_i8": (B, H, Nk, D),
            "k_scale": (B, H, T64), "k_mean": (B, H, D), "v_fp8": (B, H, D, Nk),
            "v_scale": (B, H, D)}


def workspace(op: int, B: int, N: int, H: int, D: int, device="cuda"):
    """A workspace tensor for one call (uint8, 256-byte aligned by the allocator)."""
    import torch
    n = max(sage_workspace_bytes(op, B, N, H, D), SAGE_STATUS_BYTES)
    return torch.empty(n, dtype=torch.uint8, device=device)


def fwd_quant_views(ws, B: int, N: int, H: int, D: int) -> dict:
    """Views of the quantised tensors that sage_attn_fwd leaves in its workspace."""
    import torch
    lay = sage_fwd_workspace_layout(B, N, H, D)
    shp = quant_shapes(B, N, H, D)
    dt = {"q_i8": torch.int8, "q_scale": torch.float32, "k_i8": torch.int8,
          "k_scale": torch.float32, "k_mean": torch.float32, "v_fp8": torch.uint8,
          "v_scale": torch.float32}
    out = {}
    for name, shape in shp.items():
        n = 1
        for s in shape:
            n *= s
        es = torch.empty((), dtype=dt[name]).element_size()
        out[name] = ws[lay[name]:lay[name] + n * es].view(dt[name]).view(shape)
    return out


def attention(q, k, v, out=None, sm_scale: float = 0.0, ws=None, stream=None):
    """Quantized attention of BF16 [B, N, H, D] CUDA views; returns BF16 [B, N, H, D]."""
    import torch
    B, N, H, D = q.shape
    if out is None:
        out = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=q.device)
    if ws is None:
        ws = workspace(SAGE_OP_ATTN_FWD, B, N, H, D, q.device)
    sage_attn_fwd(q, k, v, out, sm_scale, ws, stream)
    return out
