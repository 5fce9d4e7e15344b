"""Helpers for the GPU parity tests: upload generator output, run the C ABI
through the binding, and bring quantised buffers back in the oracle's
logical layouts (pure indexing; no arithmetic of the method)."""
from __future__ import annotations

import numpy as np

TOL_MAX_ABS = 2e-2   # output tolerance: max |gpu - oracle| over all compared elements
TOL_MEAN_ABS = 1e-3  # and the mean of |gpu - oracle|
# per-head ||gpu - oracle|| / ||oracle|| on the sampled rows of the full-size
# workloads: the GPU and the oracle round the same operations in the same
# order except the exponential (ex2.approx against a correctly rounded exp2,
# a few ulp) and the single rounding of the exponent argument; those flip
# isolated E4M3 probability codes, each moving an output by a fraction of one
# key's weight.  1e-3 is far below the error of the quantisation itself
# (several percent) yet above what such flips can add up to (measured: at
# most 1.2e-4 for the tcgen05 mainloop).  The legacy mma.sync mainloop's FP16
# accumulator rounds inside each 32-term slice sum instead of once (see
# tests/test_gpu_golden.py), which moves outputs further (measured: up to
# 1.15e-3): its bound is 3e-3.
TOL_REL_L2 = 1e-3
TOL_REL_L2_MMA_SYNC = 3e-3


def to_device(inp, dev):
    """Upload the generator's owning buffers and rebuild the same strided views."""
    import torch
    bufs = [torch.from_numpy(np.ascontiguousarray(b)).view(torch.bfloat16).to(dev) for b in inp.buffers]
    views = []
    for name in ("q", "k", "v"):
        a = getattr(inp, name)
        for host, dv in zip(inp.buffers, bufs):
            off = a.ctypes.data - host.ctypes.data
            if 0 <= off < host.nbytes:
                st = [s // 2 for s in a.strides]
                views.append(dv.view(-1).as_strided(a.shape, st, off // 2 + dv.storage_offset()))
                break
        else:
            raise AssertionError("view not inside a buffer")
    return views, bufs


def run_fwd(sage, q, k, v, mainloop, sm_scale=0.0, out=None):
    import torch
    B, N, H, D = q.shape
    sage.sage_set_mainloop(mainloop)
    ws = sage.workspace(sage.SAGE_OP_ATTN_FWD, B, N, H, D, q.device)
    if out is None:
        out = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=q.device)
    sage.sage_attn_fwd(q, k, v, out, sm_scale, ws)
    st = sage.sage_read_device_status(ws)
    if st != sage.SAGE_OK:
        code, where, block = ws[:12].view(torch.int32).tolist()
        raise AssertionError(f"{sage.sage_strerror(st)} (wait {where}, block {block})")
    return out, ws


def logical_quant(sage, ws, B, N, H, D, heads=None):
    """The quantised tensors of a forward call's workspace in oracle layout,
    optionally only for a list of (b, h) heads (stacked as B=1, H=len)."""
    v = sage.fwd_quant_views(ws, B, N, H, D)
    get = {k: t.cpu().numpy() for k, t in v.items()}
    res = {
        "q8": get["q_i8"][:, :, :N], "q_scale": get["q_scale"], "k8": get["k_i8"][:, :, :N],
        "k_scale": get["k_scale"], "k_mean": get["k_mean"],
        "v8": get["v_fp8"][:, :, :, :N].transpose(0, 1, 3, 2), "v_scale": get["v_scale"],
        "q_pad": get["q_i8"][:, :, N:], "k_pad": get["k_i8"][:, :, N:],
        "v_pad": get["v_fp8"][:, :, :, N:],
    }
    if heads is not None:
        res = {k: np.stack([a[b, h] for b, h in heads])[None] for k, a in res.items()}
    return res


def compare_out(got, ref, what=""):
    """BF16 outputs as float32 arrays: finite, max and mean abs error bounds."""
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert err.max() <= TOL_MAX_ABS and err.mean() <= TOL_MEAN_ABS, \
        f"{what}: max abs {err.max():.4g} mean abs {err.mean():.4g}"
    return float(err.max()), float(err.mean())
