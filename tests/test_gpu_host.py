"""sage_attn_fwd_host (inputs copied in from pinned host memory and the output
copied back, chunk by chunk of heads, overlapped with the compute) against
sage_attn_fwd on device-resident copies of the same inputs: the output bytes
must be identical, for fused-QKV and contiguous layouts, ragged last chunks
and one head per chunk; unpinned host memory is rejected."""
import numpy as np
import pytest

import gpu_util as gu
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def sage():
    import fp8_quantized_exact_b200 as s
    from fp8_quantized_exact_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    s.sage_set_mainloop(s.SAGE_MAINLOOP_DEFAULT)
    return s


def host_views(inp, pin=True):
    """Pinned host copies of the generator's buffers with the same strided views."""
    bufs = []
    for b in inp.buffers:
        t = torch.from_numpy(np.ascontiguousarray(b)).view(torch.bfloat16)
        bufs.append(t.pin_memory() if pin else t.clone())
    views = []
    for name in ("q", "k", "v"):
        a = getattr(inp, name)
        for host, hb in zip(inp.buffers, bufs):
            off = a.ctypes.data - host.ctypes.data
            if 0 <= off < host.nbytes:
                views.append(hb.view(-1).as_strided(a.shape, [s // 2 for s in a.strides], off // 2))
                break
    return views, bufs


def run_host(sage, inp, heads_per_chunk, pin=True, two_streams=True):
    dev = torch.device("cuda:0")
    (qh, kh, vh), _hb = host_views(inp, pin)
    # device buffers with the host views' layout, filled with garbage first
    (qd, kd, vd), dbufs = gu.to_device(inp, dev)
    for b in dbufs:
        b.fill_(7)
    B, N, H, D = qh.shape
    out_d = torch.full((B, N, H, D), 3, dtype=torch.bfloat16, device=dev)
    out_h = torch.empty((B, N, H, D), dtype=torch.bfloat16).pin_memory() if pin else \
        torch.empty((B, N, H, D), dtype=torch.bfloat16)
    hc = heads_per_chunk if heads_per_chunk > 0 else 4
    ws = sage.workspace(sage.SAGE_OP_ATTN_FWD_HOST, B, N, min(H, hc), D, dev)
    sage.sage_attn_fwd_host(qh, kh, vh, qd, kd, vd, out_h, out_d, 0.0, ws, heads_per_chunk,
                            two_streams=two_streams)
    st = sage.sage_read_device_status(ws)
    assert st == sage.SAGE_OK, sage.sage_strerror(st)
    return out_h, out_d


@pytest.mark.parametrize("case,hpc,two", [("fused", 4, True), ("fused", 4, False), ("fused", 3, True),
                                          ("contig_b2", 4, True), ("contig_b2", 1, False), ("fused", 0, True),
                                          ("fused", 64, True), ("fused13", 2, True)])
def test_host_pipeline_equals_device_call(sage, case, hpc, two):
    # fused: 10 heads (chunks 2, 2, 4, 2); fused13: 13 heads with 2-head
    # chunks and a ragged 1-head chunk before the tail; contig_b2: B = 2, 6 heads
    if case == "fused":
        inp = synth.make_inputs(synth.Config("hf", 1, 1000, 10, 128, layout="fused_qkv"), seed=4)
    elif case == "fused13":
        inp = synth.make_inputs(synth.Config("hf13", 1, 200, 13, 64, layout="fused_qkv"), seed=8)
    else:
        inp = synth.custom(2, 333, 6, 64, seed=5)
    out_h, out_d = run_host(sage, inp, hpc, two_streams=two)
    (q, k, v), _ = gu.to_device(inp, torch.device("cuda:0"))
    ref, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_DEFAULT)
    ref = ref.cpu()
    assert torch.equal(out_h.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(out_d.cpu().view(torch.int16), ref.view(torch.int16))


def test_host_pipeline_rejects_pageable_memory(sage):
    import ctypes
    inp = synth.custom(1, 100, 2, 64, seed=6)
    with pytest.raises(ValueError):      # the binding's own check
        run_host(sage, inp, 1, pin=False)
    # the library's check, reached directly with a pageable host buffer
    dev = torch.device("cuda:0")
    (qd, kd, vd), _ = gu.to_device(inp, dev)
    q_page = torch.from_numpy(np.ascontiguousarray(inp.q)).view(torch.bfloat16)
    hv = sage.sage_view_bf16(q_page.data_ptr(), *q_page.stride()[:3])
    out_d = torch.empty(qd.shape, dtype=torch.bfloat16, device=dev)
    out_h = torch.empty(qd.shape, dtype=torch.bfloat16).pin_memory()
    ws = sage.workspace(sage.SAGE_OP_ATTN_FWD_HOST, 1, 100, 1, 64, dev)
    s_alt, s_in, s_out, evs = sage._aux_streams(dev)
    rc = sage.lib().sage_attn_fwd_host(
        hv, hv, hv, sage._view(qd), sage._view(kd), sage._view(vd), ctypes.c_void_p(out_h.data_ptr()),
        ctypes.c_void_p(out_d.data_ptr()), *out_d.stride()[:3], 1, 100, 2, 64, 0.0, 1,
        ctypes.c_void_p(ws.data_ptr()), ws.numel(), sage._stream(None), ctypes.c_void_p(s_alt.cuda_stream),
        ctypes.c_void_p(s_in.cuda_stream),
        ctypes.c_void_p(s_out.cuda_stream), *[ctypes.c_void_p(e.cuda_event) for e in evs])
    assert rc == sage.SAGE_ERR_INVALID_ARG
