"""Failure detection on the GPU without a fault: the tcgen05 producer is
told to withhold one K/V tile, so the bounded waits behind it run out after
a short limit.  The kernel must report SAGE_ERR_TIMEOUT through the status
word, abandon the work, free its tensor memory and return; the next call on
the same context must succeed and match the oracle."""
import numpy as np
import pytest

import gpu_util as gu
import oracle
import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_withheld_tile_times_out_and_context_survives():
    import fp8_quantized_exact_b200 as sage
    from fp8_quantized_exact_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    dev = torch.device("cuda:0")
    sage.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT)
    if sage.sage_get_mainloop() != sage.SAGE_MAINLOOP_TCGEN05:
        pytest.skip("the bounded waits live in the tcgen05 mainloop")
    inp = synth.custom(1, 700, 2, 128, seed=4)
    (q, k, v), _ = gu.to_device(inp, dev)
    B, N, H, D = q.shape
    ws = sage.workspace(sage.SAGE_OP_ATTN_FWD, B, N, H, D, dev)
    out = torch.empty_like(q)
    try:
        sage.sage_debug_set_stall(3, 2_000_000)  # about 1 ms per wait
        sage.sage_attn_fwd(q, k, v, out, 0.0, ws)
        st = sage.sage_read_device_status(ws)
        code, where, block = ws[:12].view(torch.int32).tolist()
    finally:
        sage.sage_debug_set_stall(-1, 0)
    assert st == sage.SAGE_ERR_TIMEOUT and code == st, (st, where, block)
    # a wait of the mainloop gave up (the single-launch prepass, which this
    # shape runs, has sites 45-47 and no head unit 3 to withhold here)
    assert 0 < where < 40 and 0 <= block < (N + 127) // 128 * H * B
    # the context is still usable and the next call is correct
    out2, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_TCGEN05)
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    gu.compare_out(out2.float().cpu().numpy(), oracle.bf16_bits_to_float(oracle.attention(qz)), "after timeout")


def test_timeout_inside_the_host_pipeline_reaches_its_status_word():
    # a withheld tile in every chunk of sage_attn_fwd_host (chunks on both
    # compute streams): the one status word of its workspace reports the
    # timeout, and the next call gives the bytes of sage_attn_fwd
    import fp8_quantized_exact_b200 as sage
    from fp8_quantized_exact_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    dev = torch.device("cuda:0")
    sage.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT)
    if sage.sage_get_mainloop() != sage.SAGE_MAINLOOP_TCGEN05:
        pytest.skip("the bounded waits live in the tcgen05 mainloop")
    inp = synth.custom(1, 700, 8, 128, seed=7)
    host = [torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).pin_memory()
            for a in (inp.q, inp.k, inp.v)]
    (q, k, v), _ = gu.to_device(inp, dev)
    B, N, H, D = q.shape
    out_d = torch.empty_like(q)
    out_h = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    ws = sage.workspace(sage.SAGE_OP_ATTN_FWD_HOST, B, N, 2, D, dev)
    try:
        sage.sage_debug_set_stall(3, 2_000_000)
        sage.sage_attn_fwd_host(*host, q, k, v, out_h, out_d, 0.0, ws, 2)
        st = sage.sage_read_device_status(ws)
    finally:
        sage.sage_debug_set_stall(-1, 0)
    assert st == sage.SAGE_ERR_TIMEOUT, sage.sage_strerror(st)
    sage.sage_attn_fwd_host(*host, q, k, v, out_h, out_d, 0.0, ws, 2)
    assert sage.sage_read_device_status(ws) == sage.SAGE_OK
    ref, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_TCGEN05)
    assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16))
