"""Ulysses wrapper on one GPU: a one-rank NCCL group runs the real exchanges
and the library's attention on the strided head-shard views.  The output is
checked against the CPU oracle's attention on the same inputs (within the
output tolerance), and against a direct sage_attn_fwd call bit for bit (the
exchange is a pure relayout).  Several ranks are covered by the two- and
four-rank CPU tests."""
import datetime
import os
import socket

import pytest

import gpu_util as gu
import oracle
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.fixture(scope="module")
def sage():
    import fp8_quantized_exact_b200 as s
    from fp8_quantized_exact_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    return s


@pytest.mark.parametrize("shape,layout", [((1, 500, 4, 128), "fused_qkv"), ((2, 333, 2, 64), "contiguous")])
def test_one_rank_ulysses_equals_direct_call(sage, shape, layout):
    import torch.distributed as dist
    from fp8_quantized_exact_b200.ulysses import ulysses_attention
    dev = torch.device("cuda:0")
    B, N, H, D = shape
    inp = synth.make_inputs(synth.Config("u", B, N, H, D, layout=layout), seed=N)
    (q, k, v), _ = gu.to_device(inp, dev)
    sage.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT)
    ref, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_DEFAULT)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=dev)
    try:
        out = torch.empty_like(ref)
        ulysses_attention(q, k, v, out)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    want = oracle.bf16_bits_to_float(oracle.attention(qz))
    gu.compare_out(out.float().cpu().numpy(), want, f"ulysses {shape} {layout}")
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
