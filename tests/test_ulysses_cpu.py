"""Ulysses head-sharded attention with two and four gloo ranks on CPU: the exchange
layout (token shards -> head shards -> token shards, ragged token counts,
strided inputs) gives every rank exactly the rows the single-process
computation gives for its tokens.  The local attention here is the oracle's
(this is a test of the exchange, which the GPU path shares)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(case):
    import synth
    if case == "ragged":
        return synth.custom(1, 300, 4, 64, seed=17), [137, 163]
    if case == "four_ranks":  # batch of 2, one rank without tokens, 2 heads per rank
        return synth.custom(2, 160, 8, 64, seed=19), [50, 0, 77, 33]
    return synth.make_inputs(synth.Config("fused_small", 1, 200, 2, 128, layout="fused_qkv"), seed=18), [100, 100]


def _np(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _attend_oracle(qh, kh, vh, oh, sm_scale):
    import oracle
    res = oracle.attention(oracle.quantize(_np(qh), _np(kh), _np(vh)), sm_scale=sm_scale)
    oh.copy_(torch.from_numpy(res.view(np.int16)).view(torch.bfloat16))


def _worker(rank, world, port, case, out):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from fp8_quantized_exact_b200.ulysses import ulysses_attention
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        inp, counts = _inputs(case)
        o = sum(counts[:rank])
        sl = lambda a: torch.from_numpy(a[:, o:o + counts[rank]].view(np.int16)).view(torch.bfloat16)
        q, k, v = sl(inp.q), sl(inp.k), sl(inp.v)   # strided views into the generator's buffers
        res = torch.empty(q.shape, dtype=torch.bfloat16)
        ulysses_attention(q, k, v, res, 0.0, attend=_attend_oracle)
        out[rank] = _np(res).copy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", ["ragged", "fused", "four_ranks"])
def test_ulysses_matches_single_process(case):
    import oracle
    inp, counts = _inputs(case)
    world = len(counts)
    with mp.get_context("spawn").Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), case, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    ref = oracle.attention(oracle.quantize(inp.q, inp.k, inp.v))
    o = 0
    for r in range(world):
        got = res[r]
        assert got.shape == (inp.q.shape[0], counts[r]) + inp.q.shape[2:]
        assert np.array_equal(got, ref[:, o:o + counts[r]]), f"rank {r} differs"
        o += counts[r]
