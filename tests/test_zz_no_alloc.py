"""sage_attn_fwd_noalloc, the entry point for callers that cannot allocate
device memory (its scratch is a fixed array inside the library), against
the workspace-taking sage_attn_fwd on the same inputs.

Collected last on purpose, so that a run stopping at the first failure has
run every other test before it.  It must pass alone in a fresh process and
after the rest of the suite (the scratch array then holds a previous call's
bytes)."""
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
    torch.cuda.set_device(torch.device("cuda:0"))
    return s


def test_noalloc_matches_workspace_entry_point(sage):
    dev = torch.device("cuda:0")
    # two different problems in a row: the second call finds the first
    # call's bytes in the shared scratch array.  Both calls run the same
    # deterministic kernels on the same inputs, so the bytes must agree.
    for shape, seed in (((1, 1000, 8, 128), 31), ((2, 333, 3, 64), 32)):
        inp = synth.custom(*shape, seed=seed)
        (q, k, v), _ = gu.to_device(inp, dev)
        ref = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        ws = sage.workspace(sage.SAGE_OP_ATTN_FWD, *shape, dev)
        sage.sage_attn_fwd(q, k, v, ref, 0.0, ws)
        assert sage.sage_read_device_status(ws) == sage.SAGE_OK
        out = torch.full(shape, 3.0, dtype=torch.bfloat16, device=dev)
        sage.sage_attn_fwd_noalloc(q, k, v, out, 0.0)
        assert sage.sage_noalloc_read_status() == sage.SAGE_OK
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"noalloc {shape}"
    # a problem needing more scratch than the array holds is refused up front
    big = sage.sage_view_bf16(4096, 0, 0, 0)
    rc = sage.lib().sage_attn_fwd_noalloc(big, big, big, 4096, 0, 0, 0, 1, 37810, 56, 128, 0.0, None)
    assert rc == sage.SAGE_ERR_WORKSPACE


def test_noalloc_reports_a_device_timeout(sage):
    """A bounded wait that runs out inside a no-alloc call (the tcgen05
    producer withholds one K/V tile) reaches the caller through
    sage_noalloc_read_status; the next call succeeds."""
    dev = torch.device("cuda:0")
    sage.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT)
    if sage.sage_get_mainloop() != sage.SAGE_MAINLOOP_TCGEN05:
        pytest.skip("the bounded waits live in the tcgen05 mainloop")
    shape = (1, 700, 2, 128)
    inp = synth.custom(*shape, seed=4)
    (q, k, v), _ = gu.to_device(inp, dev)
    out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    try:
        sage.sage_debug_set_stall(3, 2_000_000)  # about 1 ms per wait
        sage.sage_attn_fwd_noalloc(q, k, v, out, 0.0)
        st = sage.sage_noalloc_read_status()
    finally:
        sage.sage_debug_set_stall(-1, 0)
    assert st == sage.SAGE_ERR_TIMEOUT, st
    ref = torch.empty(shape, dtype=torch.bfloat16, device=dev)
    sage.sage_attn_fwd(q, k, v, ref, 0.0, sage.workspace(sage.SAGE_OP_ATTN_FWD, *shape, dev))
    sage.sage_attn_fwd_noalloc(q, k, v, out, 0.0)
    assert sage.sage_noalloc_read_status() == sage.SAGE_OK
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
