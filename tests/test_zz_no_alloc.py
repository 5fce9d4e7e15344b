"""sage_attn_fwd_noalloc, the entry point for callers that cannot allocate
device memory (its scratch is a fixed array inside the library), against
the workspace-taking sage_attn_fwd on the same inputs.

Collected last on purpose, so that a run stopping at the first failure has
run every other test before it.  It must pass alone in a fresh process and
after the rest of the suite (the scratch array then holds a previous call's
bytes)."""
import numpy as np
import pytest

import gpu_util as gu
import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


def test_noalloc_matches_workspace_entry_point():
    import fp8_quantized_exact_b200 as sage
    from fp8_quantized_exact_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    # two different problems in a row: the second call finds the first
    # call's bytes in the shared scratch array
    for shape, seed in (((1, 1000, 8, 128), 31), ((2, 333, 3, 64), 32)):
        inp = synth.custom(*shape, seed=seed)
        (q, k, v), _ = gu.to_device(inp, dev)
        ref = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        ws = sage.workspace(sage.SAGE_OP_ATTN_FWD, *shape, dev)
        sage.sage_attn_fwd(q, k, v, ref, 0.0, ws)
        assert sage.sage_read_device_status(ws) == sage.SAGE_OK
        out = torch.full(shape, 3.0, dtype=torch.bfloat16, device=dev)
        sage.sage_attn_fwd_noalloc(q, k, v, out, 0.0)
        torch.cuda.synchronize()
        gu.compare_out(out.float().cpu().numpy(), ref.float().cpu().numpy(), f"noalloc {shape}")
    # a problem needing more scratch than the array holds is refused up front
    big = sage.sage_view_bf16(4096, 0, 0, 0)
    rc = sage.lib().sage_attn_fwd_noalloc(big, big, big, 4096, 0, 0, 0, 1, 37810, 56, 128, 0.0, None)
    assert rc == sage.SAGE_ERR_WORKSPACE
