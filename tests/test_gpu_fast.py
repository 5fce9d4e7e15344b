"""Quality gate of the fast tcgen05 variant (FP32 accumulation in TMEM and a
conditionally raised running maximum), which is not held to the oracle bit
for bit: the pages leave such a backend to its own contract with a quality
gate ("Vortex Exact", section "Scope").

Gate, per (b, h) head, against FP64 attention on the unquantised BF16
inputs and against the exact GPU path on the same inputs:
  - cosine similarity to FP64 >= 0.995 (the bar the quantised oracle itself
    clears), and not below the exact path's own cosine by more than 0.002;
  - relative L2 error to FP64 at most 1.25x the exact path's, plus 1e-3;
  - mean abs distance to the exact path <= FAST_MEAN_ABS, no NaN/Inf.
Element-wise closeness to the exact path is not asked for: the
probabilities are rounded to E4M3 relative to a different maximum, so with
peaked attention single outputs move by a few E4M3 steps of their weight.
Inputs include a case whose score maxima jump by far more than 2^8 after
the first tiles, so that the in-TMEM rescale of the accumulator runs.
"""
import numpy as np
import pytest

import gpu_util as gu
import synth

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

COS_MIN = 0.995
COS_SLACK = 0.002
REL_L2_FACTOR = 1.25
REL_L2_SLACK = 1e-3
FAST_MEAN_ABS = 1e-2


@pytest.fixture(scope="module")
def sage():
    import fp8_quantized_exact_b200 as s
    from fp8_quantized_exact_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    s.sage_set_mainloop(s.SAGE_MAINLOOP_DEFAULT)
    if s.sage_get_mainloop() != s.SAGE_MAINLOOP_TCGEN05:
        pytest.skip("tcgen05 mainloop not available")
    return s


@pytest.fixture(scope="module")
def dev():
    return torch.device("cuda:0")


def fp64_attention(inp, sm_scale=None):
    """softmax(Q K^T * sm_scale) V per head in float64 on the BF16 inputs."""
    q = synth.bf16_to_float(inp.q).astype(np.float64)
    k = synth.bf16_to_float(inp.k).astype(np.float64)
    v = synth.bf16_to_float(inp.v).astype(np.float64)
    B, N, H, D = q.shape
    sc = 1.0 / np.sqrt(D) if sm_scale is None else sm_scale
    out = np.empty((B, N, H, D))
    for b in range(B):
        for h in range(H):
            s = q[b, :, h] @ k[b, :, h].T * sc
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            out[b, :, h] = (p @ v[b, :, h]) / p.sum(axis=1, keepdims=True)
    return out


def head_cosines(got, ref):
    B, N, H, D = ref.shape
    cs = []
    for b in range(B):
        for h in range(H):
            x, y = got[b, :, h].ravel(), ref[b, :, h].ravel()
            cs.append(float(x @ y / max(np.linalg.norm(x) * np.linalg.norm(y), 1e-300)))
    return np.array(cs)


def head_rel_l2(got, ref):
    B, N, H, D = ref.shape
    return np.array([np.linalg.norm(got[b, :, h] - ref[b, :, h]) / max(np.linalg.norm(ref[b, :, h]), 1e-300)
                     for b in range(B) for h in range(H)])


def gate(sage, dev, inp, what):
    (q, k, v), _bufs = gu.to_device(inp, dev)
    fast, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_TCGEN05_F32)
    exact, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_TCGEN05)
    sage.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT)
    fast = fast.float().cpu().numpy()
    exact = exact.float().cpu().numpy()
    assert np.isfinite(fast).all(), f"{what}: non-finite output"
    ref = fp64_attention(inp)
    cf, ce = head_cosines(fast, ref), head_cosines(exact, ref)
    assert cf.min() >= COS_MIN, f"{what}: cosine {cf.min():.5f} < {COS_MIN}"
    assert (cf >= ce - COS_SLACK).all(), f"{what}: cosine {cf.min():.5f} vs exact {ce.min():.5f}"
    lf, le = head_rel_l2(fast, ref), head_rel_l2(exact, ref)
    assert (lf <= REL_L2_FACTOR * le + REL_L2_SLACK).all(), \
        f"{what}: relative L2 {lf.max():.4g} vs exact {le.max():.4g}"
    err = np.abs(fast.astype(np.float64) - exact.astype(np.float64))
    assert err.mean() <= FAST_MEAN_ABS, f"{what}: vs exact mean abs {err.mean():.4g}"
    print(f"{what}: cos {cf.min():.5f} (exact {ce.min():.5f}) relL2 {lf.max():.4g} (exact {le.max():.4g}) "
          f"vs exact max {err.max():.3g} mean {err.mean():.3g}")
    return cf.min(), float(err.max()), float(err.mean())


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("N", [1, 33, 64, 65, 200, 1000])
def test_fast_quality_tails(sage, dev, N, D):
    gate(sage, dev, synth.custom(1, N, 2, D, seed=N + D), f"N={N} D={D}")


@pytest.mark.parametrize("cfg", ["small", "ragged"])
def test_fast_quality_configs(sage, dev, cfg):
    gate(sage, dev, synth.make_inputs(synth.CONFIGS[cfg], seed=3), cfg)


def _scale_keys(inp, start, mult):
    """Multiply the K rows from token `start` on by `mult` (BF16 round to
    nearest even), in the generator's own buffer."""
    k = inp.k
    f = synth.bf16_to_float(k) * np.float32(mult)
    bits = f.view(np.uint32).astype(np.uint64)
    rounded = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)
    k[:, start:] = rounded[:, start:]


@pytest.mark.parametrize("D", [128, 64])
def test_fast_rescale_path(sage, dev, D):
    # scores of the late keys are ~4x larger: the per-row maximum jumps by far
    # more than 8 (log2 units) after the first tiles, so the accumulator rows
    # are rescaled in TMEM at least once
    inp = synth.custom(1, 700, 2, D, seed=11, k_offset=0.0)
    _scale_keys(inp, 300, 4.0)
    gate(sage, dev, inp, f"rescale D={D}")


def test_fast_outlier_sampled(sage, dev):
    # the outlier workload's distribution (1% of Q entries x8) on a shape the
    # FP64 reference finishes quickly
    cfg = synth.Config("outlier_small", 1, 2048, 4, 128, scale=0.5, k_offset=3.0,
                       q_outlier_prob=0.01, q_outlier_mult=8.0)
    gate(sage, dev, synth.make_inputs(cfg, seed=5), "outlier_small")


def test_fast_repeat_is_deterministic(sage, dev):
    inp = synth.custom(1, 1000, 4, 128, seed=9)
    (q, k, v), _ = gu.to_device(inp, dev)
    a, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_TCGEN05_F32)
    b, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_TCGEN05_F32)
    sage.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_fast_repeat_with_rescales_status_and_bits(sage, dev):
    # hundreds of CTAs, each rescaling its accumulator on several tiles (the
    # key scale doubles three times along the sequence), launched repeatedly:
    # every launch must end with a clean status (no bounded wait ran out) and
    # give the same bits
    inp = synth.custom(1, 4096, 8, 128, seed=21, k_offset=0.0)
    for start in (1024, 2048, 3072):
        _scale_keys(inp, start, 2.0)
    (q, k, v), _ = gu.to_device(inp, dev)
    ref = None
    for _ in range(8):
        out, _ = gu.run_fwd(sage, q, k, v, sage.SAGE_MAINLOOP_TCGEN05_F32)
        if ref is None:
            ref = out.clone()
        else:
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    sage.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT)
