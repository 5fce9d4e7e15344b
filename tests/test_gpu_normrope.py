"""RMSNorm + split-half RoPE Q/K producer (sage_norm_rope_quant_qk) against
the oracle's producer followed by its Q/K quantisation: INT8 Q/K bytes,
scales and the K mean bit-exact, padding zero; and the attention output on
the produced tensors within the output tolerance."""
import numpy as np
import pytest

import gpu_util as gu
import oracle
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
    return s


@pytest.fixture(scope="module")
def dev():
    return torch.device("cuda:0")


def producer_inputs(N, D, seed):
    """BF16 weights near 1 and RoPE tables from random angles (synthetic:
    the pages' model weights and position tables are not available)."""
    rng = np.random.default_rng(seed)
    w = rng.uniform(0.5, 1.5, (2, D)).astype(np.float32)
    wb = (w.view(np.uint32) + 0x7FFF + ((w.view(np.uint32) >> 16) & 1)) >> 16
    ang = rng.uniform(-np.pi, np.pi, (N, D // 2))
    return wb[0].astype(np.uint16), wb[1].astype(np.uint16), np.cos(ang).astype(np.float32), \
        np.sin(ang).astype(np.float32)


def run_producer(sage, dev, inp, wq, wk, cs, sn, eps):
    (q, k, v), _ = gu.to_device(inp, dev)
    B, N, H, D = q.shape
    shp = sage.quant_shapes(B, N, H, D)
    t = {n: torch.full(s, 5, dtype=dt, device=dev) for (n, s), dt in zip(
        shp.items(), (torch.int8, torch.float32, torch.int8, torch.float32, torch.float32, torch.uint8,
                      torch.float32))}
    g = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)
    wq_d, wk_d = g(wq.view(np.int16)), g(wk.view(np.int16))
    cs_d, sn_d = g(cs), g(sn)
    sage.sage_norm_rope_quant_qk(q, k, wq_d, wk_d, cs_d, sn_d, eps, t["q_i8"], t["q_scale"], t["k_i8"],
                                 t["k_scale"], t["k_mean"], sage.workspace(sage.SAGE_OP_QUANT_QK, B, N, H, D, dev))
    sage.sage_quant_v(v, t["v_fp8"], t["v_scale"], sage.workspace(sage.SAGE_OP_QUANT_V, B, N, H, D, dev))
    torch.cuda.synchronize()
    return t


def check_against_oracle(t, qz, N):
    got = {"q8": t["q_i8"].cpu().numpy()[:, :, :N], "k8": t["k_i8"].cpu().numpy()[:, :, :N],
           "q_scale": t["q_scale"].cpu().numpy(), "k_scale": t["k_scale"].cpu().numpy(),
           "k_mean": t["k_mean"].cpu().numpy()}
    for name in got:
        a, b = got[name], getattr(qz, name)
        assert a.shape == b.shape, name
        bad = np.argwhere(a.view(np.uint8 if a.dtype.itemsize == 1 else np.uint32) !=
                          b.view(np.uint8 if b.dtype.itemsize == 1 else np.uint32))
        assert bad.size == 0, f"{name} differs at {bad[:4].tolist()}"
    assert not t["q_i8"].cpu().numpy()[:, :, N:].any() and not t["k_i8"].cpu().numpy()[:, :, N:].any()


@pytest.mark.parametrize("shape", [(1, 200, 2, 128), (2, 333, 3, 64), (1, 65, 1, 128), (1, 1, 1, 64),
                                   (1, 1000, 2, 128)])
def test_norm_rope_producer_bit_exact(sage, dev, shape):
    B, N, H, D = shape
    inp = synth.custom(B, N, H, D, seed=N + H)
    wq, wk, cs, sn = producer_inputs(N, D, N)
    t = run_producer(sage, dev, inp, wq, wk, cs, sn, 1e-6)
    qz = oracle.quantize_normed(inp.q, inp.k, inp.v, wq, wk, cs, sn, 1e-6)
    check_against_oracle(t, qz, N)


def test_norm_rope_producer_fused_strides_and_eps(sage, dev):
    inp = synth.make_inputs(synth.Config("fused_small", 1, 500, 4, 128, layout="fused_qkv"), seed=2)
    wq, wk, cs, sn = producer_inputs(500, 128, 3)
    for eps in (0.0, 1e-5, 0.5):
        t = run_producer(sage, dev, inp, wq, wk, cs, sn, eps)
        check_against_oracle(t, oracle.quantize_normed(inp.q, inp.k, inp.v, wq, wk, cs, sn, eps), 500)


def test_norm_rope_producer_feeds_the_mainloop(sage, dev):
    B, N, H, D = 1, 300, 2, 128
    inp = synth.custom(B, N, H, D, seed=31)
    wq, wk, cs, sn = producer_inputs(N, D, 4)
    t = run_producer(sage, dev, inp, wq, wk, cs, sn, 1e-6)
    out = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=dev)
    sage.sage_set_mainloop(sage.SAGE_MAINLOOP_DEFAULT)
    sage.sage_attn_from_quant(t["q_i8"], t["q_scale"], t["k_i8"], t["k_scale"], t["v_fp8"], t["v_scale"], out, 0.0,
                              sage.workspace(sage.SAGE_OP_ATTN_FROM_QUANT, B, N, H, D, dev))
    qz = oracle.quantize_normed(inp.q, inp.k, inp.v, wq, wk, cs, sn, 1e-6)
    ref = oracle.bf16_bits_to_float(oracle.attention(qz))
    gu.compare_out(out.float().cpu().numpy(), ref, "norm+rope producer -> mainloop")
