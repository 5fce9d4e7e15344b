"""GPU path (through the C ABI) against the CPU oracle, element by element.

Bit-exact: INT8 Q/K bytes, E4M3 V bytes, every FP32 scale, the K mean, the
int32 QK^T scores and the zero padding.  Within tolerance (max abs 2e-2,
mean abs 1e-3, no NaN/Inf): the BF16 output.  Small shapes are compared in
full over tile-boundary lengths; the full-size workloads on sampled heads
and query groups (first, middle and last, which holds the ragged tail).
"""
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


def mainloops(sage_mod=None):
    import fp8_quantized_exact_b200 as s
    loops = [s.SAGE_MAINLOOP_MMA_SYNC]
    try:
        s.sage_set_mainloop(s.SAGE_MAINLOOP_DEFAULT)
        if s.sage_get_mainloop() == s.SAGE_MAINLOOP_TCGEN05:
            loops.append(s.SAGE_MAINLOOP_TCGEN05)
    except Exception:
        pass
    return loops


def check_quant(got, qz, N):
    for name in ("q8", "k8", "v8", "q_scale", "k_scale", "k_mean", "v_scale"):
        a, b = got[name], getattr(qz, name)
        assert a.shape == b.shape, name
        bad = np.argwhere(a.view(np.uint8 if a.dtype.itemsize == 1 else np.uint32) !=
                          b.view(np.uint8 if b.dtype.itemsize == 1 else np.uint32))
        assert bad.size == 0, f"{name} differs at {bad[:4].tolist()}: {a[tuple(bad[0])]} vs {b[tuple(bad[0])]}"
    assert not got["q_pad"].any() and not got["k_pad"].any() and not got["v_pad"].any()


TAILS = [1, 31, 32, 33, 63, 64, 65, 127, 128, 129, 191, 255, 1000]


@pytest.mark.parametrize("D", [128, 64])
@pytest.mark.parametrize("N", TAILS)
def test_tail_lengths_full_parity(sage, dev, N, D):
    H = 2
    inp = synth.custom(1, N, H, D, seed=1000 + N + D)
    (q, k, v), _ = gu.to_device(inp, dev)
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    ref = oracle.bf16_bits_to_float(oracle.attention(qz))
    for ml in mainloops():
        out, ws = gu.run_fwd(sage, q, k, v, ml)
        check_quant(gu.logical_quant(sage, ws, 1, N, H, D), qz, N)
        gu.compare_out(out.float().cpu().numpy(), ref, f"N={N} D={D} mainloop={ml}")


@pytest.mark.parametrize("cfg", ["small", "ragged"])
def test_small_configs_full_parity(sage, dev, cfg):
    c = synth.CONFIGS[cfg]
    inp = synth.make_inputs(c, seed=0)
    (q, k, v), _ = gu.to_device(inp, dev)
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    ref = oracle.bf16_bits_to_float(oracle.attention(qz))
    for ml in mainloops():
        out, ws = gu.run_fwd(sage, q, k, v, ml)
        check_quant(gu.logical_quant(sage, ws, c.B, c.N, c.H, c.D), qz, c.N)
        gu.compare_out(out.float().cpu().numpy(), ref, f"{cfg} mainloop={ml}")


def test_fused_projection_strides(sage, dev):
    """Q/K/V as column slices of one [B, N, 3*H*D] buffer, output strided too."""
    c = synth.Config("fused", 2, 300, 3, 128, layout="fused_qkv")
    inp = synth.make_inputs(c, seed=9)
    (q, k, v), _ = gu.to_device(inp, dev)
    assert q.stride(1) == 3 * 3 * 128
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    ref = oracle.bf16_bits_to_float(oracle.attention(qz))
    big = torch.full((2, 300, 5, 128), 7.0, dtype=torch.bfloat16, device=dev)
    out = big[:, :, 1:4, :]   # strided output view; heads 0 and 4 are canaries
    for ml in mainloops():
        out.zero_()
        gu.run_fwd(sage, q, k, v, ml, out=out)
        gu.compare_out(out.float().cpu().numpy(), ref, f"fused mainloop={ml}")
        assert (big[:, :, 0].float() == 7.0).all() and (big[:, :, 4].float() == 7.0).all()


@pytest.mark.parametrize("D", [128, 64])
def test_int32_scores_bit_exact(sage, dev, D):
    """The int32 scores as the selected mainloop itself computes them (for the
    tcgen05 mainloops: one CTA of the mainloop copies the tile its softmax
    owners read).  Key tiles cover both 64-key halves of 128-key groups 0, 3
    and 7, so the three-stage K ring has wrapped, and the ragged last tile
    (keys past N read as zero)."""
    N, H = 1000, 2
    inp = synth.custom(1, N, H, D, seed=77)
    (q, k, v), _ = gu.to_device(inp, dev)
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    for ml in mainloops():
        _, ws = gu.run_fwd(sage, q, k, v, ml)
        vw = sage.fwd_quant_views(ws, 1, N, H, D)
        dws = sage.workspace(sage.SAGE_OP_DEBUG_QK, 1, N, H, D, dev)
        s_out = torch.empty((128, 64), dtype=torch.int32, device=dev)
        for h, qt, kt in ((0, 0, 0), (1, 1, 1), (1, 2, 6), (0, 7, 7), (1, 3, 14), (0, 7, 15)):
            s_out.fill_(-1)
            sage.sage_debug_qk_s32(vw["q_i8"], vw["q_scale"], vw["k_i8"], vw["k_scale"], vw["v_fp8"],
                                   vw["v_scale"], 1, N, H, D, 0, h, qt, kt, s_out, dws)
            assert sage.sage_read_device_status(dws) == sage.SAGE_OK
            ref = oracle.qk_s32(qz, 0, h, 128 * qt, 128, 64 * kt, 64)
            assert np.array_equal(s_out.cpu().numpy(), ref), (ml, h, qt, kt)


def test_repeat_is_deterministic(sage, dev):
    inp = synth.custom(1, 777, 4, 128, seed=5)
    (q, k, v), _ = gu.to_device(inp, dev)
    for ml in mainloops():
        a, _ = gu.run_fwd(sage, q, k, v, ml)
        b, _ = gu.run_fwd(sage, q, k, v, ml)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_explicit_prepass_and_from_quant(sage, dev):
    """The three-call form (sage_quant_qk, sage_quant_v, sage_attn_from_quant)
    gives the same bytes and output as sage_attn_fwd."""
    B, N, H, D = 2, 333, 3, 64
    inp = synth.custom(B, N, H, D, seed=12)
    (q, k, v), _ = gu.to_device(inp, dev)
    shp = sage.quant_shapes(B, N, H, D)
    t = {n: torch.empty(s, dtype=dt, device=dev) for (n, s), dt in zip(
        shp.items(), (torch.int8, torch.float32, torch.int8, torch.float32, torch.float32,
                      torch.uint8, torch.float32))}
    sage.sage_quant_qk(q, k, t["q_i8"], t["q_scale"], t["k_i8"], t["k_scale"], t["k_mean"],
                       sage.workspace(sage.SAGE_OP_QUANT_QK, B, N, H, D, dev))
    sage.sage_quant_v(v, t["v_fp8"], t["v_scale"], sage.workspace(sage.SAGE_OP_QUANT_V, B, N, H, D, dev))
    for ml in mainloops():
        ref, ws = gu.run_fwd(sage, q, k, v, ml)
        views = sage.fwd_quant_views(ws, B, N, H, D)
        for n in shp:
            assert torch.equal(views[n].view(torch.uint8), t[n].view(torch.uint8)), n
        out = torch.empty_like(ref)
        sage.sage_attn_from_quant(t["q_i8"], t["q_scale"], t["k_i8"], t["k_scale"], t["v_fp8"],
                                  t["v_scale"], out, 0.0,
                                  sage.workspace(sage.SAGE_OP_ATTN_FROM_QUANT, B, N, H, D, dev))
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def _quant_buffers(sage, B, N, H, D, dev, fill):
    shp = sage.quant_shapes(B, N, H, D)
    return {n: torch.full(s, fill, dtype=dt, device=dev) for (n, s), dt in zip(
        shp.items(), (torch.int8, torch.float32, torch.int8, torch.float32, torch.float32,
                      torch.uint8, torch.float32))}


@pytest.mark.parametrize("shape,cfg", [((1, 1000, 3, 128), None), ((2, 333, 3, 64), None),
                                       ((1, 65, 2, 128), None), ((1, 1, 1, 64), None),
                                       (None, "ragged"), (None, "fused_small")])
def test_single_launch_prepass_matches_separate(sage, dev, shape, cfg):
    """sage_quant_qkv (one persistent launch) writes the same bytes, scales
    and K mean as sage_quant_qk + sage_quant_v, padding included, and the
    oracle's (bit-exact), on contiguous and fused-projection strides."""
    if cfg == "fused_small":
        inp = synth.make_inputs(synth.Config("fused_small", 1, 777, 4, 128, layout="fused_qkv"), seed=4)
    elif cfg is not None:
        inp = synth.make_inputs(synth.CONFIGS[cfg], seed=4)
    else:
        inp = synth.custom(*shape, seed=sum(shape))
    B, N, H, D = inp.q.shape
    (q, k, v), _ = gu.to_device(inp, dev)
    a = _quant_buffers(sage, B, N, H, D, dev, 7)
    b = _quant_buffers(sage, B, N, H, D, dev, 9)
    sage.sage_quant_qkv(q, k, v, a["q_i8"], a["q_scale"], a["k_i8"], a["k_scale"], a["k_mean"],
                        a["v_fp8"], a["v_scale"], sage.workspace(sage.SAGE_OP_QUANT_QKV, B, N, H, D, dev))
    sage.sage_quant_qk(q, k, b["q_i8"], b["q_scale"], b["k_i8"], b["k_scale"], b["k_mean"],
                       sage.workspace(sage.SAGE_OP_QUANT_QK, B, N, H, D, dev))
    sage.sage_quant_v(v, b["v_fp8"], b["v_scale"], sage.workspace(sage.SAGE_OP_QUANT_V, B, N, H, D, dev))
    torch.cuda.synchronize()
    for n in a:
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    got = {"q8": a["q_i8"].cpu().numpy()[:, :, :N], "k8": a["k_i8"].cpu().numpy()[:, :, :N],
           "v8": a["v_fp8"].cpu().numpy()[:, :, :, :N].transpose(0, 1, 3, 2),
           "q_scale": a["q_scale"].cpu().numpy(), "k_scale": a["k_scale"].cpu().numpy(),
           "k_mean": a["k_mean"].cpu().numpy(), "v_scale": a["v_scale"].cpu().numpy(),
           "q_pad": a["q_i8"].cpu().numpy()[:, :, N:], "k_pad": a["k_i8"].cpu().numpy()[:, :, N:],
           "v_pad": a["v_fp8"].cpu().numpy()[:, :, :, N:]}
    check_quant(got, qz, N)


def test_custom_softmax_scale(sage, dev):
    inp = synth.custom(1, 200, 2, 128, seed=21)
    (q, k, v), _ = gu.to_device(inp, dev)
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    ref = oracle.bf16_bits_to_float(oracle.attention(qz, sm_scale=0.3))
    for ml in mainloops():
        out, _ = gu.run_fwd(sage, q, k, v, ml, sm_scale=0.3)
        gu.compare_out(out.float().cpu().numpy(), ref, f"sm_scale mainloop={ml}")


def test_degenerate_inputs(sage, dev):
    """Q = 0 (uniform attention: the exact mean of V), an all-zero V channel
    (scale 0), and a constant K channel (removed exactly by the mean)."""
    N, H, D = 150, 1, 128
    rng = np.random.default_rng(0)
    vf = rng.choice(np.array([0, 1, -1, 2, -2, 4, -4], np.float32), size=(N, H, D))
    vf[0] = 4.0
    vf[:, :, 5] = 0.0
    kf = rng.standard_normal((N, H, D)).astype(np.float32).round()
    kf[:, :, 3] = 2.0
    import pins
    qb, kb, vb = pins.make_qkv(np.zeros((N, H, D), np.float32), kf, vf)
    qz = oracle.quantize(qb, kb, vb)
    ref = oracle.bf16_bits_to_float(oracle.attention(qz))
    dv = [torch.from_numpy(a).view(torch.bfloat16).to(dev) for a in (qb, kb, vb)]
    for ml in mainloops():
        out, ws = gu.run_fwd(sage, *dv, ml)
        check_quant(gu.logical_quant(sage, ws, 1, N, H, D), qz, N)
        got = out.float().cpu().numpy()
        gu.compare_out(got, ref, f"degenerate mainloop={ml}")
        assert (got[..., 5] == 0).all()


def _sampled_rows(N):
    last = (N - 1) // 32
    return sorted({0, last // 2, last})


@pytest.mark.parametrize("cfg", ["outlier", "long_fused", "d64_batch"])
def test_full_size_sampled_parity(sage, dev, cfg):
    """Full-size workloads in the benchmark's launch configuration: bytes and
    scales of two sampled heads bit-exact, output rows of three 32-row query
    groups per sampled head (first, middle, last/ragged) within tolerance,
    and every output element finite."""
    c = synth.CONFIGS[cfg]
    inp = synth.make_inputs(c, seed=0)
    (q, k, v), _ = gu.to_device(inp, dev)
    heads = [(0, 0), (c.B - 1, c.H - 1)]
    for ml in mainloops():
        out, ws = gu.run_fwd(sage, q, k, v, ml)
        # a property of every row: no NaN or infinity anywhere in the output
        assert bool(torch.isfinite(out).all()), f"{cfg} ml={ml}: non-finite output"
        got = gu.logical_quant(sage, ws, c.B, c.N, c.H, c.D, heads=heads)
        outh = out.float().cpu().numpy()
        for i, (b, h) in enumerate(heads):
            sl = lambda a: a[b:b + 1, :, h:h + 1, :]
            qz = oracle.quantize(sl(inp.q), sl(inp.k), sl(inp.v))
            one = {kk: vv[:, i:i + 1] for kk, vv in got.items()}
            check_quant(one, qz, c.N)
            gots, refs = [], []
            for g in _sampled_rows(c.N):
                r0, rows = 32 * g, min(32, c.N - 32 * g)
                ref = oracle.bf16_bits_to_float(oracle.attn_rows(qz, 0, 0, r0, rows))
                gu.compare_out(outh[b, r0:r0 + rows, h, :], ref, f"{cfg} b{b} h{h} g{g} ml={ml}")
                gots.append(outh[b, r0:r0 + rows, h, :])
                refs.append(ref)
            # scale-aware: the error relative to the output's own size, per head
            gg, rr = np.concatenate(gots).astype(np.float64), np.concatenate(refs).astype(np.float64)
            rel = np.linalg.norm(gg - rr) / np.linalg.norm(rr)
            err = np.abs(gg - rr)
            print(f"{cfg} b{b} h{h} ml={ml}: max abs {err.max():.3g} mean abs {err.mean():.3g} "
                  f"rel L2 {rel:.3g} (output rms {np.sqrt((rr ** 2).mean()):.3g})")
            bound = gu.TOL_REL_L2_MMA_SYNC if ml == sage.SAGE_MAINLOOP_MMA_SYNC else gu.TOL_REL_L2
            assert rel <= bound, f"{cfg} b{b} h{h} ml={ml}: rel L2 {rel:.3g}"
        del out, ws
        torch.cuda.empty_cache()
