"""Pins that tie the CPU oracle to facts outside itself.

Each ``pin_*`` function raises AssertionError when the oracle (optionally a
deliberately wrong build of it, ``plant > 0``) disagrees with:

* library conversions (E4M3 via ml_dtypes/torch, FP16 via NumPy, BF16 via
  torch) for the number formats;
* the hand-worked four-token example in ``tests/golden``;
* hand-worked group-boundary scales and half-way INT8 cases;
* closed forms (Q = 0 gives the exact mean of exactly-representable V, and
  the per-K32 FP16 buffers' roundings on hand-worked slice sums);
* textbook FP64 softmax attention on small shapes (cosine and norm error);
* invariants: K-offset invariance of the smoothed path, the online-softmax
  denominator, and dominance of one key;
* the online softmax against the global-maximum form, bit for bit, where
  every rescale is an exact power of two;
* brute-force integer QK^T via NumPy;
* the K channel mean against the correctly rounded mean of the exact sum.

They are collected by ``test_oracle_pins.py``; ``test_oracle_plants.py``
checks that each planted mistake fails at least one of them.
"""
from __future__ import annotations

import json
import os

import numpy as np

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def f32(x):
    return np.float32(x)


def bits_f32(s: str) -> np.float32:
    return np.array([int(s, 16)], np.uint32).view(np.float32)[0]


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> BF16 bits (exact for the BF16-representable values used here)."""
    u = np.asarray(x, np.float32).view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not representable in BF16"
    return (u >> 16).astype(np.uint16)


def make_qkv(qf, kf, vf):
    """[N, H, D] float arrays of BF16-exact values -> B=1 uint16 views."""
    return (bf16_bits(qf)[None], bf16_bits(kf)[None], bf16_bits(vf)[None])


def fp64_attention(q, k, v, sm_scale=None):
    """Textbook softmax(Q K^T * scale) V in float64 for [B, N, H, D] BF16 bits."""
    Q = synth.bf16_to_float(q).astype(np.float64)
    K = synth.bf16_to_float(k).astype(np.float64)
    V = synth.bf16_to_float(v).astype(np.float64)
    B, N, H, D = Q.shape
    sc = sm_scale if sm_scale else 1.0 / np.sqrt(D)
    out = np.zeros_like(Q)
    for b in range(B):
        for h in range(H):
            s = Q[b, :, h, :] @ K[b, :, h, :].T * sc
            s -= s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ V[b, :, h, :]
    return out


# ------------------------------------------------------------------ formats
def pin_e4m3_decode(plant=0):
    import torch
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes, plant)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def pin_e4m3_encode(plant=0):
    import ml_dtypes
    rng = np.random.default_rng(1234)
    # every representable magnitude, every midpoint between neighbours, random values
    mags = np.unique(np.abs(oracle.e4m3_decode(np.arange(127, dtype=np.uint8), plant)))
    mids = (mags[1:] + mags[:-1]) / 2
    vals = np.concatenate([mags, mids, mids * (1 + 2 ** -20), mids * (1 - 2 ** -20),
                           rng.uniform(-448, 448, 4000), rng.uniform(-1, 1, 2000) * 2.0 ** -7,
                           np.exp2(rng.uniform(-12, 8.8, 2000))]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    vals = vals[np.abs(vals) <= 448]
    ref = vals.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    got = oracle.e4m3_encode(vals, plant)
    # the library returns +0 for negative underflow; the reading keeps the sign (0x80)
    neg_zero = (ref == 0) & (vals < 0)
    ref = np.where(neg_zero, np.uint8(0x80), ref)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"E4M3 mismatch at {vals[bad[:5]]}: {got[bad[:5]]} vs {ref[bad[:5]]}"
    # saturation (satfinite) and NaN
    sat = oracle.e4m3_encode(np.array([448.0, 449.0, 464.0, 1e6, -500.0, np.inf, -np.inf], np.float32), plant)
    assert list(sat) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]
    assert oracle.e4m3_encode(np.array([np.nan], np.float32), plant)[0] & 0x7F == 0x7F


def pin_f16_round(plant=0):
    rng = np.random.default_rng(99)
    x = np.concatenate([rng.standard_normal(3000) * 1000, np.exp2(rng.uniform(-30, 16, 3000)),
                        rng.integers(-65504, 65504, 2000).astype(np.float64) + 0.5,
                        np.array([0.0, -0.0, 65504.0, 65519.99, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26])])
    x = np.concatenate([x, -x])
    ref = x.astype(np.float16).view(np.uint16)
    got = oracle.f16_round(x, plant)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"FP16 mismatch at {x[bad[:5]]}"


def pin_bf16_round(plant=0):
    import torch
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.standard_normal(5000).astype(np.float32),
                        np.exp2(rng.uniform(-130, 120, 3000)).astype(np.float32)])
    # exact ties in the low 16 bits
    ties = (rng.integers(0, 2 ** 31, 1000, dtype=np.uint32) & 0xFFFF0000 | 0x8000).view(np.float32)
    x = np.concatenate([x, ties, -x])
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round(x, plant)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------ worked example
def _worked_inputs():
    with open(os.path.join(GOLDEN, "worked_quant_4token.json")) as f:
        g = json.load(f)
    N, H, D = 4, 1, 64
    qf = np.zeros((N, H, D), np.float32); qf[:, 0, 0] = g["q_col0"]
    kf = np.zeros((N, H, D), np.float32); kf[:, 0, 0] = g["k_col0"]
    vf = np.zeros((N, H, D), np.float32); vf[:, 0, 0] = g["v_col0"]
    return g, qf, kf, vf


def pin_worked_example(plant=0):
    g, qf, kf, vf = _worked_inputs()
    q, k, v = make_qkv(qf, kf, vf)
    qz = oracle.quantize(q, k, v, plant)
    assert list(qz.q8[0, 0, :, 0]) == g["q_bytes_col0"]
    assert qz.q_scale[0, 0, 0] == bits_f32(g["q_scale_bits"])
    assert qz.k_mean[0, 0, 0] == g["k_mean_col0"] and np.all(qz.k_mean[0, 0, 1:] == 0)
    assert list(qz.k8[0, 0, :, 0]) == g["k_bytes_col0"]
    assert qz.k_scale[0, 0, 0] == bits_f32(g["k_scale_bits"])
    assert list(qz.v8[0, 0, :, 0]) == g["v_bytes_col0"]
    assert qz.v_scale[0, 0, 0] == bits_f32(g["v_scale_bits"])
    assert np.all(qz.q8[0, 0, :, 1:] == 0) and np.all(qz.v8[0, 0, :, 1:] == 0)
    # closed form with Q = 0
    q0, _, _ = make_qkv(np.zeros_like(qf), kf, vf)
    qz0 = oracle.quantize(q0, k, v, plant)
    out = oracle.bf16_bits_to_float(oracle.attention(qz0, 0.0, plant))
    assert np.all(out[0, :, 0, 0] == g["q_zero_out_col0"]), out[0, :, 0, 0]
    assert np.all(out[0, :, 0, 1:] == 0)


def pin_group_boundaries(plant=0):
    """Q: 40 rows = one full 32-row group + a ragged 8-row group; K: 70 rows =
    one 64-row block + a ragged 6-row block; V: per-channel scales.  The
    expected scales and bytes are worked by hand."""
    N, H, D = 70, 1, 64
    qf = np.zeros((N, H, D), np.float32)
    qf[5, 0, 3] = 2.0        # group 0 amax 2 -> scale 2/127, byte of 2 is 127
    qf[7, 0, 9] = -1.0       # group 0: -1 * 63.5 = -63.5 -> tie -> -64
    qf[33, 0, 1] = 0.5       # group 1 amax 0.5 -> byte 127
    qf[39, 0, 2] = -0.25     # group 1: -0.25 * 254 = -63.5 -> -64
    qf[64, 0, 0] = 4.0       # group 2 amax 4 (rows 64..69)
    kf = np.zeros((N, H, D), np.float32)
    kf[:, 0, 0] = 1.0        # constant column: removed exactly by the mean
    kf[0, 0, 1] = 70.0       # column 1 mean = 1 -> block 0 has 69 at row 0, -1 elsewhere
    kf[66, 0, 2] = 35.0      # column 2 mean 0.5 -> block 1 amax 34.5 at row 66
    vf = np.zeros((N, H, D), np.float32)
    vf[10, 0, 0] = 3.0       # channel 0 amax 3 -> scale 3/448
    vf[69, 0, 1] = -0.5      # channel 1 amax 0.5 -> byte -448 = 0xFE
    q, k, v = make_qkv(qf, kf, vf)
    qz = oracle.quantize(q, k, v, plant)
    qs = qz.q_scale[0, 0]
    assert qs.shape == (3,)
    assert qs[0] == f32(2) / f32(127) and qs[1] == f32(0.5) / f32(127) and qs[2] == f32(4) / f32(127)
    assert qz.q8[0, 0, 5, 3] == 127 and qz.q8[0, 0, 7, 9] == -64
    assert qz.q8[0, 0, 33, 1] == 127 and qz.q8[0, 0, 39, 2] == -64 and qz.q8[0, 0, 64, 0] == 127
    assert np.count_nonzero(qz.q8) == 5
    km = qz.k_mean[0, 0]
    assert km[0] == 1.0 and km[1] == 1.0 and km[2] == 0.5 and np.all(km[3:] == 0)
    ks = qz.k_scale[0, 0]
    assert ks.shape == (2,)
    assert ks[0] == f32(69) / f32(127) and ks[1] == f32(34.5) / f32(127)
    assert qz.k8[0, 0, 0, 1] == 127 and qz.k8[0, 0, 1, 1] == -2   # -1 * 127/69 = -1.84 -> -2
    assert qz.k8[0, 0, 66, 2] == 127 and qz.k8[0, 0, 65, 2] == -2  # -0.5 * 127/34.5 = -1.84
    assert qz.k8[0, 0, 3, 2] == -1                                 # block 0: -0.5 * 127/69 = -0.92
    assert qz.k8[0, 0, 64, 1] == -4                                # block 1: -1 * 127/34.5 = -3.68
    assert np.all(qz.k8[0, 0, :, 0] == 0)
    vs = qz.v_scale[0, 0]
    assert vs[0] == f32(3) / f32(448) and vs[1] == f32(0.5) / f32(448) and np.all(vs[2:] == 0)
    assert qz.v8[0, 0, 10, 0] == 0x7E and qz.v8[0, 0, 69, 1] == 0xFE


# ----------------------------------------------------------- closed forms
def pin_q_zero_mean(plant=0):
    """Q = 0: all scores 0, p = 1 exactly, d = N; V values drawn from
    {0, +-1, +-2, +-4} per channel with amax 4 quantise exactly (x * 112 is
    0, 112, 224 or 448, all E4M3 values) and the FP16 sums of 32 such terms
    are exact, so the output is the mean of V up to the final FP32/BF16
    roundings."""
    rng = np.random.default_rng(5)
    for N in (1, 31, 64, 65, 200):
        H, D = 2, 64
        vf = rng.choice(np.array([0, 1, -1, 2, -2, 4, -4], np.float32), size=(N, H, D))
        vf[0] = 4.0  # every channel has amax 4
        kf = rng.standard_normal((N, H, D)).astype(np.float32)
        kf = synth.bf16_to_float(bf16_bits_round(kf))
        q, k, v = make_qkv(np.zeros((N, H, D), np.float32), kf, vf)
        qz = oracle.quantize(q, k, v, plant)
        out = oracle.bf16_bits_to_float(oracle.attention(qz, 0.0, plant))[0]
        mean = vf.astype(np.float64).mean(axis=0)
        err = np.abs(out - mean)
        assert np.all(err <= 2.0 ** -8 * np.abs(mean) + 1e-6), (N, err.max())


def bf16_bits_round(x):
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------ FP64 brute force
def pin_fp64_bruteforce(plant=0):
    """Quantized oracle vs textbook FP64 softmax attention: cosine >= 0.995
    per head and relative L2 error <= 0.08, over tile-boundary lengths."""
    for N, H, D, qscale in ((1, 2, 128, 1.0), (31, 2, 64, 1.0), (33, 2, 128, 2.0), (64, 1, 64, 1.0),
                            (65, 2, 128, 1.0), (129, 2, 64, 3.0), (200, 2, 128, 1.5), (256, 2, 128, 1.0)):
        inp = synth.custom(1, N, H, D, seed=N)
        q = inp.q
        if qscale != 1.0:  # sharper softmax: larger logits
            q = bf16_bits_round(synth.bf16_to_float(q) * qscale)
        qz = oracle.quantize(q, inp.k, inp.v, plant)
        out = oracle.bf16_bits_to_float(oracle.attention(qz, 0.0, plant)).astype(np.float64)
        ref = fp64_attention(q, inp.k, inp.v)
        for h in range(H):
            a, r = out[0, :, h, :].ravel(), ref[0, :, h, :].ravel()
            with np.errstate(invalid="ignore"):  # a planted mistake may give NaN, which fails below
                cos = a @ r / (np.linalg.norm(a) * np.linalg.norm(r))
                rel = np.linalg.norm(a - r) / np.linalg.norm(r)
            assert cos >= 0.995 and rel <= 0.08, (N, h, cos, rel)


def pin_dominance(plant=0):
    """One key whose logit exceeds all others by about 40 (natural log units)
    takes all the weight: the output row is that key's dequantized V row up to
    the final BF16 rounding."""
    N, H, D = 150, 1, 128
    rng = np.random.default_rng(11)
    kf = rng.choice(np.array([-1, 1], np.float32), size=(N, H, D)) * 0.25
    star = 97
    kf[star] = 1.0
    qf = np.full((N, H, D), 4.0, np.float32)
    vf = synth.bf16_to_float(bf16_bits_round(rng.standard_normal((N, H, D)).astype(np.float32)))
    q, k, v = make_qkv(qf, kf, vf)
    qz = oracle.quantize(q, k, v, plant)
    out = oracle.bf16_bits_to_float(oracle.attention(qz, 0.0, plant))[0, :, 0, :]
    vdq = oracle.e4m3_decode(qz.v8[0, 0, star]) * qz.v_scale[0, 0]
    assert np.allclose(out, vdq[None, :], rtol=2 ** -7, atol=1e-6), np.abs(out - vdq).max()


# -------------------------------------------------------------- invariants
def pin_k_offset_invariance(plant=0):
    """Adding an integer offset per K channel changes km by exactly that
    offset when the columns have an exactly representable mean, so the
    smoothed K bytes, the scales and the output must not change at all."""
    N, H, D = 96, 2, 64
    rng = np.random.default_rng(3)
    half = rng.integers(-6, 7, size=(N // 2, H, D)).astype(np.float32)
    kf = np.concatenate([half, -half])          # zero column means
    qf = rng.integers(-3, 4, size=(N, H, D)).astype(np.float32)
    vf = rng.integers(-8, 9, size=(N, H, D)).astype(np.float32)
    off = rng.integers(-20, 21, size=(1, H, D)).astype(np.float32)
    q, k, v = make_qkv(qf, kf, vf)
    _, k2, _ = make_qkv(qf, kf + off, vf)
    a = oracle.quantize(q, k, v, plant)
    b = oracle.quantize(q, k2, v, plant)
    assert np.array_equal(b.k_mean, a.k_mean + off[0][None])
    assert np.array_equal(a.k8, b.k8) and np.array_equal(a.k_scale, b.k_scale)
    assert np.array_equal(oracle.attention(a, 0.0, plant), oracle.attention(b, 0.0, plant))
    # and the smoothing is real: the unsmoothed offset K would not quantise to the same bytes
    assert not np.array_equal(a.k8, oracle.quant_k(k2, np.zeros_like(a.k_mean), plant)[0])


def pin_denominator(plant=0):
    """Online softmax invariants per row: the final max is the max score and
    d = sum_j 2^(s_j - m) over all keys (FP32 p before FP8)."""
    for N in (70, 257):
        inp = synth.custom(1, N, 1, 128, seed=40 + N)
        qz = oracle.quantize(inp.q, inp.k, inp.v, plant)
        out, st = oracle.attn_rows(qz, 0, 0, 0, N, 0.0, plant, with_stats=True)
        S = qz.q8[0, 0].astype(np.int64) @ qz.k8[0, 0].astype(np.int64).T
        sl2 = np.float32(np.float64(np.float32(1 / np.sqrt(128.0))) * 1.4426950408889634074)
        g = np.arange(N) // 32
        t = np.arange(N) // 64
        c = (qz.q_scale[0, 0][g][:, None] * qz.k_scale[0, 0][t][None, :]).astype(np.float32) * sl2
        s = S.astype(np.float32) * c.astype(np.float32)
        assert np.array_equal(st[:, 0], s.max(axis=1))
        d_ref = np.exp2(s.astype(np.float64) - st[:, :1].astype(np.float64)).sum(axis=1)
        assert np.allclose(st[:, 1], d_ref, rtol=2e-5), np.abs(st[:, 1] / d_ref - 1).max()


def pin_qk_s32(plant=0):
    inp = synth.custom(1, 100, 2, 128, seed=77)
    qz = oracle.quantize(inp.q, inp.k, inp.v, plant)
    S = oracle.qk_s32(qz, 0, 1, 0, 128, 0, 128)
    ref = np.zeros((128, 128), np.int64)
    ref[:100, :100] = qz.q8[0, 1].astype(np.int64) @ qz.k8[0, 1].astype(np.int64).T
    assert np.array_equal(S, ref)


# ------------------------------------------- producer: RMSNorm + RoPE (R11)
def _rope_tables(N, half, seed):
    rng = np.random.default_rng(seed)
    ang = rng.uniform(-np.pi, np.pi, (N, half))
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def pin_norm_rope_fp64(plant=0):
    """Against RMSNorm and split-half RoPE written in float64 from their
    definitions: within the three BF16 roundings of the reading."""
    rng = np.random.default_rng(5)
    N, H, D = 6, 2, 16
    x = bf16_bits_round(rng.standard_normal((1, N, H, D)) * 1.7)
    w = bf16_bits_round(rng.uniform(0.5, 1.5, D))
    c, s_ = _rope_tables(N, D // 2, 6)
    eps = 1e-6
    z = synth.bf16_to_float(oracle.norm_rope(x, w, c, s_, eps, plant)).astype(np.float64)
    X = synth.bf16_to_float(x).astype(np.float64)
    W = synth.bf16_to_float(w).astype(np.float64)
    y = X / np.sqrt((X * X).mean(axis=-1, keepdims=True) + eps) * W
    a, b = y[..., : D // 2], y[..., D // 2:]
    C, S = c.astype(np.float64)[None, :, None, :], s_.astype(np.float64)[None, :, None, :]
    ref = np.concatenate([a * C - b * S, b * C + a * S], axis=-1)
    scale = np.concatenate([np.abs(a) + np.abs(b)] * 2, axis=-1)
    assert np.all(np.abs(z - ref) <= 2.0 ** -6 * scale + 1e-6), np.abs(z - ref).max()


def pin_norm_rope_exact(plant=0):
    """Closed forms: a constant row normalises to exactly +-1; a quarter turn
    (cos 0, sin 1) swaps the halves with a sign; a weight of 2 doubles z."""
    N, H, D = 3, 1, 8
    ones_w = bf16_bits(np.ones(D, np.float32))
    ident_c, ident_s = np.ones((N, D // 2), np.float32), np.zeros((N, D // 2), np.float32)
    const = np.stack([np.full((H, D), v, np.float32) for v in (2.0, -0.5, 3.0)])[None]
    z = synth.bf16_to_float(oracle.norm_rope(bf16_bits(const), ones_w, ident_c, ident_s, 1e-6, plant))
    assert np.array_equal(z, np.sign(const)), z
    rng = np.random.default_rng(8)
    x = bf16_bits_round(rng.standard_normal((1, N, H, D)))
    y = synth.bf16_to_float(oracle.norm_rope(x, ones_w, ident_c, ident_s, 1e-6, plant))
    qt = synth.bf16_to_float(oracle.norm_rope(x, ones_w, np.zeros_like(ident_c), np.ones_like(ident_s), 1e-6, plant))
    assert np.array_equal(qt[..., : D // 2], -y[..., D // 2:]) and np.array_equal(qt[..., D // 2:], y[..., : D // 2])
    two = bf16_bits(np.full(D, 2.0, np.float32))
    z2 = synth.bf16_to_float(oracle.norm_rope(x, two, ident_c, ident_s, 1e-6, plant))
    assert np.array_equal(z2, 2.0 * y)


def pin_int8_ties(plant=0):
    """Half-way cases of the INT8 rule (hand-worked in the golden file): the
    bytes of Q and K round to the even integer."""
    with open(os.path.join(GOLDEN, "worked_int8_ties.json")) as f:
        g = json.load(f)
    N, H, D = 64, 1, 64
    qf = np.zeros((N, H, D), np.float32)
    kf = np.zeros((N, H, D), np.float32)
    qc, kc = g["q_col0_rows0_9"], g["k_col0_rows0_11"]
    qf[: len(qc), 0, 0] = qc
    kf[: len(kc), 0, 0] = kc
    q, k, v = make_qkv(qf, kf, np.zeros((N, H, D), np.float32))
    qz = oracle.quantize(q, k, v, plant)
    assert qz.q_scale[0, 0, 0] == 1.0 and qz.k_scale[0, 0, 0] == 1.0 and qz.k_mean[0, 0, 0] == 0.0
    assert list(qz.q8[0, 0, : len(qc), 0]) == g["q_bytes_rows0_9"], qz.q8[0, 0, : len(qc), 0]
    assert list(qz.k8[0, 0, : len(kc), 0]) == g["k_bytes_rows0_11"], qz.k8[0, 0, : len(kc), 0]


def pin_f16_slice_buffers(plant=0):
    """Closed form of the per-K32 FP16 buffers (hand-worked in the golden
    file): with every probability exactly 1, RO is the in-order FP32 sum of
    the FP16-rounded slice sums, chosen so that skipping the FP16 rounding or
    merging the two slices of a tile changes the BF16 output."""
    q, k, v, want = f16_slice_case()
    qz = oracle.quantize(q, k, v, plant)
    out = oracle.bf16_bits_to_float(oracle.attention(qz, 0.0, plant))[0, :, 0, :]
    assert np.array_equal(out, np.broadcast_to(want, out.shape)), (out[0, :4], want[:4])


def f16_slice_case():
    """Inputs of the hand-worked FP16-slice fixture (B=1, N=104, H=1, D=64 BF16
    bits) and its expected output row (every row is the same): the epilogue
    bf16(fl32(fl32(RO * fl32(1/d)) * 1)) applied to the hand-worked RO."""
    import torch
    with open(os.path.join(GOLDEN, "worked_fp16_slices.json")) as f:
        g = json.load(f)
    N, H, D = g["n"], 1, 64
    vf = np.zeros((N, H, D), np.float32)
    for ch, col in g["v"].items():
        for tok, val in col.items():
            vf[int(tok), 0, int(ch)] = val
    zero = np.zeros((N, H, D), np.float32)
    q, k, v = make_qkv(zero, zero, vf)
    rcp = np.float32(1.0) / np.float32(N)
    want = np.zeros(D, np.float32)
    for ch, ro in g["ro"].items():
        want[int(ch)] = torch.tensor(np.float32(ro) * rcp).to(torch.bfloat16).float().item()
    return q, k, v, want


# ------------------------------------------------ online softmax, exactly
def _rising_max_inputs(N, seed):
    """Q, K, V for which every score is an integer in log2 units and each
    64-key tile raises every row's running maximum by exactly one.

    The score scale is exactly 1: sm_scale = fl32(ln 2) gives
    fl32(sm_scale * log2 e) = 1, and every Q group and K block has amax 127
    (one entry of 127 in a column that meets only zeros on the other side),
    so q_scale = k_scale = 1 and the bytes are the values themselves.  K
    column 0 carries the scores: tile t holds one key of value t and others
    in [t - 4, t - 2]; its mean is made an integer, so smoothing keeps every
    byte integral.  Q column 1 and K column 1 (zero mean, +-1) make the rows
    differ.  Every score lies within 8 of the row's final maximum, so every
    probability is a power of two that E4M3 holds exactly.  V is drawn from
    {0, +-1, +-2, +-4} with amax 4, whose E4M3 codes are exact."""
    rng = np.random.default_rng(seed)
    D, T = 64, -(-N // 64)
    qf = np.zeros((N, 1, D), np.float32)
    kf = np.zeros((N, 1, D), np.float32)
    qf[:, 0, 0] = 1.0
    qf[:, 0, 1] = rng.integers(0, 2, N)
    qf[::32, 0, 2] = 127.0
    tile = np.arange(N) // 64
    star = np.arange(N) % 64 == 0
    t = rng.integers(tile - 4, tile - 1)
    t[star] = tile[star]
    excess = t.sum() % N                       # lower non-maximum keys until the mean is integral
    for j in np.flatnonzero(~star & (t > tile - 4))[:excess]:
        t[j] -= 1
    assert t.sum() % N == 0, "not enough keys to adjust"
    kf[:, 0, 0] = t
    k1 = rng.integers(-1, 2, N)
    k1[star] = 0
    for j in np.flatnonzero(~star):            # zero mean: move keys towards 0 until balanced
        if k1.sum() == 0:
            break
        if k1[j] != 0 and np.sign(k1[j]) == np.sign(k1.sum()):
            k1[j] = 0
    assert k1.sum() == 0
    kf[:, 0, 1] = k1
    kf[star, 0, 3] = 127.0
    kf[np.flatnonzero(star) + 1, 0, 3] = -127.0
    vf = rng.choice(np.array([0, 1, -1, 2, -2, 4, -4], np.float32), size=(N, 1, D))
    vf[0] = 4.0
    return qf, kf, vf


def pin_online_rescale_exact(plant=0):
    """With power-of-two rescales the online softmax must equal, bit for bit,
    the same arithmetic done once against the global row maximum: every
    rescale r = 2^-1 is exact, as is its effect on the E4M3 probabilities,
    the FP16 slice sums, the FP32 accumulator and the denominator.  The
    global form here is NumPy and torch conversions only."""
    import torch
    sm = np.float32(np.log(2.0))
    for N in (256, 230, 100):
        qf, kf, vf = _rising_max_inputs(N, 7 + N)
        q, k, v = make_qkv(qf, kf, vf)
        qz = oracle.quantize(q, k, v, plant)
        got = oracle.attention(qz, float(sm), plant)[0, :, 0, :]
        S = qz.q8[0, 0].astype(np.int64) @ qz.k8[0, 0].astype(np.int64).T
        tmax = [S[:, j:j + 64].max(axis=1) for j in range(0, N, 64)]
        assert all(np.all(b == a + 1) for a, b in zip(tmax, tmax[1:])), "inputs: maxima must rise by one"
        e = S - S.max(axis=1, keepdims=True)
        assert e.min() >= -9, "inputs: a probability would underflow E4M3"
        p = np.ldexp(1.0, e)
        p8 = torch.from_numpy(p.astype(np.float32)).to(torch.float8_e4m3fn).double().numpy()
        v8 = torch.from_numpy(np.ascontiguousarray(qz.v8[0, 0])).view(torch.float8_e4m3fn).double().numpy()
        RO = np.zeros(got.shape, np.float32)
        for j0 in range(0, N, 32):  # K32 slices in order: FP16 sum, then the FP32 add
            RO = RO + (p8[:, j0:j0 + 32] @ v8[j0:j0 + 32]).astype(np.float16).astype(np.float32)
        rcp = np.float32(1.0) / p.sum(axis=1).astype(np.float32)
        o = (RO * rcp[:, None]) * qz.v_scale[0, 0][None, :]
        want = torch.from_numpy(o.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, want), (N, int((got != want).sum()))


# ------------------------------------------------------------ K mean (R1)
def f32_nearest(fr):
    """A Fraction rounded to the nearest float32, ties to even (exact: the
    float64 value from the correctly rounded Fraction division only brackets
    the answer; the Fraction comparison decides it)."""
    from fractions import Fraction
    x = np.float32(float(fr))
    cands = {x, np.nextafter(x, np.float32(np.inf)), np.nextafter(x, np.float32(-np.inf))}
    best = min(cands, key=lambda c: (abs(Fraction(float(c)) - fr), int(np.array(c).view(np.uint32)) & 1))
    return np.float32(best)


def pin_k_mean_exact(plant=0):
    """Reading R1 without trusting its summation order: on random BF16 K of
    37,810 tokens (the long-context length) with per-channel offsets of up to
    2^10 and N(0,1) noise, every channel mean equals float32(sum / N) of the
    exact rational sum, rounded once to nearest even.  The sum is exact in
    FP64 for these values (they span fewer than 53 bits), so the FP64 reading
    meets it; a sum kept in FP32 does not."""
    from fractions import Fraction
    N, D = 37810, 128
    rng = np.random.default_rng(2024)
    offs = rng.uniform(-2.0, 2.0, D) * np.exp2(rng.integers(0, 11, D))
    x = rng.standard_normal((N, D)) + offs[None, :]
    kb = bf16_bits_round(x.astype(np.float32))                     # [N, D] BF16 bits
    xf = synth.bf16_to_float(kb).astype(np.float64)
    km = oracle.k_mean(kb[None, :, None, :], plant)[0, 0]
    shift = 48                                                     # every value is a multiple of 2^-48
    scaled = xf * 2.0 ** shift
    assert np.all(scaled == np.round(scaled)) and np.abs(scaled).max() < 2.0 ** 62
    ints = scaled.astype(np.int64)
    hi, lo = ints >> 31, ints & ((1 << 31) - 1)                   # both column sums fit in int64
    sums = [(int(a) << 31) + int(b) for a, b in zip(hi.sum(axis=0), lo.sum(axis=0))]
    want = np.array([f32_nearest(Fraction(int(s), N << shift)) for s in sums], np.float32)
    bad = np.flatnonzero(km.view(np.uint32) != want.view(np.uint32))
    assert bad.size == 0, (bad[:4].tolist(), km[bad[:4]].tolist(), want[bad[:4]].tolist())


ALL_PINS = [pin_e4m3_decode, pin_e4m3_encode, pin_f16_round, pin_bf16_round, pin_worked_example,
            pin_group_boundaries, pin_q_zero_mean, pin_fp64_bruteforce, pin_dominance,
            pin_k_offset_invariance, pin_denominator, pin_qk_s32, pin_norm_rope_fp64,
            pin_norm_rope_exact, pin_int8_ties, pin_f16_slice_buffers, pin_online_rescale_exact,
            pin_k_mean_exact]
