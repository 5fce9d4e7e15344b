"""The seeded input generator against its stated definition (CPU only).

The generator is counter based: splitmix64's finaliser (Steele, Lea and
Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014) keyed
by (seed, stream) and the flat element index, uniforms from its top 53
bits, Box-Muller normals, BF16 by round-to-nearest-even.  These tests
restate that definition in plain Python, tie the restated finaliser to the
splitmix64 sequence published with the algorithm, and check sampled
elements of every tensor, the independence from the thread count, and the
workloads' value distributions."""
import math

import numpy as np
import pytest
import torch

import synth

M64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15


def mix64(z):
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M64
    return z ^ (z >> 31)


def key(seed, stream):
    return mix64((seed * 0xD1B54A32D192ED03 + stream + 1) & M64)


def uniform(k, i):
    w = mix64((k + (i + 1) * GOLDEN) & M64)
    return ((w >> 11) + 0.5) * 2.0 ** -53


def normal(k, i):
    p = i >> 1
    u1, u2 = uniform(k, 2 * p), uniform(k, 2 * p + 1)
    r = math.sqrt(-2.0 * math.log(u1))
    return r * (math.sin if i & 1 else math.cos)(2.0 * math.pi * u2)


def bf16_bits(x):
    return int(torch.tensor([x], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF


def test_finaliser_matches_the_published_sequence():
    # splitmix64 from state 0: the state advances by the golden gamma and each
    # output is the finaliser of the state
    state, outs = 0, []
    for _ in range(3):
        state = (state + GOLDEN) & M64
        outs.append(mix64(state))
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


@pytest.mark.parametrize("cfg_name", ["ragged", "small"])
def test_sampled_elements_follow_the_definition(cfg_name):
    cfg = synth.CONFIGS[cfg_name]
    seed = 5
    inp = synth.make_inputs(cfg, seed=seed)
    B, N, H, D = cfg.B, cfg.N, cfg.H, cfg.D
    koff = [float(np.float32(-cfg.k_offset + 2 * cfg.k_offset * uniform(key(seed, synth.STREAM_K_OFFSET), j)))
            for j in range(H * D)]
    assert np.array_equal(inp.k_offset.ravel(), np.array(koff, np.float32))
    rng = np.random.default_rng(0)
    for name, stream in (("q", synth.STREAM_Q), ("k", synth.STREAM_K), ("v", synth.STREAM_V)):
        arr = getattr(inp, name)
        k = key(seed, stream)
        for _ in range(40):
            b, n, h, d = (int(rng.integers(0, x)) for x in (B, N, H, D))
            i = ((b * N + n) * H + h) * D + d
            x = cfg.scale * normal(k, i)
            if name == "k":
                x += koff[h * D + d]
            assert int(arr[b, n, h, d]) == bf16_bits(float(np.float32(x))), (name, b, n, h, d)


def test_thread_count_does_not_change_the_bytes():
    cfg = synth.Config("t", 2, 333, 3, 64, layout="fused_qkv", q_outlier_prob=0.05, q_outlier_mult=8.0)
    a = synth.make_inputs(cfg, seed=9, threads=1)
    b = synth.make_inputs(cfg, seed=9, threads=7)
    assert all(np.array_equal(x, y) for x, y in zip(a.buffers, b.buffers))
    assert not np.array_equal(a.q, synth.make_inputs(cfg, seed=10, threads=1).q)


def test_distributions():
    cfg = synth.Config("d", 1, 4096, 4, 64, scale=0.5, k_offset=3.0, q_outlier_prob=0.01, q_outlier_mult=8.0)
    inp = synth.make_inputs(cfg, seed=2)
    v = synth.bf16_to_float(inp.v).astype(np.float64)
    assert abs(v.mean()) < 0.01 and abs(v.std() - 0.5) < 0.01
    # K = 0.5 N(0,1) + one offset per (head, channel), fixed across tokens
    k = synth.bf16_to_float(inp.k).astype(np.float64)[0]
    assert np.all(np.abs(inp.k_offset) <= 3.0)
    assert np.abs(k.mean(axis=0) - inp.k_offset).max() < 0.05
    # about 1% of Q entries are scaled by 8: compare with the same draw without outliers
    plain = synth.make_inputs(synth.Config("d", 1, 4096, 4, 64, scale=0.5, k_offset=3.0), seed=2)
    q, q0 = synth.bf16_to_float(inp.q), synth.bf16_to_float(plain.q)
    hit = q != q0
    assert 0.008 < hit.mean() < 0.012, hit.mean()
    assert np.array_equal(q[hit], q0[hit] * 8.0)  # a power of two commutes with the BF16 rounding
