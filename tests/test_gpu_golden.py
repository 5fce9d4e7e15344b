"""Hand-worked and exactly-known cases through the GPU path (the C ABI), bit
for bit against the oracle, and a large-magnitude Q/K case within tolerance.

* The FP16-slice fixture (tests/golden/worked_fp16_slices.json): Q = K = 0,
  so every probability is exactly 1, and V slice sums chosen so that the
  FP16 rounding of each K32 buffer survives into the BF16 output ("Sage2
  Blackwell Mainloop", section Existing Contract: the fp32 + fp16
  instantaneous-buffer accumulation; "State-Ownership Architecture
  Decision", section Non-Negotiable Dataflow: two K32 FP16 PV MMAs per tile,
  each added into the FP32 RO in order).  It shows whether the tensor core's
  FP16 accumulator rounds the 32-term sum once, as the oracle does.
* Integer scores whose running maximum rises by one every tile, so every
  old-max rescale is an exact power of two ("State-Ownership Architecture
  Decision", exact handoff record: ro_rescale applied before the tile's PV).
* Q and K with amax near 122, so that the score scale c is about 0.12 and
  the exponent arguments reach hundreds of log2 units.
"""
import numpy as np
import pytest

import gpu_util as gu
import oracle
import pins
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


EXACT = {"tcgen05": 1, "mma_sync": 2}  # the exact mainloops (SAGE_MAINLOOP_* values)
# The legacy mma.sync m16n8k32 E4M3 MMA with an FP16 accumulator does not round
# a K32 slice sum once: on this fixture it returns 448 where the exact sum
# 448.1875 rounds to 448.25 (consistent with rounding to FP16 inside the
# 32-term sum), so channels 1 and 2 come out 0 instead of +-0.5/104.  The
# tcgen05 kind::f8f6f4 MMA with an FP16 accumulator matches the single
# rounding bit for bit.  Measured on B200.
MMA_SYNC_F16 = "mma.sync's FP16 accumulator does not round the 32-term slice sum once (measured on B200)"


def _upload(dev, *arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev) for a in arrs]


def _bits(out):
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


MAINLOOPS = pytest.mark.parametrize("ml", sorted(EXACT.values()), ids=sorted(EXACT, key=EXACT.get))


@pytest.mark.parametrize("ml", [1, pytest.param(2, marks=pytest.mark.xfail(strict=True, reason=MMA_SYNC_F16))],
                         ids=["tcgen05", "mma_sync"])
def test_f16_slice_fixture_bit_exact(sage, dev, ml):
    q, k, v, want = pins.f16_slice_case()
    ref_bits = oracle.attention(oracle.quantize(q, k, v))
    assert np.array_equal(oracle.bf16_bits_to_float(ref_bits)[0, :, 0, :],
                          np.broadcast_to(want, (q.shape[1], want.size)))
    out, _ = gu.run_fwd(sage, *_upload(dev, q, k, v), ml)
    got = _bits(out)
    bad = np.argwhere(got != ref_bits)
    assert bad.size == 0, (bad[:4].tolist(), got[tuple(bad[0])], ref_bits[tuple(bad[0])])


@MAINLOOPS
@pytest.mark.parametrize("N", [256, 230, 100])
def test_power_of_two_rescales_bit_exact(sage, dev, N, ml):
    qf, kf, vf = pins._rising_max_inputs(N, 7 + N)
    q, k, v = pins.make_qkv(qf, kf, vf)
    sm = float(np.float32(np.log(2.0)))
    ref_bits = oracle.attention(oracle.quantize(q, k, v), sm)
    out, _ = gu.run_fwd(sage, *_upload(dev, q, k, v), ml, sm_scale=sm)
    got = _bits(out)
    bad = np.argwhere(got != ref_bits)
    assert bad.size == 0, (int(bad.shape[0]), bad[:4].tolist())


@MAINLOOPS
@pytest.mark.parametrize("N,D", [(1000, 128), (333, 64)])
def test_large_magnitude_qk(sage, dev, N, D, ml):
    """Q and K of standard deviation 35 (amax about 122, score scale c about
    0.12 at D = 128): scores of hundreds of log2 units, so the exponent
    arguments are large and the attention is sharply peaked."""
    inp = synth.custom(1, N, 2, D, seed=91)
    scale = lambda a, f: pins.bf16_bits_round(synth.bf16_to_float(a) * f)
    q, k = scale(inp.q, 35.0), scale(inp.k, 35.0)
    qz = oracle.quantize(q, k, inp.v)
    c = qz.q_scale.max() * qz.k_scale.max() * np.float32(np.log2(np.e) / np.sqrt(D))
    assert c >= 0.1, c
    ref = oracle.bf16_bits_to_float(oracle.attention(qz))
    out, _ = gu.run_fwd(sage, *_upload(dev, q, k, inp.v), ml)
    mx, mean = gu.compare_out(out.float().cpu().numpy(), ref, f"large Q/K N={N} D={D}")
    print(f"large Q/K N={N} D={D} mainloop={ml}: max abs {mx:.3g} mean abs {mean:.3g}")
