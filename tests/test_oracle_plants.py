"""Each deliberately wrong oracle build (a mistake planted in the C source
behind ORACLE_PLANT=n, CPU only) must fail at least one pin; this shows the
pins can see a dropped term, a wrong sign or index, or a transposed operand."""
import pytest

import pins

PLANTS = {
    1: "K smoothing dropped (km forced to 0)",
    2: "Q/K scale and its inverse swapped",
    3: "Q group of 64 rows instead of 32",
    4: "log2(e) missing from the score scale",
    5: "K channel index reversed in QK^T",
    6: "old-max rescale of RO and d skipped",
    7: "max not subtracted before exp2",
    8: "V scale not applied in the epilogue",
    9: "RoPE rotation sign flipped in the first half",
    10: "denominator summed from the E4M3 probabilities",
    11: "FP16 rounding of the K32 buffers skipped",
    12: "one K64 FP16 buffer per tile instead of two K32 ones",
    13: "keys past N in the last tile not masked",
    14: "INT8 ties rounded away from zero",
    15: "K mean taken over the 64-padded length",
    16: "Q scale read per 64 rows in the score scale",
    17: "accumulator rescaled after the tile's PV instead of before",
    18: "accumulator not rescaled (the denominator is)",
    19: "K channel sums kept in FP32",
}


@pytest.mark.parametrize("plant", sorted(PLANTS), ids=lambda n: f"plant{n}")
def test_planted_mistake_is_caught(plant):
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(plant)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught planted mistake {plant}: {PLANTS[plant]}"
