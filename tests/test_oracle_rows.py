"""The oracle's row-range entry (used for the sampled full-size GPU parity
and the CPU baseline) gives exactly the rows of the full attention, for
ranges that start inside a 32-row Q group, end in the ragged last tile, and
for every head and batch."""
import numpy as np
import pytest

import oracle
import synth


@pytest.mark.parametrize("D", [128, 64])
def test_row_ranges_equal_the_full_attention(D):
    inp = synth.custom(2, 300, 3, D, seed=21)
    qz = oracle.quantize(inp.q, inp.k, inp.v)
    full = oracle.attention(qz)
    for b, h, r0, n in [(0, 0, 0, 300), (0, 1, 5, 40), (1, 2, 31, 2), (1, 0, 257, 43), (0, 2, 299, 1)]:
        part = oracle.attn_rows(qz, b, h, r0, n)
        assert part.shape == (n, D)
        assert np.array_equal(part, full[b, r0:r0 + n, h]), (b, h, r0, n)
