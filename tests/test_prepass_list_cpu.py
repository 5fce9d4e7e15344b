"""The work list of the single-launch prepass, read from the library on the
host (no GPU): every 64-token tile of every kind appears exactly once, and
each head's K and V statistics tiles come before its K and V code tiles.
The code tiles' bounded waits rely on both (a CTA waits only for tiles
earlier in the list, which running CTAs already hold), and the lag puts
about two grids of tiles between a head's statistics and its codes."""
import numpy as np
import pytest

import fp8_quantized_exact_b200 as sage

SHAPES = [(1, 256, 2, 128), (1, 1000, 8, 128), (2, 8192, 32, 128), (1, 37810, 56, 128), (4, 16384, 24, 64),
          (1, 1, 1, 64), (3, 65, 5, 128), (1, 4000, 1, 64), (24, 100, 64, 64)]


@pytest.fixture(scope="module")
def lib():
    from fp8_quantized_exact_b200 import build
    build.build()
    return sage.lib()


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("grid", [1, 40, 888])
def test_every_tile_once_and_statistics_first(lib, shape, grid):
    B, N, H, D = shape
    U, I, T64 = B * H, -(-N // 128) * 2, -(-N // 64)
    lag, items = sage.sage_debug_prepass_list(B, N, H, D, grid)
    assert items.shape == (5 * U * I, 3)
    kind, unit, tile = items.T
    assert kind.min() >= 0 and kind.max() <= 4 and unit.min() >= 0 and unit.max() < U
    assert tile.min() >= 0 and tile.max() < I
    key = (kind.astype(np.int64) * U + unit) * I + tile
    assert np.array_equal(np.sort(key), np.arange(5 * U * I))  # each (kind, head, tile) once
    pos = np.empty(5 * U * I, dtype=np.int64)
    pos[key] = np.arange(5 * U * I)
    pos = pos.reshape(5, U, I)
    last_stats = pos[:2].max(axis=(0, 2))
    first_codes = pos[3:].min(axis=(0, 2))
    assert np.all(last_stats < first_codes)
    # the lag: R heads, at least one; about two grids of tiles between a
    # head's statistics and its codes unless all heads fit in the lag
    assert 1 <= lag <= max(U, 1)
    assert lag == U or (5 * lag + 2) * I >= 2 * grid
    # tiles past the last 64-token chunk exist only so that Q's 128-row
    # padding has a tile; the kernel skips their K and V work
    assert I >= T64


def test_wrong_count_is_refused(lib):
    import ctypes
    items = np.zeros((10, 3), dtype=np.int32)
    assert lib.sage_debug_prepass_list(1, 256, 2, 128, 40, None, 10, items.ctypes.data) == sage.SAGE_ERR_INVALID_ARG
    assert lib.sage_debug_prepass_list(1, 256, 2, 128, 0, None, 40, items.ctypes.data) == sage.SAGE_ERR_INVALID_ARG
    assert lib.sage_debug_prepass_list(1, 256, 2, 96, 40, None, 40, items.ctypes.data) == sage.SAGE_ERR_UNSUPPORTED
    assert lib.sage_debug_prepass_list(1, 256, 2, 128, 40, None, 40, None) == sage.SAGE_ERR_INVALID_ARG
