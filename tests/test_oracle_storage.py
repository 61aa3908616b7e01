"""Pins for the oracle's Gilbert-ordered block storage (token <-> block scatter).

"Velox: Spatial Memory Makes World Models Efficient", Key Contributions 3:
KV is stored in 128-token blocks along the Gilbert order; the pages give no
worked example, so the scatter is pinned by its defining properties.
"""
import numpy as np
import pytest

import oracle
from oracle.gilbert import gilbert_cells


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("grid", [(2, 8, 16), (5, 30, 52), (1, 3, 5)])
def test_round_trip_identity(grid):
    T, H, W = grid
    x = _rand((2, T * H * W, 3, 4), 7)
    blk = oracle.tokens_to_blocks(x, T, H, W)
    back = oracle.blocks_to_tokens(blk, T, H, W)
    assert np.array_equal(back, x)


def test_pads_zero_and_valid_counts():
    T, H, W = 5, 30, 52                      # 7800 tokens -> 61 blocks, 8 pads
    x = _rand((1, T * H * W, 2, 4), 1) + 10.0  # no token is zero
    blk = oracle.tokens_to_blocks(x, T, H, W)
    assert blk.shape == (1, 2, 61, 128, 4)
    valid = oracle.block_valid_for(T, H, W)
    assert valid.tolist() == [128] * 60 + [120]
    assert np.all(blk[:, :, 60, 120:] == 0)
    assert np.all(blk[:, :, 60, :120] != 0)


def test_slot_is_curve_position():
    T, H, W = 2, 8, 16
    N = T * H * W
    # Encode the raster index in the payload, then read it back per slot.
    x = np.arange(N, dtype=np.float64).reshape(1, N, 1, 1)
    blk = oracle.tokens_to_blocks(x, T, H, W).reshape(-1)
    cells = gilbert_cells(T, H, W)
    for p, (t, h, w) in enumerate(cells):
        assert blk[p] == (t * H + h) * W + w


def test_append_places_chunks_consecutively():
    T, H, W = 2, 8, 16
    B, Hh, D = 1, 2, 4
    nb = oracle.n_blocks_for(T, H, W)
    ck = np.zeros((B, Hh, 3 * nb, 128, D))
    cv = np.zeros_like(ck)
    valid = np.zeros(3 * nb, dtype=np.int64)
    n = 0
    chunks = []
    for c in range(3):
        k = _rand((B, T * H * W, Hh, D), 10 + c)
        v = _rand((B, T * H * W, Hh, D), 20 + c)
        n = oracle.kv_append(ck, cv, valid, n, k, v, T, H, W)
        chunks.append((k, v))
    assert n == 3 * nb
    for c, (k, v) in enumerate(chunks):
        got = oracle.blocks_to_tokens(ck[:, :, c * nb:(c + 1) * nb], T, H, W)
        assert np.array_equal(got, k)
    with pytest.raises(ValueError):
        oracle.kv_append(ck, cv, valid, n, *chunks[0], T, H, W)
