"""Pins for the oracle's Gilbert (generalised Hilbert) order.

The Velox page ("Velox: Spatial Memory Makes World Models Efficient", Key
Contributions 3 and Methodology Step 6) names the order but prints no
example, so the curve is pinned by what a generalised Hilbert curve must be:
a bijection onto the grid, unit steps between consecutive cells, a
classical Hilbert curve on power-of-two squares and cubes, and the hand-derived
small cases under ``tests/golden/``.
"""
import itertools
import os
import random

import numpy as np
import pytest

from oracle.gilbert import feasible, gilbert_cells, gilbert_perm, top_box

CONFIG_GRIDS = [(2, 8, 16), (4, 16, 32), (5, 30, 52), (4, 30, 52), (4, 32, 32)]


def _check_curve(T, H, W):
    cells = gilbert_cells(T, H, W)
    assert len(cells) == T * H * W
    assert len(set(cells)) == T * H * W, "not a bijection"
    for t, h, w in cells:
        assert 0 <= t < T and 0 <= h < H and 0 <= w < W
    for p, q in zip(cells, cells[1:]):
        assert sum(abs(x - y) for x, y in zip(p, q)) == 1, ("non-unit step", p, q)
    assert cells[0] == (0, 0, 0)
    return cells


@pytest.mark.parametrize("grid", CONFIG_GRIDS)
def test_config_grids_bijective_unit_step(grid):
    _check_curve(*grid)


def test_all_small_boxes():
    for T, H, W in itertools.product(range(1, 8), range(1, 8), range(1, 8)):
        bx = top_box(T, H, W)
        assert feasible(bx.a, bx.b, bx.c)
        _check_curve(T, H, W)


def test_random_boxes():
    rnd = random.Random(1234)
    for _ in range(60):
        _check_curve(rnd.randint(1, 7), rnd.randint(1, 40), rnd.randint(1, 60))


def test_perm_is_inverse_of_cells():
    T, H, W = 4, 30, 52
    cells = gilbert_cells(T, H, W)
    perm = gilbert_perm(T, H, W)
    assert perm.dtype == np.int32
    assert sorted(perm.tolist()) == list(range(T * H * W))
    for p, (t, h, w) in enumerate(cells):
        assert perm[(t * H + h) * W + w] == p


def _dyadic_runs_ok(cells, levels):
    for lev in range(1, levels + 1):
        seen = set()
        last = None
        for t, h, w in cells:
            key = (t >> lev, h >> lev, w >> lev)
            if key != last:
                assert key not in seen, ("dyadic cell visited twice", lev, key)
                seen.add(key)
                last = key


@pytest.mark.parametrize("k", [1, 2, 3, 4])
def test_hilbert_property_on_cubes(k):
    n = 1 << k
    cells = _check_curve(n, n, n)
    _dyadic_runs_ok(cells, k)


def _textbook_hilbert(order):
    """Classical Hilbert curve on a 2^order square by the recursive quadrant
    construction: transpose, shift up, shift up-right, anti-transpose."""
    pts = [(0, 0)]
    n = 1
    for _ in range(order):
        q1 = [(y, x) for x, y in pts]
        q2 = [(x, y + n) for x, y in pts]
        q3 = [(x + n, y + n) for x, y in pts]
        q4 = [(2 * n - 1 - y, n - 1 - x) for x, y in pts]
        pts = q1 + q2 + q3 + q4
        n *= 2
    return pts


def _square_symmetries(pts, n):
    maps = [
        lambda x, y: (x, y), lambda x, y: (y, x),
        lambda x, y: (n - 1 - x, y), lambda x, y: (x, n - 1 - y),
        lambda x, y: (n - 1 - x, n - 1 - y), lambda x, y: (n - 1 - y, n - 1 - x),
        lambda x, y: (y, n - 1 - x), lambda x, y: (n - 1 - y, x),
    ]
    out = []
    for f in maps:
        img = [f(x, y) for x, y in pts]
        out.append(img)
        out.append(img[::-1])
    return out


@pytest.mark.parametrize("k", [1, 2, 3, 4, 5])
def test_square_is_textbook_hilbert(k):
    n = 1 << k
    cells = _check_curve(1, n, n)
    mine = [(w, h) for _, h, w in cells]
    assert mine in _square_symmetries(_textbook_hilbert(k), n)
    _dyadic_runs_ok(cells, k)


def _read_golden(name):
    path = os.path.join(os.path.dirname(__file__), "golden", name)
    rows = []
    with open(path) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(tuple(int(v) for v in line.split()))
    return rows


@pytest.mark.parametrize("name,grid", [("gilbert_2x2x2.txt", (2, 2, 2)),
                                       ("gilbert_1x4x4.txt", (1, 4, 4))])
def test_hand_derived_golden(name, grid):
    assert gilbert_cells(*grid) == _read_golden(name)


def test_same_shape_same_order():
    # Global alignment: every chunk of one shape shares the order.
    a = gilbert_perm(4, 30, 52)
    b = gilbert_perm(4, 30, 52)
    assert np.array_equal(a, b)


def test_blocks_are_compact():
    # Locality: the cells of one 128-token block span a small box, far
    # smaller than a raster run of 128 tokens would on a 30 x 52 frame.
    T, H, W = 4, 30, 52
    cells = np.array(gilbert_cells(T, H, W))
    spans = []
    for b0 in range(0, len(cells) - 127, 128):
        blk = cells[b0:b0 + 128]
        spans.append(int((blk.max(0) - blk.min(0) + 1).prod()))
    assert np.median(spans) <= 4 * 128


def test_rejects_empty_grid():
    with pytest.raises(ValueError):
        gilbert_cells(0, 4, 4)
