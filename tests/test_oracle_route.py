"""Pins for the oracle's router: pooling, scoring, prior fusion and top-K.

"Velox: Spatial Memory Makes World Models Efficient", Methodology Step 4
(block importance from mean query and mean key; soft geometric boost of at
most 1 + lambda, none where there is no overlap) and Step 5 (a budgeted
top-K route with reserved blocks added outside the budget).  The pages
print no worked example, so these pins are closed forms, invariants and
brute force on tiny inputs.
"""
import itertools

import numpy as np
import pytest

import oracle


def test_pool_constant_block():
    x = np.full((1, 1, 2, 128, 8), 3.25)
    m = oracle.pool_blocks(x, [128, 128])
    assert np.all(m == 3.25)


def test_pool_ramp_closed_form_and_pad_exclusion():
    x = np.zeros((1, 1, 1, 128, 2))
    x[0, 0, 0, :, 0] = np.arange(128)
    x[0, 0, 0, :, 1] = 1.0
    v = 77
    x[0, 0, 0, v:, :] = 1e9                        # pad rows hold garbage
    m = oracle.pool_blocks(x, [v])
    assert m[0, 0, 0, 0] == pytest.approx((v - 1) / 2, abs=1e-12)
    assert m[0, 0, 0, 1] == pytest.approx(1.0, abs=1e-15)


def test_scores_closed_form():
    q = np.zeros((1, 1, 2, 4))
    k = np.zeros((1, 1, 3, 4))
    q[0, 0, 0, 0] = 2.0
    q[0, 0, 1, 1] = -1.0
    k[0, 0, 0, 0] = 3.0            # parallel to q0
    k[0, 0, 1, 1] = 5.0            # parallel to q1 (opposite sign)
    k[0, 0, 2, 2] = 7.0            # orthogonal to both
    s = oracle.block_scores(q, k, 0.5)
    assert s[0, 0].tolist() == [[3.0, 0.0, 0.0], [0.0, -2.5, 0.0]]


def test_fuse_invariants():
    rng = np.random.default_rng(3)
    s = rng.standard_normal((2, 3, 4, 50))
    g = rng.beta(0.5, 2.0, size=(2, 4, 50))
    g[rng.random(g.shape) < 0.3] = 0.0
    lam, g_ref = 2.0, 0.2
    assert np.array_equal(oracle.fuse_prior(s, None, lam, g_ref), s)
    f = oracle.fuse_prior(s, g, lam, g_ref)
    d = f - s
    assert np.all(d >= 0) and np.all(d <= lam + 1e-12)           # at most a lambda boost
    zero = np.broadcast_to((g == 0)[:, None], d.shape)
    assert np.all(d[zero] == 0)                                   # no overlap, no change
    full = np.broadcast_to((g >= g_ref)[:, None], d.shape)
    assert np.allclose(d[full], lam, atol=1e-12)                  # saturated at +lambda
    half = np.full((2, 4, 50), g_ref / 2)
    assert np.allclose(oracle.fuse_prior(s, half, lam, g_ref) - s, lam / 2)
    # The prior is per (b, query block, kv block): the same for every head.
    assert np.allclose(d[:, 0], d[:, 2])


def _brute_top_k(row, k):
    """The unique k-set whose every member beats every non-member under
    (higher score, then lower index); found by trying all k-subsets."""
    n = len(row)
    if k >= n:
        return list(range(n))
    beats = lambda i, j: row[i] > row[j] or (row[i] == row[j] and i < j)
    hits = [c for c in itertools.combinations(range(n), k)
            if all(beats(i, j) for i in c for j in range(n) if j not in c)]
    assert len(hits) == 1
    return list(hits[0])


def test_top_k_brute_force():
    rng = np.random.default_rng(5)
    for trial in range(200):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(0, 10))
        row = rng.integers(-3, 4, size=n).astype(np.float64)   # many exact ties
        got = oracle.top_k_with_own(row, k, 100, 3)
        assert got.tolist() == sorted(_brute_top_k(row, k)) + [100, 101, 102]


def test_top_k_special_cases():
    row = np.zeros(10)
    assert oracle.top_k_with_own(row, 4, 10, 2).tolist() == [0, 1, 2, 3, 10, 11]
    row = np.arange(10.0)
    assert oracle.top_k_with_own(row, 99, 10, 1).tolist() == list(range(11))
    assert oracle.top_k_with_own(row, 0, 10, 2).tolist() == [10, 11]
    assert oracle.top_k_with_own(np.zeros(0), 3, 0, 2).tolist() == [0, 1]
    assert oracle.top_k_with_own(row, 3, 10, 1).tolist() == [7, 8, 9, 10]


def test_route_picks_planted_blocks():
    # Each query block j is planted with a mean direction e_j; history block
    # 2j+1 carries the same direction, every other block is orthogonal.  With
    # top_k = 1 the route of j must be [2j+1] + own chunk.
    B, Hh, D = 1, 2, 16
    n_own, n_hist = 3, 8
    q = np.zeros((B, Hh, n_own * 128, D))
    kc = np.zeros((B, Hh, n_hist + n_own, 128, D))
    for j in range(n_own):
        q[:, :, j * 128:(j + 1) * 128, j] = 1.0
        kc[:, :, 2 * j + 1, :, j] = 1.0
    for n in range(n_hist):
        if n % 2 == 0 or n // 2 >= n_own:
            kc[:, :, n, :, D - 1] = 1.0
    valid = np.full(n_hist + n_own, 128)
    idx, s = oracle.route(q, kc, valid, n_hist, n_hist, n_own, None, 2.0, 0.2, 0.25, 1)
    for h in range(Hh):
        for j in range(n_own):
            assert idx[0][h][j].tolist() == [2 * j + 1, 8, 9, 10]
    # And a saturating prior on block 6 overrides the model score for j = 0.
    g = np.zeros((B, n_own, n_hist))
    g[0, 0, 6] = 1.0
    idx, _ = oracle.route(q, kc, valid, n_hist, n_hist, n_own, g, 2.0, 0.2, 0.25, 1)
    assert idx[0][0][0].tolist() == [6, 8, 9, 10]
    assert idx[0][0][1].tolist() == [3, 8, 9, 10]


def test_route_respects_pad_rows_of_query():
    B, Hh, D = 1, 1, 4
    q = np.zeros((B, Hh, 128, D))
    q[0, 0, :10, 0] = 1.0
    q[0, 0, 10:, 1] = 50.0                    # pad rows: must not steer the route
    kc = np.zeros((B, Hh, 3, 128, D))
    kc[0, 0, 0, :, 0] = 1.0
    kc[0, 0, 1, :, 1] = 1.0
    valid = np.array([128, 128, 10])
    idx, _ = oracle.route(q, kc, valid, 2, 2, 1, None, 2.0, 0.2, 1.0, 1, q_valid=[10])
    assert idx[0][0][0].tolist() == [0, 2]
