"""Pins for the oracle's implementation of the page's full route.

"Velox: Spatial Memory Makes World Models Efficient", Methodology Step 4
(importance from mean query and mean key; for well-covered regions the
distribution is multiplied by 1 + lambda * g_hat, g_hat the overlap above the
noise threshold tau rescaled by g_ref, then renormalised) and Step 5 (covered
query blocks: previous chunk reserved, best remaining blocks up to K_cov;
uncovered: smallest prefix of the model distribution reaching a mass
threshold, capped at K_unc; both joined with a local window in the Gilbert
block order and optional reference blocks outside the budget).
"""
import itertools
import math

import numpy as np
import pytest

import oracle

DEF = dict(lam=2.0, g_ref=0.2, tau=0.1, k_cov=80, k_unc=150, mass=0.9, prev_first=0,
           n_prev=0, window_half=0, ref_first=0, n_ref=0, own_first=100, n_own=2)


def row(s, g=None, covered=False, j=0, **kw):
    args = dict(DEF)
    args.update(kw)
    return oracle.velox_route_row(np.asarray(s, float), None if g is None else np.asarray(g, float),
                                  covered, j, **args).tolist()


def test_vetted_overlap_gate_and_rescale():
    g = np.array([0.0, 0.05, 0.1, 0.1000001, 0.15, 0.2, 0.9])
    gh = oracle.vetted_overlap(g, 0.1, 0.2)
    assert gh[:3].tolist() == [0.0, 0.0, 0.0]          # at or below tau: no overlap
    assert gh[4] == pytest.approx(0.75)
    assert gh[5] == 1.0 and gh[6] == 1.0               # saturates at 1


def test_multiplicative_fusion_ranks_like_renormalised_distribution():
    # Multiply softmax(s) by (1 + lam g_hat) and renormalise: the order equals
    # the order of s + log1p(lam g_hat), which the route uses.
    rng = np.random.default_rng(0)
    for _ in range(20):
        s = rng.standard_normal(30)
        g = rng.beta(0.5, 2.0, 30)
        p = np.exp(s - s.max()); p /= p.sum()
        gh = oracle.vetted_overlap(g, 0.1, 0.2)
        p2 = p * (1 + 2.0 * gh); p2 /= p2.sum()
        by_dist = sorted(range(30), key=lambda n: (-p2[n], n))
        got = row(s, g, covered=True, k_cov=10, own_first=30, n_own=0)
        assert got == sorted(by_dist[:10])


def test_covered_reserves_previous_chunk_inside_budget():
    s = np.arange(20.0)[::-1]                          # block 0 scores best
    got = row(s, covered=True, k_cov=8, prev_first=14, n_prev=5, own_first=20, n_own=1)
    # previous chunk 14..18 reserved, then the 3 best others (0, 1, 2)
    assert got == [0, 1, 2, 14, 15, 16, 17, 18, 20]
    # budget smaller than the reservation: the previous chunk alone
    got = row(s, covered=True, k_cov=3, prev_first=14, n_prev=5, own_first=20, n_own=1)
    assert got == [14, 15, 16, 17, 18, 20]


def test_uncovered_takes_smallest_mass_prefix_capped():
    # masses 0.5, 0.25, 0.125, ... (s = -n ln 2): prefix reaching 0.9 has 4 blocks
    s = np.array([-n * math.log(2.0) for n in range(12)])
    p = np.exp(s - s.max()); p /= p.sum()
    need = int(np.searchsorted(np.cumsum(p), 0.9) + 1)
    got = row(s, covered=False, mass=0.9, own_first=12, n_own=0)
    assert got == list(range(need)) and need == 4
    assert row(s, covered=False, mass=0.9, k_unc=2, own_first=12, n_own=0) == [0, 1]
    assert row(s, covered=False, mass=1.0 + 1e-9, own_first=12, n_own=0) == list(range(12))


def test_uncovered_ignores_geometry():
    s = np.zeros(10); s[7] = 1.0
    g = np.ones(10)
    assert row(s, g, covered=False, mass=0.05, own_first=10, n_own=0) == [7]


def test_window_and_reference_blocks_are_outside_the_budget():
    s = np.zeros(40)
    got = row(s, covered=False, mass=0.0, k_unc=1, j=3, prev_first=30, n_prev=10, window_half=2,
              ref_first=5, n_ref=2, own_first=40, n_own=3)
    # mass 0 -> the single best block (0); window positions 1..5 of the previous
    # chunk -> 31..35; references 5, 6; own chunk 40..42
    assert got == [0, 5, 6, 31, 32, 33, 34, 35, 40, 41, 42]


def test_brute_force_covered_selection():
    rng = np.random.default_rng(7)
    for _ in range(100):
        n = int(rng.integers(3, 9))
        s = rng.integers(-2, 3, n).astype(float)
        g = rng.choice([0.0, 0.05, 0.15, 0.4], n)
        k = int(rng.integers(0, n + 2))
        f = s + np.log1p(2.0 * oracle.vetted_overlap(g, 0.1, 0.2))
        beats = lambda i, j: f[i] > f[j] or (f[i] == f[j] and i < j)
        want = [c for kk in [min(k, n)] for c in itertools.combinations(range(n), kk)
                if all(beats(i, j) for i in c for j in range(n) if j not in c)]
        assert len(want) == 1
        got = row(s, g, covered=True, k_cov=k, own_first=n, n_own=0)
        assert got == sorted(want[0])
