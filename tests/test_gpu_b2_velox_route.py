"""GPU parity: bsa_route_velox (the page's full route) against the oracle.

"Velox: Spatial Memory Makes World Models Efficient", Methodology Steps 4-5,
with the page's calibrated constants (tau 0.1, g_ref 0.2, lambda 2, eta_cov
0.9, K_cov 80, K_unc 150) and a 26-neighbour (+/-13) window in the previous
chunk.  Routes must equal the oracle's except for near-ties: a differing
block must sit at the budget cut with a fused score within 1e-5 relative of
the cut, or at the mass cut with the cumulative mass within 1e-4 of it.
"""
import numpy as np
import pytest
import torch

import block_sparse_kv_bsa_b200 as bsa
import oracle
import synth
from tests import _harness as hx

pytestmark = pytest.mark.gpu
DEV = "cuda"
P = dict(tau=0.1, eta_cov=0.9, k_cov=80, k_unc=150, mass=0.9, window_half=13)


def _coverage(w, n_own, seed):
    rng = np.random.default_rng(seed)
    cov = rng.uniform(0.5, 1.0, size=(w.B, n_own)).astype(np.float32)   # about 20% >= 0.9
    return cov


def _check_rows(step, idx, cnt, scores, cov, heads, n_ref, ref_first, P=P):
    w = step.w
    nbc = step.n_own
    prev_first, n_prev = step.own_first - nbc, nbc
    g = step.g_np
    ties = 0
    for b in range(w.B):
        for hi, h in enumerate(heads):
            for j in range(nbc):
                s_row = scores[b, hi, j]
                covered = cov[b, j] >= P["eta_cov"]
                want = oracle.velox_route_row(
                    s_row, None if g is None else g[b, j], covered, j, w.lam, w.g_ref, P["tau"],
                    P["k_cov"], P["k_unc"], P["mass"], prev_first, n_prev, P["window_half"],
                    ref_first, n_ref, step.own_first, nbc).tolist()
                c = int(cnt[b, h, j])
                got = idx[b, h, j, :c].tolist()
                assert all(x == -1 for x in idx[b, h, j, c:].tolist())
                assert got == sorted(set(got)), "route must be ascending without repeats"
                assert got[-nbc:] == list(range(step.own_first, step.own_first + nbc))
                if got == want:
                    continue
                fixed = set(range(step.own_first, step.own_first + nbc))
                fixed |= {prev_first + p for p in range(j - P["window_half"], j + P["window_half"] + 1)
                          if 0 <= p < n_prev}
                fixed |= {ref_first + r for r in range(n_ref)}
                diff = (set(got) ^ set(want)) - fixed
                n_hist = s_row.shape[0]
                if covered:
                    f = s_row + (np.log1p(w.lam * oracle.vetted_overlap(g[b, j], P["tau"], w.g_ref))
                                 if g is not None else 0.0)
                    res = set(range(prev_first, prev_first + n_prev))
                    rest = sorted((n for n in range(n_hist) if n not in res), key=lambda n: (-f[n], n))
                    K = max(P["k_cov"] - len(res), 0)
                    cut = f[rest[K - 1]] if K > 0 else 0.0
                    tol = 1e-5 * max(abs(cut), np.mean(np.abs(f)))
                    for n in diff:
                        assert abs(f[n] - cut) <= tol, ("covered", b, h, j, n, f[n], cut)
                else:
                    order = sorted(range(n_hist), key=lambda n: (-s_row[n], n))
                    p = np.exp(s_row - s_row.max()); p /= p.sum()
                    cum = np.cumsum(p[order])
                    rank = {n: r for r, n in enumerate(order)}
                    m = len([x for x in want if x < n_hist and x not in fixed])
                    for n in diff:
                        r = rank[n]
                        near_mass = abs(cum[min(r, len(cum) - 1)] - P["mass"]) <= 1e-4 or \
                            abs(cum[max(r - 1, 0)] - P["mass"]) <= 1e-4
                        cut = s_row[order[max(m - 1, 0)]]
                        near_score = abs(s_row[n] - cut) <= 1e-5 * max(abs(cut), np.mean(np.abs(s_row)))
                        assert near_mass or near_score, ("uncovered", b, h, j, n, r, m)
                ties += 1
    return ties


@pytest.mark.parametrize("chunk,heads,k_unc", [(6, None, 150), (48, [7], 150), (12, [3, 20], 300)])
def test_velox_route_matches_oracle(chunk, heads, k_unc):
    # K_unc = 150 orders the uncovered budget by counting ranks; K_unc = 300
    # (more than 256) takes the sorting network.
    prm = dict(P, k_unc=k_unc)
    w = synth.CONFIGS[4]
    step = hx.build_step(w, DEV, chunk=chunk, pooled_keys=True)
    nbc = step.n_own
    cov = _coverage(w, nbc, seed=chunk)
    n_ref, ref_first = 4, 0
    idx, cnt = bsa.bsa_route_velox(
        step.q_blk, step.cache, step.n_hist, step.own_first, nbc, g=step.g,
        coverage=torch.from_numpy(cov).to(DEV), lam=w.lam, g_ref=w.g_ref, sm_scale=w.sm_scale,
        prev_first=step.own_first - nbc, n_prev=nbc, ref_first=ref_first, n_ref=n_ref,
        q_valid=step.q_valid, **prm)
    bsa.raise_on_device_error(DEV)
    heads = list(range(w.Hh)) if heads is None else heads
    scores = hx.oracle_scores_model(step, heads)
    ties = _check_rows(step, idx.cpu().numpy(), cnt.cpu().numpy(), scores, cov, heads, n_ref,
                       ref_first, prm)
    rows = w.B * len(heads) * nbc
    assert ties <= max(2, rows // 20), f"{ties} near-tie rows of {rows}"
    # Both kinds of rows occur, and the routes really differ in size.
    assert (cov >= P["eta_cov"]).any() and (cov < P["eta_cov"]).any()
    assert len(set(cnt.cpu().numpy().ravel().tolist())) > 1


def test_velox_route_no_coverage_no_prior_is_pure_mass_prefix():
    w = synth.CONFIGS[2]
    step = hx.build_step(w, DEV)
    idx, cnt = bsa.bsa_route_velox(step.q_blk, step.cache, step.n_hist, step.own_first,
                                   step.n_own, g=None, coverage=None, sm_scale=w.sm_scale,
                                   mass=0.5, k_unc=150, window_half=0, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    scores = hx.oracle_scores_model(step, list(range(w.Hh)))
    for h in range(w.Hh):
        for j in range(step.n_own):
            want = oracle.velox_route_row(scores[0, h, j], None, False, j, w.lam, w.g_ref, 0.1,
                                          80, 150, 0.5, 0, 0, 0, 0, 0, step.own_first,
                                          step.n_own).tolist()
            got = idx[0, h, j, :cnt[0, h, j]].cpu().tolist()
            assert got == want, (h, j)


def test_velox_route_rejects_small_max_sel():
    w = synth.CONFIGS[2]
    step = hx.build_step(w, DEV)
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_route_velox(step.q_blk, step.cache, step.n_hist, step.own_first, step.n_own,
                            max_sel=10)
    assert e.value.status == 3


@pytest.mark.parametrize("chunk", [12, 48])
def test_velox_route_from_query_means_equals_from_query_blocks(chunk):
    # bsa_route_velox_qmean on the means of bsa_tokens_to_blocks_mean gives
    # bsa_route_velox's routes (query blocks pooled by the route) bit for bit.
    w = synth.CONFIGS[4]
    T, H, W = w.grid
    step = hx.build_step(w, DEV, chunk=chunk, pooled_keys=True)
    nbc = step.n_own
    cov = torch.from_numpy(_coverage(w, nbc, seed=chunk)).to(DEV)
    kw = dict(g=step.g, coverage=cov, lam=w.lam, g_ref=w.g_ref, sm_scale=w.sm_scale,
              prev_first=step.own_first - nbc, n_prev=nbc, ref_first=0, n_ref=4, **P)
    i1, c1 = bsa.bsa_route_velox(step.q_blk, step.cache, step.n_hist, step.own_first, nbc,
                                 q_valid=step.q_valid, **kw)
    _, qm = bsa.bsa_tokens_to_blocks_mean(step.q_tok, T, H, W)
    i2, c2 = bsa.bsa_route_velox(None, step.cache, step.n_hist, step.own_first, nbc, q_mean=qm,
                                 **kw)
    bsa.raise_on_device_error(DEV)
    assert torch.equal(i1, i2) and torch.equal(c1, c2)
