"""Pins for the oracle's indexed block-sparse attention.

"Velox: Spatial Memory Makes World Models Efficient", Methodology Step 6:
a skipped block contributes neither its QK^T tile nor its KV load, so the
sparse call over a route is softmax attention over exactly the keys of the
selected blocks.  Pinned by closed forms, by a library routine (torch's
scaled_dot_product_attention in float64) on the dense case, by brute-force
dense-masked attention on tiny inputs, and by invariances.  A final test
plants mistakes in the oracle and checks that these pins catch each one.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
from oracle import bsa as obsa


def _setup(seed, B=1, Hh=2, n_blocks=5, n_q=2, D=8, valid=None):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, Hh, n_q * 128, D))
    kc = rng.standard_normal((B, Hh, n_blocks, 128, D))
    vc = rng.standard_normal((B, Hh, n_blocks, 128, D))
    if valid is None:
        valid = np.full(n_blocks, 128)
    valid = np.asarray(valid)
    for n in range(n_blocks):
        kc[:, :, n, valid[n]:] = 0.0
        vc[:, :, n, valid[n]:] = 0.0
    return q, kc, vc, valid


def _full_route(B, Hh, n_q, sel):
    idx = np.zeros((B, Hh, n_q, len(sel)), dtype=np.int64)
    idx[...] = np.asarray(sel)
    cnt = np.full((B, Hh, n_q), len(sel))
    return idx, cnt


def test_all_blocks_equals_library_dense_attention():
    B, Hh, nb, nq, D = 1, 2, 4, 2, 8
    q, kc, vc, valid = _setup(0, B, Hh, nb, nq, D)
    idx, cnt = _full_route(B, Hh, nq, list(range(nb)))
    sm = 1 / math.sqrt(D)
    o, lse = oracle.attn(q, kc, vc, valid, [128] * nq, idx, cnt, sm)
    qt = torch.from_numpy(q)
    kt = torch.from_numpy(kc.reshape(B, Hh, nb * 128, D))
    vt = torch.from_numpy(vc.reshape(B, Hh, nb * 128, D))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=sm).numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
    logits = sm * np.einsum("bhqd,bhkd->bhqk", q, kc.reshape(B, Hh, nb * 128, D))
    assert np.allclose(lse, logsumexp(logits, axis=-1), rtol=1e-12, atol=1e-12)


def test_single_key_returns_its_value_row():
    B, Hh, nb, nq, D = 1, 1, 3, 1, 8
    q, kc, vc, valid = _setup(1, B, Hh, nb, nq, D, valid=[128, 1, 128])
    idx, cnt = _full_route(B, Hh, nq, [1])
    sm = 0.3
    o, lse = oracle.attn(q, kc, vc, valid, [128], idx, cnt, sm)
    assert np.allclose(o[0, 0], vc[0, 0, 1, 0][None, :], atol=1e-14)
    assert np.allclose(lse[0, 0], sm * q[0, 0] @ kc[0, 0, 1, 0], atol=1e-12)


def test_zero_query_gives_mean_of_selected_values():
    B, Hh, nb, nq, D = 1, 1, 4, 1, 8
    q, kc, vc, valid = _setup(2, B, Hh, nb, nq, D, valid=[128, 40, 128, 7])
    q[:] = 0.0
    sel = [1, 3]
    idx, cnt = _full_route(B, Hh, nq, sel)
    o, lse = oracle.attn(q, kc, vc, valid, [128], idx, cnt, 0.125)
    rows = np.concatenate([vc[0, 0, 1, :40], vc[0, 0, 3, :7]])
    assert np.allclose(o[0, 0], rows.mean(axis=0)[None, :], atol=1e-13)
    assert np.allclose(lse[0, 0], math.log(47), atol=1e-13)


def test_index_order_invariance():
    B, Hh, nb, nq, D = 1, 2, 6, 2, 8
    q, kc, vc, valid = _setup(3, B, Hh, nb, nq, D, valid=[128, 128, 60, 128, 128, 3])
    a, ca = _full_route(B, Hh, nq, [0, 2, 3, 5])
    b, cb = _full_route(B, Hh, nq, [5, 3, 0, 2])
    o1, l1 = oracle.attn(q, kc, vc, valid, [128, 128], a, ca, 0.4)
    o2, l2 = oracle.attn(q, kc, vc, valid, [128, 128], b, cb, 0.4)
    assert np.allclose(o1, o2, atol=1e-13) and np.allclose(l1, l2, atol=1e-13)


def test_brute_force_dense_masked_agrees():
    B, Hh, nb, nq, D = 1, 2, 5, 2, 8
    valid = [128, 90, 128, 128, 17]
    q, kc, vc, valid = _setup(4, B, Hh, nb, nq, D, valid=valid)
    rng = np.random.default_rng(9)
    idx = np.zeros((B, Hh, nq, 3), dtype=np.int64)
    cnt = np.full((B, Hh, nq), 3)
    for h in range(Hh):
        for j in range(nq):
            idx[0, h, j] = np.sort(rng.choice(nb, 3, replace=False))
    q_valid = [128, 100]
    o, lse = oracle.attn(q, kc, vc, valid, q_valid, idx, cnt, 0.35)
    for h in range(Hh):
        keys = kc[0, h].reshape(nb * 128, D)
        vals = vc[0, h].reshape(nb * 128, D)
        allowed = np.zeros((nq * 128, nb * 128), dtype=bool)
        for j in range(nq):
            for n in idx[0, h, j]:
                allowed[j * 128:j * 128 + q_valid[j], n * 128:n * 128 + valid[n]] = True
        ob, lb = oracle.dense_masked_attn(q[0, h], keys, vals, allowed, 0.35)
        assert np.allclose(o[0, h], ob, atol=1e-12)
        assert np.array_equal(np.isinf(lse[0, h]), np.isinf(lb))
        fin = np.isfinite(lb)
        assert np.allclose(lse[0, h][fin], lb[fin], atol=1e-12)


def test_pad_queries_and_pad_keys():
    B, Hh, nb, nq, D = 1, 1, 2, 1, 8
    q, kc, vc, valid = _setup(5, B, Hh, nb, nq, D, valid=[128, 33])
    idx, cnt = _full_route(B, Hh, nq, [0, 1])
    o1, l1 = oracle.attn(q, kc, vc, valid, [50], idx, cnt, 0.3)
    assert np.all(o1[0, 0, 50:] == 0) and np.all(np.isneginf(l1[0, 0, 50:]))
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[0, 0, 1, 33:] = 1e3                       # garbage in pad key rows
    vc2[0, 0, 1, 33:] = -1e3
    o2, l2 = oracle.attn(q, kc2, vc2, valid, [50], idx, cnt, 0.3)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# --- planted mistakes: each mutant of the attention core must fail a pin ---

def _mut_no_scale(q, k, v, s):
    return obsa._orig_attn_rows(q, k, v, 1.0)


def _mut_log2_lse(q, k, v, s):
    o, l = obsa._orig_attn_rows(q, k, v, s)
    return o, l / math.log(2.0)


def _mut_no_normalise(q, k, v, s):
    logits = s * (q @ k.T)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    return p @ v, (m + np.log(p.sum(axis=1, keepdims=True)))[:, 0]


def _mut_max_not_restored(q, k, v, s):
    o, l = obsa._orig_attn_rows(q, k, v, s)
    logits = s * (q @ k.T)
    return o, l - logits.max(axis=1)


def _mut_drop_last_key(q, k, v, s):
    return obsa._orig_attn_rows(q, k[:-1], v[:-1], s)


PINS = [test_all_blocks_equals_library_dense_attention, test_single_key_returns_its_value_row,
        test_zero_query_gives_mean_of_selected_values, test_brute_force_dense_masked_agrees]


@pytest.mark.parametrize("mutant", [_mut_no_scale, _mut_log2_lse, _mut_no_normalise,
                                    _mut_max_not_restored, _mut_drop_last_key])
def test_pins_catch_planted_mistakes(monkeypatch, mutant):
    monkeypatch.setattr(obsa, "_orig_attn_rows", obsa.attn_rows, raising=False)
    monkeypatch.setattr(obsa, "attn_rows", mutant)
    failures = 0
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError):
            failures += 1
    assert failures >= 1, "no pin noticed the planted mistake"
