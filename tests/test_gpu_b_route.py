"""GPU parity: bsa_route against the oracle's pooled-score top-K.

"Velox: Spatial Memory Makes World Models Efficient", Methodology Steps 4-5.
Block indices must match the oracle exactly, apart from near-ties within
1e-5 relative of the K-th score (fp32 on the GPU, fp64 in the oracle), where
either choice is accepted.
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_kv_bsa_b200 as bsa
import synth
from tests import _harness as hx

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check(step, heads=None, top_k=None):
    if top_k is not None:
        step.top_k = top_k
    idx, cnt = hx.route(step)
    bsa.raise_on_device_error(DEV)
    heads = list(range(step.w.Hh)) if heads is None else list(heads)
    scores = hx.oracle_scores(step, heads)
    ties = hx.check_route_rows(idx[:, heads].cpu().numpy(), cnt[:, heads].cpu().numpy(), scores,
                               step.top_k, step.own_first, step.n_own)
    rows = step.w.B * len(heads) * step.n_own
    assert ties <= max(2, rows // 50), f"{ties} near-tie rows of {rows}"
    return idx, cnt


def test_route_config1_tiny():
    _check(hx.build_step(synth.CONFIGS[1], DEV))


def test_route_config2_block_offsets():
    _check(hx.build_step(synth.CONFIGS[2], DEV))


def test_route_config3_velox_budget_with_prior():
    _check(hx.build_step(synth.CONFIGS[3], DEV))


@pytest.mark.parametrize("top_k", [256, 32])
def test_route_config5_head_sample(top_k):
    _check(hx.build_step(synth.CONFIGS[5], DEV, top_k=top_k), heads=[0, 17, 39])


@pytest.mark.parametrize("chunk", [1, 2, 3, 12, 48, 49])
def test_route_config4_sweep_chunks(chunk):
    # chunk 1: no history (own chunk only); chunk 2: K >= history (all);
    # chunk 3: K < history; chunk 48: the headline size, one head checked.
    # The row lengths 98, 539, 2303 and 2352 take each register width of the
    # register top-K (up to 512, 1280, 2304 and 3072 blocks).
    step = hx.build_step(synth.CONFIGS[4], DEV, chunk=chunk)
    _check(step, heads=[5] if chunk >= 12 else [0, 23])


def test_route_rows_longer_than_the_register_select():
    # 193 history chunks of 16 blocks: rows of 3088 history blocks are longer
    # than the register top-K takes (3072), so the shared-memory radix select
    # routes them.
    step = hx.build_step(synth.CONFIGS[2], DEV, chunk=194)
    assert step.n_hist > 32 * 96
    _check(step, heads=[7])


def test_route_without_prior_equals_prior_of_zeros():
    step = hx.build_step(synth.CONFIGS[3], DEV)
    a, ca = hx.route(step)
    g0 = step.g
    step.g = torch.zeros_like(g0)
    b, cb = hx.route(step)
    step.g = None
    c, cc = hx.route(step)
    assert torch.equal(b, c) and torch.equal(cb, cc)
    assert not torch.equal(a, c)  # the prior does change the route


def test_route_all_equal_scores_take_lowest_indices():
    # Q = 0 makes every model score 0, so with no prior the route is 0..K-1.
    step = hx.build_step(synth.CONFIGS[2], DEV)
    step.q_blk.zero_()
    step.g = None
    idx, cnt = hx.route(step)
    K = step.top_k
    exp = torch.arange(K, dtype=torch.int32, device=DEV)
    assert torch.all(idx[..., :K] == exp)


@pytest.mark.parametrize("n_top", [100, 1000])
def test_route_exact_ties_at_the_cut_take_lowest_indices(n_top):
    # Q = 0 and a prior of three levels: every fused score is the prior
    # alone, with exact ties.  n_top history blocks per row at the top level
    # (K = 64 of them are taken): 100 leaves few candidates at the cut (the
    # row top-K's pivot pass settles it), 1000 too many for that pass (the
    # search over the whole row does).  Either way the route is the top K
    # with ties to the lower block, exactly as the oracle's.
    import oracle
    w = synth.CONFIGS[4]
    step = hx.build_step(w, DEV, chunk=48)
    step.q_blk.zero_()
    nh, J = step.n_hist, step.n_own
    rng = np.random.default_rng(11 + n_top)
    g = np.zeros((w.B, J, nh), np.float32)
    for b in range(w.B):
        for j in range(J):
            p = rng.permutation(nh)
            g[b, j, p[:n_top]] = w.g_ref
            g[b, j, p[n_top:n_top + 300]] = 0.5 * w.g_ref
    step.g = torch.from_numpy(g).to(DEV)
    idx, cnt = hx.route(step)
    bsa.raise_on_device_error(DEV)
    fused = oracle.fuse_prior(np.zeros((w.B, 1, J, nh)), g.astype(np.float64), w.lam, w.g_ref)
    idx_h = idx.cpu().numpy()
    for b in range(w.B):
        for j in range(J):
            want = oracle.top_k_with_own(fused[b, 0, j], step.top_k, step.own_first, J)
            for h in (0, 13):
                assert np.array_equal(idx_h[b, h, j, :len(want)], want), (b, h, j)


def test_route_rejects_bad_arguments():
    step = hx.build_step(synth.CONFIGS[1], DEV)
    with pytest.raises(bsa.BsaError) as e:     # max_sel too small
        hx.route(step, max_sel=2)
    assert e.value.status == 3
    with pytest.raises(bsa.BsaError) as e:     # own chunk overlapping the history
        bsa.bsa_route(step.q_blk, step.cache, step.n_hist + 1, step.own_first, step.n_own,
                      step.top_k)
    assert e.value.status == 2


@pytest.mark.parametrize("key,chunk", [(1, None), (2, None), (3, None), (4, 48), (5, None)])
def test_route_from_pooled_keys(key, chunk):
    # Routing from the pooled-key cache (block key means written at append
    # time, scored by a small product kernel) against the oracle, with the
    # same near-tie rule as the streaming route; its fp32 sums run in another
    # order than the streaming route's, so the two may differ only at
    # near-ties.
    w = synth.CONFIGS[key]
    b = hx.build_step(w, DEV, chunk=chunk, pooled_keys=True)
    ib, cb = _check(b, heads=[5] if key == 4 else [0, 39] if key == 5 else None)
    # The no-allocation entry point takes the same path, bit for bit.
    import ctypes
    idx = torch.full_like(ib, -7)
    cnt = torch.full_like(cb, -7)
    cs = b.cache.c_struct()
    st = bsa.lib().bsa_route_noalloc(
        ctypes.c_void_p(b.q_blk.data_ptr()), ctypes.byref(cs), ctypes.c_void_p(b.q_valid.data_ptr()),
        b.n_hist, b.own_first, b.n_own, None if b.g is None else ctypes.c_void_p(b.g.data_ptr()),
        w.lam, w.g_ref, w.sm_scale, b.top_k, ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(cnt.data_ptr()), ib.shape[-1], None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    torch.cuda.synchronize()
    assert torch.equal(idx, ib) and torch.equal(cnt, cb)


@pytest.mark.parametrize("grid", [(8, 32, 32), (5, 26, 64)])
def test_route_from_pooled_keys_at_the_tensor_core_product_limit(grid):
    # 64 query blocks (8 x 32 x 32): the most the tensor-core product holds,
    # every row of its query-mean operand in use; 65 (5 x 26 x 64): the first
    # count scored on the FMA pipes instead.  211 history blocks: one full
    # 128-block tile and a ragged one.
    w = dataclasses.replace(synth.CONFIGS[3], grid=grid, Hh=4, hist_direct=211)
    b = hx.build_step(w, DEV, pooled_keys=True)
    assert b.n_own == (64 if grid == (8, 32, 32) else 65)
    _check(b)


def test_route_from_pooled_keys_many_query_blocks():
    # 98 query blocks (an 8 x 30 x 52 chunk): more than the pipelined pooled
    # product takes (64), so the one-shot kernel scores them.
    w = dataclasses.replace(synth.CONFIGS[3], grid=(8, 30, 52), Hh=4, hist_direct=300)
    b = hx.build_step(w, DEV, pooled_keys=True)
    assert b.n_own > 64
    _check(b)
