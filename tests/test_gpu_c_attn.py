"""GPU parity: bsa_attn (tcgen05 / TMEM / TMA kernel) against the fp64 oracle.

"Velox: Spatial Memory Makes World Models Efficient", Methodology Step 6:
attention over exactly the keys of the selected blocks.  The compared query
blocks attend, in the library and in the oracle, over the oracle's own route
(the library is a pure function of its index list), so a near-tie routing
swap can never show up here as an attention error.  Bar: O relative L2 <=
1e-2 and max abs <= 2e-2, LSE max abs <= 1e-3 over valid rows; pad query rows
exactly O = 0, LSE = -inf.
"""
import numpy as np
import pytest
import torch

import block_sparse_kv_bsa_b200 as bsa
import synth
from tests import _harness as hx

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _compare(step, routes, o, lse, items, sm_scale=None):
    refs = hx.oracle_attn_items(step, routes, items, sm_scale=sm_scale)
    o_np = o.cpu().double().numpy()
    l_np = lse.cpu().double().numpy()
    qv = hx.oracle_valid(step)[step.own_first:step.own_first + step.n_own]
    worst = (0.0, 0.0, 0.0)
    for (b, h, j), (ro, rl) in zip(items, refs):
        rows = slice(j * 128, (j + 1) * 128)
        rel, mabs, lerr = hx.attn_errors(o_np[b, h, rows], l_np[b, h, rows], ro, rl, int(qv[j]))
        worst = tuple(max(x, y) for x, y in zip(worst, (rel, mabs, lerr)))
        assert rel <= hx.O_REL_L2 and mabs <= hx.O_MAX_ABS and lerr <= hx.LSE_MAX_ABS, \
            ((b, h, j), rel, mabs, lerr)
    return worst


def _all_items(step):
    return [(b, h, j) for b in range(step.w.B) for h in range(step.w.Hh) for j in range(step.n_own)]


def test_attn_config1_every_element():
    step = hx.build_step(synth.CONFIGS[1], DEV)
    idx, cnt, routes = hx.attn_routes(step, range(step.w.Hh))
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    _compare(step, routes, o, lse, _all_items(step))


def test_attn_config2_every_element():
    step = hx.build_step(synth.CONFIGS[2], DEV)
    idx, cnt, routes = hx.attn_routes(step, range(step.w.Hh))
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    _compare(step, routes, o, lse, _all_items(step))


def test_attn_config3_two_heads_with_tail_block():
    step = hx.build_step(synth.CONFIGS[3], DEV)
    idx, cnt, routes = hx.attn_routes(step, (0, 23))
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    items = [(0, h, j) for h in (0, 23) for j in range(step.n_own)]
    _compare(step, routes, o, lse, items)


def test_attn_config4_chunk48_sample():
    step = hx.build_step(synth.CONFIGS[4], DEV, chunk=48)
    idx, cnt, routes = hx.attn_routes(step, (0, 11, 23))
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    items = [(0, h, j) for h in (0, 11, 23) for j in (0, 17, 48)]
    _compare(step, routes, o, lse, items)


def test_attn_config4_chunk48_every_query_block_of_two_heads():
    # The launch the bench times (all 24 heads, 49 query blocks of 113 tiles)
    # compared on every query block of two heads, the tail block included.
    step = hx.build_step(synth.CONFIGS[4], DEV, chunk=48)
    heads = (5, 18)
    idx, cnt, routes = hx.attn_routes(step, heads)
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    items = [(0, h, j) for h in heads for j in range(step.n_own)]
    _compare(step, routes, o, lse, items)


def _velox_attn_routes(step, heads, cov):
    """The page's route (Velox constants: tau 0.1, eta_cov 0.9, K_cov 80,
    K_unc 150, mass 0.9, +/-13 window in the previous chunk) for every query
    block: the library's own for all heads, replaced on ``heads`` by the
    oracle's, so both sides attend over the oracle's variable-length lists."""
    import oracle
    w = step.w
    nbc = step.n_own
    prev_first = step.own_first - nbc
    idx, cnt = bsa.bsa_route_velox(
        step.q_blk, step.cache, step.n_hist, step.own_first, nbc, g=step.g,
        coverage=torch.from_numpy(cov).to(DEV), lam=w.lam, g_ref=w.g_ref, sm_scale=w.sm_scale,
        tau=0.1, eta_cov=0.9, k_cov=80, k_unc=150, mass=0.9, prev_first=prev_first, n_prev=nbc,
        window_half=13, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    scores = hx.oracle_scores_model(step, heads)
    idx_h, cnt_h = idx.cpu(), cnt.cpu()
    routes = {}
    for b in range(w.B):
        for hi, h in enumerate(heads):
            for j in range(nbc):
                r = oracle.velox_route_row(scores[b, hi, j], step.g_np[b, j], cov[b, j] >= 0.9, j,
                                           w.lam, w.g_ref, 0.1, 80, 150, 0.9, prev_first, nbc, 13,
                                           0, 0, step.own_first, nbc)
                assert len(r) <= idx_h.shape[-1]
                idx_h[b, h, j] = -1
                idx_h[b, h, j, :len(r)] = torch.from_numpy(np.asarray(r, dtype=np.int32))
                cnt_h[b, h, j] = len(r)
                routes[(b, h, j)] = r
    return idx_h.to(DEV), cnt_h.to(DEV), routes


def test_attn_on_the_pages_variable_length_routes_chunk48():
    # Velox, Methodology Steps 5-6: covered query blocks get the previous
    # chunk plus the best blocks up to K_cov, uncovered ones a mass prefix of
    # up to K_unc, both joined with the window and the own chunk, so one
    # launch mixes routes of very different lengths (the bench's velox_route
    # and geometry_prior lines time exactly this).
    w = synth.CONFIGS[4]
    step = hx.build_step(w, DEV, chunk=48, pooled_keys=True)
    cov = synth.coverage(w, 48, step.n_own)
    heads = (7, 16)
    idx, cnt, routes = _velox_attn_routes(step, heads, cov)
    lens = sorted({len(r) for r in routes.values()})
    assert len(lens) > 5 and lens[0] < 140 and lens[-1] > 200, lens
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    items = [(0, h, j) for h in heads for j in range(step.n_own)]
    _compare(step, routes, o, lse, items)


@pytest.mark.parametrize("top_k", [256, 32])
def test_attn_config5_sample(top_k):
    step = hx.build_step(synth.CONFIGS[5], DEV, top_k=top_k)
    idx, cnt, routes = hx.attn_routes(step, (0, 39))
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    items = [(b, h, j) for b in (0, 1) for h in (0, 39) for j in (0, 31)]
    _compare(step, routes, o, lse, items)


def test_attn_dense_route_equals_dense_attention():
    # Selecting every block is dense attention over the cache (config 5 shape
    # with fewer heads): compare a full head against the oracle.
    w = synth.CONFIGS[5]
    step = hx.build_step(w, DEV, top_k=10 ** 6)
    idx, cnt = hx.route(step)
    assert torch.all(cnt == step.cache.n_blocks)
    assert torch.equal(idx[0, 0, 0], torch.arange(step.cache.n_blocks, dtype=torch.int32, device=DEV))
    idx, cnt, routes = hx.attn_routes(step, (7,))
    assert all(len(r) == step.cache.n_blocks for r in routes.values())
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    items = [(1, 7, j) for j in range(step.n_own)]
    _compare(step, routes, o, lse, items)


def test_attn_index_order_invariance():
    step = hx.build_step(synth.CONFIGS[2], DEV)
    idx, cnt = hx.route(step)
    o1, l1 = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    g = torch.Generator().manual_seed(3)
    perm = torch.randperm(idx.shape[-1], generator=g).to(DEV)
    idx2 = idx[..., perm].contiguous()
    o2, l2 = bsa.bsa_attn(step.q_blk, step.cache, idx2, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    assert (l1 - l2).abs().max().item() <= 1e-4


def test_attn_empty_route_and_single_key():
    w = synth.CONFIGS[1]
    step = hx.build_step(w, DEV)
    B, Hh, J = w.B, w.Hh, step.n_own
    idx = torch.full((B, Hh, J, 1), -1, dtype=torch.int32, device=DEV)
    cnt = torch.zeros((B, Hh, J), dtype=torch.int32, device=DEV)
    # (b, h, j) = (0, 1, 1) attends to one block whose only valid row is row 0.
    step.cache.block_valid[3] = 1
    idx[0, 1, 1, 0] = 3
    cnt[0, 1, 1] = 1
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    assert torch.all(o[0, 0] == 0) and torch.all(torch.isneginf(lse[0, 0]))
    assert torch.all(o[0, 1, :128] == 0)
    q, kc, vc = hx.oracle_blocks(step, [(0, 1)])[(0, 1)]     # the oracle's own cache
    v0 = torch.from_numpy(vc[0, 0, 3, 0]).float()
    got = o[0, 1, 128:256].float().cpu()
    assert torch.allclose(got, v0.expand_as(got), atol=1e-2)
    exp_lse = torch.from_numpy(q[0, 0, 128:256] @ kc[0, 0, 3, 0]) * w.sm_scale
    assert torch.allclose(lse[0, 1, 128:256].double().cpu(), exp_lse, atol=1e-3)


def test_attn_zero_query_is_mean_of_values():
    step = hx.build_step(synth.CONFIGS[2], DEV)
    idx, cnt, routes = hx.attn_routes(step, (3,))
    step.q_blk.zero_()
    o, lse = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    sel = [int(x) for x in routes[(0, 3, 5)]]
    _, _, vc = hx.oracle_blocks(step, [(0, 3)])[(0, 3)]     # the oracle's own cache
    valid = hx.oracle_valid(step)
    vals = np.concatenate([vc[0, 0, n, :valid[n]] for n in sel])
    mean = torch.from_numpy(vals.mean(0)).float()
    assert torch.allclose(o[0, 3, 5 * 128:6 * 128].float().cpu(), mean.expand(128, -1), atol=1e-2)
    n_keys = int(sum(valid[n] for n in sel))
    assert torch.allclose(lse[0, 3, 5 * 128:6 * 128],
                          torch.full((128,), float(np.log(n_keys)), device=DEV), atol=1e-3)


def test_attn_bad_index_reported_not_faulted():
    step = hx.build_step(synth.CONFIGS[1], DEV)
    idx, cnt = hx.route(step)
    idx[0, 0, 0, 0] = 10 ** 6
    bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    status, code = bsa.bsa_check_device_error(DEV)
    assert status == 6 and code == 1
    cnt[0, 0, 0] = idx.shape[-1] + 5
    idx[0, 0, 0, 0] = 0
    bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    status, code = bsa.bsa_check_device_error(DEV)
    assert status == 6 and code == 2


@pytest.mark.parametrize("key", [1, 3, 4])
def test_attn_tokens_equals_attn_then_reorder(key):
    # O and LSE written straight to raster token order: the same numbers as
    # bsa_attn followed by bsa_blocks_to_tokens (same arithmetic, only the
    # destination differs), and the pad rows of the tail block write nothing.
    w = synth.CONFIGS[key]
    T, H, W = w.grid
    step = hx.build_step(w, DEV, chunk=6 if key == 4 else None)
    idx, cnt = hx.route(step)
    o_blk, lse_blk = bsa.bsa_attn(step.q_blk, step.cache, idx, cnt, q_valid=step.q_valid)
    o_ref = bsa.bsa_blocks_to_tokens(o_blk, T, H, W)
    N = T * H * W
    o_tok = torch.full((w.B, N, w.Hh, w.D), 7.0, dtype=torch.bfloat16, device=DEV)
    lse_tok = torch.full((w.B, N, w.Hh), 7.0, dtype=torch.float32, device=DEV)
    bsa.bsa_attn_tokens(step.q_blk, step.cache, idx, cnt, T, H, W, q_valid=step.q_valid,
                        o=o_tok, lse=lse_tok)
    bsa.raise_on_device_error(DEV)
    assert torch.equal(o_tok.view(torch.int16), o_ref.view(torch.int16))
    perm = torch.from_numpy(bsa.bsa_gilbert_perm(T, H, W).astype(np.int64)).to(DEV)
    lse_ref = lse_blk[:, :, perm].permute(0, 2, 1)            # [B, N, Hh]
    assert torch.equal(lse_tok, lse_ref)
    # Without a permutation table the kernel locates the rows' tokens on the
    # Gilbert curve itself: the same output.
    o2 = torch.full_like(o_tok, 7.0)
    l2 = torch.full_like(lse_tok, 7.0)
    bsa.bsa_attn_tokens(step.q_blk, step.cache, idx, cnt, T, H, W, q_valid=step.q_valid,
                        o=o2, lse=l2, table=False)
    bsa.raise_on_device_error(DEV)
    assert torch.equal(o2.view(torch.int16), o_tok.view(torch.int16))
    assert torch.equal(l2, lse_tok)


def test_attn_tokens_against_the_oracle_config3():
    # Parity of the token-order output itself: the oracle's O and LSE of two
    # heads, gathered back to raster order by the oracle's own curve.
    import oracle
    w = synth.CONFIGS[3]
    T, H, W = w.grid
    step = hx.build_step(w, DEV)
    heads = (2, 21)
    idx, cnt, routes = hx.attn_routes(step, heads)
    o_tok, lse_tok = bsa.bsa_attn_tokens(step.q_blk, step.cache, idx, cnt, T, H, W,
                                         q_valid=step.q_valid)
    bsa.raise_on_device_error(DEV)
    items = [(0, h, j) for h in heads for j in range(step.n_own)]
    refs = hx.oracle_attn_items(step, routes, items)
    for hi, h in enumerate(heads):
        ro = np.concatenate([refs[hi * step.n_own + j][0] for j in range(step.n_own)])
        rl = np.concatenate([refs[hi * step.n_own + j][1] for j in range(step.n_own)])
        ro_tok = oracle.blocks_to_tokens(ro[None, None], T, H, W)[0, :, 0]       # [N, D]
        rl_tok = oracle.blocks_to_tokens(rl[None, None, :, None], T, H, W)[0, :, 0, 0]
        got = o_tok[0, :, h].double().cpu().numpy()
        rel = np.linalg.norm(got - ro_tok) / np.linalg.norm(ro_tok)
        assert rel <= hx.O_REL_L2 and np.max(np.abs(got - ro_tok)) <= hx.O_MAX_ABS, (h, rel)
        assert np.max(np.abs(lse_tok[0, :, h].double().cpu().numpy() - rl_tok)) <= hx.LSE_MAX_ABS
