"""GPU parity: Gilbert-ordered KV append and token/block reordering.

Bit-exact against the oracle's scatter ("Velox: Spatial Memory Makes World
Models Efficient", Key Contributions 3): the same bf16 values must land in
the same cache slots, pads must be zero and block_valid must be right.
"""
import numpy as np
import pytest
import torch

import block_sparse_kv_bsa_b200 as bsa
import oracle
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy()


def bf16_of(x: np.ndarray) -> np.ndarray:
    """fp64 oracle values (exact bf16 numbers) -> their bf16 bit patterns."""
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy()


@pytest.mark.parametrize("key", [1, 2, 5])
def test_append_bit_exact(key):
    w = synth.CONFIGS[key]
    T, H, W = w.grid
    n_chunks = 3
    cache = bsa.KVCache(w.B, w.Hh, w.D, n_chunks * w.blocks_per_chunk + 1, device=DEV)
    toks = []
    for c in range(1, n_chunks + 1):
        t = synth.chunk_tokens(w, c, device=DEV, want=("k", "v"))
        first = bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
        assert first == (c - 1) * w.blocks_per_chunk
        toks.append(t)
    bsa.raise_on_device_error(DEV)
    assert cache.n_blocks == n_chunks * w.blocks_per_chunk
    nb = w.blocks_per_chunk
    valid = cache.block_valid.cpu().numpy()
    for c, t in enumerate(toks):
        exp_k = oracle.tokens_to_blocks(t["k"].cpu().double().numpy(), T, H, W)
        exp_v = oracle.tokens_to_blocks(t["v"].cpu().double().numpy(), T, H, W)
        got_k = bits(cache.k[:, :, c * nb:(c + 1) * nb])
        got_v = bits(cache.v[:, :, c * nb:(c + 1) * nb])
        assert np.array_equal(got_k, bf16_of(exp_k))
        assert np.array_equal(got_v, bf16_of(exp_v))
        assert np.array_equal(valid[c * nb:(c + 1) * nb], oracle.block_valid_for(T, H, W))
    assert valid[-1] == 0  # untouched spare block


@pytest.mark.parametrize("key", [3, 4])
def test_append_full_size_head_sample(key):
    # Full-size chunk with padding (7800 -> 61 blocks, 6240 -> 49 blocks);
    # the oracle checks a sample of heads bit for bit.
    w = synth.CONFIGS[key]
    T, H, W = w.grid
    nb = w.blocks_per_chunk
    cache = bsa.KVCache(w.B, w.Hh, w.D, 2 * nb, device=DEV)
    t1 = synth.chunk_tokens(w, 1, device=DEV, want=("k", "v"))
    t2 = synth.chunk_tokens(w, 2, device=DEV, want=("k", "v"))
    bsa.bsa_kv_append(cache, t1["k"], t1["v"], T, H, W)
    bsa.bsa_kv_append(cache, t2["k"], t2["v"], T, H, W)
    bsa.raise_on_device_error(DEV)
    for h in (0, w.Hh // 2, w.Hh - 1):
        exp = oracle.tokens_to_blocks(t2["v"][:, :, h:h + 1].cpu().double().numpy(), T, H, W)
        assert np.array_equal(bits(cache.v[:, h:h + 1, nb:2 * nb]), bf16_of(exp))
        exp = oracle.tokens_to_blocks(t1["k"][:, :, h:h + 1].cpu().double().numpy(), T, H, W)
        assert np.array_equal(bits(cache.k[:, h:h + 1, :nb]), bf16_of(exp))
    pad = (nb * 128) - T * H * W
    assert torch.all(cache.k[:, :, 2 * nb - 1, 128 - pad:] == 0)


@pytest.mark.parametrize("grid,D", [((3, 5, 7), 64), ((1, 1, 1), 128), ((2, 8, 16), 128),
                                    ((5, 30, 52), 64)])
def test_tokens_blocks_round_trip(grid, D):
    T, H, W = grid
    x = synth.random_bf16((2, T * H * W, 3, D), seed=7, device=DEV)
    blk = bsa.bsa_tokens_to_blocks(x, T, H, W)
    back = bsa.bsa_blocks_to_tokens(blk, T, H, W)
    bsa.raise_on_device_error(DEV)
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))
    exp = oracle.tokens_to_blocks(x.cpu().double().numpy(), T, H, W)
    assert np.array_equal(bits(blk).reshape(exp.shape), bf16_of(exp))


def test_append_capacity_error_leaves_cache_unchanged():
    w = synth.CONFIGS[1]
    T, H, W = w.grid
    cache = bsa.KVCache(w.B, w.Hh, w.D, w.blocks_per_chunk + 1, device=DEV)
    t = synth.chunk_tokens(w, 1, device=DEV, want=("k", "v"))
    bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
    before = cache.k.clone()
    with pytest.raises(bsa.BsaError) as e:
        bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
    assert e.value.status == 3
    assert cache.n_blocks == w.blocks_per_chunk
    assert torch.equal(cache.k, before)


def test_bad_permutation_is_reported_not_faulted():
    # A permutation entry outside the chunk is skipped and reported.
    import ctypes
    w = synth.CONFIGS[1]
    T, H, W = w.grid
    cache = bsa.KVCache(w.B, w.Hh, w.D, w.blocks_per_chunk, device=DEV)
    t = synth.chunk_tokens(w, 1, device=DEV, want=("k", "v"))
    perm = bsa.gilbert_perm_device(T, H, W, DEV).clone()
    perm[5] = 10 ** 6
    cs = cache.c_struct()
    err = bsa.error_word(DEV)
    st = bsa.lib().bsa_kv_append(ctypes.byref(cs), ctypes.c_void_p(t["k"].data_ptr()),
                                 ctypes.c_void_p(t["v"].data_ptr()), T, H, W,
                                 ctypes.c_void_p(perm.data_ptr()), ctypes.c_void_p(err.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    status, code = bsa.bsa_check_device_error(DEV)
    assert status == 6 and code == 4
    assert bsa.bsa_check_device_error(DEV) == (0, 0)  # cleared


@pytest.mark.parametrize("key", [2, 4])
def test_pooled_key_means_written_at_append(key):
    # The optional pooled-key cache holds the mean of every block's valid key
    # rows (Velox, Methodology Step 4: importance from mean key vectors).
    w = synth.CONFIGS[key]
    T, H, W = w.grid
    nb = w.blocks_per_chunk
    cache = bsa.KVCache(w.B, w.Hh, w.D, 2 * nb, device=DEV, pooled_keys=True)
    heads = list(range(w.Hh)) if w.Hh <= 12 else [0, 9, w.Hh - 1]
    blocks = []                                    # the oracle's own scatter of the tokens
    for c in (1, 2):
        t = synth.chunk_tokens(w, c, device=DEV, want=("k", "v"))
        bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
        blocks.append(oracle.tokens_to_blocks(t["k"][:, :, heads].cpu().double().numpy(), T, H, W))
    bsa.raise_on_device_error(DEV)
    valid = np.tile(oracle.block_valid_for(T, H, W), 2)
    exp = oracle.pool_blocks(np.concatenate(blocks, axis=2), valid)
    got = cache.kmean[:, heads].cpu().double().numpy()
    assert np.allclose(got, exp, rtol=2e-6, atol=2e-7)


def test_pool_means_for_directly_written_blocks():
    w = synth.CONFIGS[3]
    cache = bsa.KVCache(w.B, w.Hh, w.D, 20, device=DEV, pooled_keys=True)
    kd, vd = synth.direct_blocks(w, 20, device=DEV)
    cache.k.copy_(kd)
    cache.v.copy_(vd)
    cache.block_valid.fill_(128)
    cache.block_valid[7] = 33                      # a ragged block
    cache.n_blocks = 20
    bsa.bsa_kv_pool_means(cache, 0, 20)
    bsa.raise_on_device_error(DEV)
    valid = np.full(20, 128)
    valid[7] = 33
    exp = oracle.pool_blocks(kd[:, [0, 23]].cpu().double().numpy(), valid)
    assert np.allclose(cache.kmean[:, [0, 23]].cpu().double().numpy(), exp, rtol=2e-6, atol=2e-7)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_kv_pool_means(cache, 15, 10)       # past max_blocks


def _append_raw(cache, k, v, T, H, W, perm):
    import ctypes
    cs = cache.c_struct()
    st = bsa.lib().bsa_kv_append(ctypes.byref(cs), ctypes.c_void_p(k.data_ptr()),
                                 ctypes.c_void_p(v.data_ptr()), T, H, W,
                                 ctypes.c_void_p(perm.data_ptr()),
                                 ctypes.c_void_p(bsa.error_word(DEV).data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    cache.n_blocks = int(cs.n_blocks)


def test_append_any_permutation():
    # The ABI accepts any permutation of the chunk's tokens, not only the
    # Gilbert table: token i lands in curve slot perm[i] (block perm[i] / 128,
    # row perm[i] % 128), every head, pads zero.
    w = synth.CONFIGS[2]
    T, H, W = w.grid
    N = T * H * W
    nb = w.blocks_per_chunk
    perm_np = np.random.default_rng(7).permutation(N).astype(np.int32)
    perm = torch.from_numpy(perm_np).to(DEV)
    cache = bsa.KVCache(w.B, w.Hh, w.D, nb, device=DEV, pooled_keys=True)
    t = synth.chunk_tokens(w, 1, device=DEV, want=("k", "v"))
    _append_raw(cache, t["k"], t["v"], T, H, W, perm)
    bsa.raise_on_device_error(DEV)
    placed = {}
    for name in ("k", "v"):
        x = t[name].cpu()                                   # [B, N, Hh, D]
        exp = torch.zeros(w.B, w.Hh, nb * 128, w.D, dtype=torch.bfloat16)
        exp[:, :, torch.from_numpy(perm_np).long()] = x.permute(0, 2, 1, 3)
        got = getattr(cache, name).cpu().reshape(w.B, w.Hh, nb * 128, w.D)
        assert torch.equal(got.view(torch.int16), exp.view(torch.int16)), name
        placed[name] = exp
    valid = np.bincount(perm_np // 128, minlength=nb)      # tokens landing in each block
    exp_m = oracle.pool_blocks(placed["k"].double().numpy().reshape(w.B, w.Hh, nb, 128, w.D),
                               valid)
    assert np.allclose(cache.kmean.cpu().double().numpy(), exp_m, rtol=2e-6, atol=2e-7)


@pytest.mark.parametrize("key", [1, 2, 4])
def test_append_means_equal_pool_means_bitwise(key):
    # The append pools the keys while it moves them, with the router's own
    # summation order: recomputing the means from the cache gives the same
    # bits (and so the pooled and the streaming route score the same means).
    w = synth.CONFIGS[key]
    T, H, W = w.grid
    nb = w.blocks_per_chunk
    cache = bsa.KVCache(w.B, w.Hh, w.D, 2 * nb, device=DEV, pooled_keys=True)
    for c in (1, 2):
        t = synth.chunk_tokens(w, c, device=DEV, want=("k", "v"))
        bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
    bsa.raise_on_device_error(DEV)
    at_append = cache.kmean.clone()
    bsa.bsa_kv_pool_means(cache, 0, 2 * nb)
    bsa.raise_on_device_error(DEV)
    assert torch.equal(cache.kmean.view(torch.int32), at_append.view(torch.int32))


def test_append_large_chunk():
    # Chunks above 16384 tokens take the scatter kernel and a separate pooling
    # pass; the cache and the means are the same as the oracle's.
    w = synth.Workload(90, "large-chunk", B=1, Hh=2, D=64, grid=(2, 96, 101))
    T, H, W = w.grid
    nb = w.blocks_per_chunk                                # 19392 tokens: 152 blocks, tail of 64
    cache = bsa.KVCache(w.B, w.Hh, w.D, nb + 1, device=DEV, pooled_keys=True)
    t = synth.chunk_tokens(w, 1, device=DEV, want=("k", "v"))
    bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
    bsa.raise_on_device_error(DEV)
    exp_k = oracle.tokens_to_blocks(t["k"].cpu().double().numpy(), T, H, W)
    assert np.array_equal(bits(cache.k[:, :, :nb]), bf16_of(exp_k))
    valid = cache.block_valid.cpu().numpy()
    assert np.array_equal(valid[:nb], oracle.block_valid_for(T, H, W))
    exp_m = oracle.pool_blocks(exp_k, oracle.block_valid_for(T, H, W))
    assert np.allclose(cache.kmean[:, :, :nb].cpu().double().numpy(), exp_m, rtol=2e-6, atol=2e-7)


@pytest.mark.parametrize("key", [1, 3, 5])
def test_tokens_to_blocks_mean(key):
    # One pass that reorders the query chunk and pools its blocks (Velox,
    # Methodology Step 4: block importance from the mean query).  The blocks
    # must equal bsa_tokens_to_blocks bit for bit, the means the oracle's
    # fp64 means of the valid rows (pads excluded).
    w = synth.CONFIGS[key]
    T, H, W = w.grid
    t = synth.chunk_tokens(w, 1, device=DEV, want=("q",))
    ref = bsa.bsa_tokens_to_blocks(t["q"], T, H, W)
    blk, mean = bsa.bsa_tokens_to_blocks_mean(t["q"], T, H, W)
    bsa.raise_on_device_error(DEV)
    assert torch.equal(blk.view(torch.int16), ref.view(torch.int16))
    heads = list(range(w.Hh)) if w.Hh <= 12 else [0, 17, w.Hh - 1]
    exp_blk = oracle.tokens_to_blocks(t["q"][:, :, heads].cpu().double().numpy(), T, H, W)
    exp = oracle.pool_blocks(exp_blk, oracle.block_valid_for(T, H, W))
    assert np.allclose(mean[:, heads].cpu().double().numpy(), exp, rtol=2e-6, atol=2e-7)


@pytest.mark.parametrize("key,chunk,pooled", [(1, None, False), (3, None, True),
                                              (4, 12, True), (5, None, False)])
def test_route_from_query_means_equals_route(key, chunk, pooled):
    # bsa_route_qmean on the means of bsa_tokens_to_blocks_mean selects what
    # bsa_route selects from the query blocks, bit for bit: every block mean
    # of the library comes from one summation.
    from tests import _harness as hx
    w = synth.CONFIGS[key]
    T, H, W = w.grid
    step = hx.build_step(w, DEV, chunk=chunk, pooled_keys=pooled)
    idx, cnt = hx.route(step)
    _, qm = bsa.bsa_tokens_to_blocks_mean(step.q_tok, T, H, W)
    idx2, cnt2 = bsa.bsa_route_qmean(qm, step.cache, step.n_hist, step.own_first, step.n_own,
                                     step.top_k, g=step.g, lam=w.lam, g_ref=w.g_ref,
                                     sm_scale=w.sm_scale)
    bsa.raise_on_device_error(DEV)
    assert torch.equal(cnt2, cnt)
    assert torch.equal(idx2, idx)


@pytest.mark.parametrize("grid,D", [((3, 5, 7), 64), ((2, 8, 16), 128), ((5, 30, 52), 64),
                                    ((4, 39, 40), 128), ((2, 96, 101), 64)])
def test_without_table_equals_with_table(grid, D):
    # With no permutation table (d_perm NULL) every kernel locates its slots
    # on the Gilbert curve itself; the results equal the table path bit for
    # bit: reordering both ways, reordering with means, and the append
    # (including, at 19392 tokens, the scatter path for large chunks).
    T, H, W = grid
    n = T * H * W
    x = synth.random_bf16((2, n, 3, D), seed=11, device=DEV)
    a = bsa.bsa_tokens_to_blocks(x, T, H, W)
    b = bsa.bsa_tokens_to_blocks(x, T, H, W, table=False)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    ta = bsa.bsa_blocks_to_tokens(a, T, H, W)
    tb = bsa.bsa_blocks_to_tokens(a, T, H, W, table=False)
    assert torch.equal(ta.view(torch.int16), tb.view(torch.int16))
    if n <= 16384:
        am, mm = bsa.bsa_tokens_to_blocks_mean(x, T, H, W)
        bm, nm = bsa.bsa_tokens_to_blocks_mean(x, T, H, W, table=False)
        assert torch.equal(am.view(torch.int16), bm.view(torch.int16))
        assert torch.equal(mm, nm)
    nb = (n + 127) // 128
    caches = []
    for table in (True, False):
        c = bsa.KVCache(2, 3, D, nb + 2, device=DEV, pooled_keys=True)
        bsa.bsa_kv_append(c, x, x.flip(0).contiguous(), T, H, W, table=table)
        caches.append(c)
    bsa.raise_on_device_error(DEV)
    c0, c1 = caches
    assert torch.equal(c0.k.view(torch.int16), c1.k.view(torch.int16))
    assert torch.equal(c0.v.view(torch.int16), c1.v.view(torch.int16))
    assert torch.equal(c0.kmean, c1.kmean)
    assert torch.equal(c0.block_valid, c1.block_valid)
