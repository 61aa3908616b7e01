"""Shared helpers of the GPU parity tests: build a workload's state on the
device through the library, and build the oracle's own inputs from the same
seeded generators.  The oracle never reads an output of the library: its
cache is its own Gilbert scatter of the generated tokens, its valid-row
counts its own, and where a test needs a route for attention, the route is
the oracle's and the library attends over the same list."""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

import block_sparse_kv_bsa_b200 as bsa
import synth

BLK = 128


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


@dataclass
class Step:
    """Everything one query chunk's routing and attention needs."""
    w: synth.Workload
    cache: bsa.KVCache
    q_tok: torch.Tensor
    q_blk: torch.Tensor
    g: Optional[torch.Tensor]
    g_np: Optional[np.ndarray]
    n_hist: int
    own_first: int
    n_own: int
    q_valid: torch.Tensor
    chunk: int
    top_k: int
    hist_chunks: int = 0      # chunks 1..hist_chunks appended as history (after any direct blocks)
    qc: int = 1               # the chunk whose tokens form the own chunk
    device: str = "cuda"


def build_step(w: synth.Workload, device="cuda", chunk: Optional[int] = None,
               top_k: Optional[int] = None, extra_blocks: int = 0,
               pooled_keys: bool = False) -> Step:
    """Fill a cache with the workload's history, append the query chunk, and
    lay out Q in block order.  ``chunk`` selects the query chunk of the
    48-chunk sweep (1-based; default: the workload's own history length)."""
    T, H, W = w.grid
    nbc = w.blocks_per_chunk
    if chunk is None:
        chunk = w.hist_chunks + 1
    hist_chunks = chunk - 1 if w.hist_direct == 0 else 0
    n_hist = w.hist_direct + hist_chunks * nbc
    cache = bsa.KVCache(w.B, w.Hh, w.D, n_hist + nbc + extra_blocks, device=device,
                        pooled_keys=pooled_keys)
    if w.hist_direct:
        kd, vd = synth.direct_blocks(w, w.hist_direct, device=device)
        cache.k[:, :, :w.hist_direct] = kd
        cache.v[:, :, :w.hist_direct] = vd
        cache.block_valid[:w.hist_direct] = BLK
        cache.n_blocks = w.hist_direct
        if pooled_keys:
            bsa.bsa_kv_pool_means(cache, 0, w.hist_direct)
    for c in range(1, hist_chunks + 1):
        t = synth.chunk_tokens(w, c, device=device, want=("k", "v"))
        bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
    qc = chunk if w.hist_direct == 0 else 1
    t = synth.chunk_tokens(w, qc, device=device)
    own_first = bsa.bsa_kv_append(cache, t["k"], t["v"], T, H, W)
    q_blk = bsa.bsa_tokens_to_blocks(t["q"], T, H, W)
    g_np = synth.prior(w, qc, nbc, n_hist) if n_hist > 0 else None
    g = torch.from_numpy(g_np).to(device) if g_np is not None else None
    q_valid = cache.block_valid[own_first:own_first + nbc].clone()
    return Step(w, cache, t["q"], q_blk, g, g_np, n_hist, own_first, nbc, q_valid, chunk,
                w.top_k[0] if top_k is None else top_k, hist_chunks, qc, str(device))


def route(step: Step, **kw):
    return bsa.bsa_route(step.q_blk, step.cache, step.n_hist, step.own_first, step.n_own,
                         step.top_k, g=step.g, lam=step.w.lam, g_ref=step.w.g_ref,
                         sm_scale=step.w.sm_scale, q_valid=step.q_valid, **kw)


def oracle_valid(step: Step) -> np.ndarray:
    """The oracle's valid-row count of every cache block: direct blocks full,
    each appended chunk's from its own grid."""
    import oracle
    T, H, W = step.w.grid
    per = np.asarray(oracle.block_valid_for(T, H, W), dtype=np.int64)
    return np.concatenate([np.full(step.w.hist_direct, BLK, dtype=np.int64),
                           np.tile(per, step.hist_chunks + 1)])


def oracle_blocks(step: Step, pairs, want_v: bool = True) -> dict:
    """The oracle's Q blocks and K/V cache of each (b, h) in ``pairs``, fp64:
    {(b, h): (q [1, 1, n_own*128, D], k [1, 1, n_hist+n_own, 128, D], v or
    None)}.  Built from the seeded generators (the same draws the library
    appended) by the oracle's own Gilbert scatter."""
    import oracle
    w = step.w
    T, H, W = w.grid
    pairs = sorted(set(pairs))
    ks = {p: [] for p in pairs}
    vs = {p: [] for p in pairs}
    if w.hist_direct:
        kd, vd = synth.direct_blocks(w, w.hist_direct, device=step.device)
        for b, h in pairs:
            ks[(b, h)].append(f64(kd[b:b + 1, h:h + 1]))
            if want_v:
                vs[(b, h)].append(f64(vd[b:b + 1, h:h + 1]))
    for c in list(range(1, step.hist_chunks + 1)) + [step.qc]:
        t = synth.chunk_tokens(w, c, device=step.device, want=("k", "v"))
        for b, h in pairs:
            ks[(b, h)].append(oracle.tokens_to_blocks(f64(t["k"][b:b + 1, :, h:h + 1]), T, H, W))
            if want_v:
                vs[(b, h)].append(oracle.tokens_to_blocks(f64(t["v"][b:b + 1, :, h:h + 1]),
                                                          T, H, W))
    out = {}
    for b, h in pairs:
        q = oracle.tokens_to_blocks(f64(step.q_tok[b:b + 1, :, h:h + 1]), T, H, W)
        out[(b, h)] = (q.reshape(1, 1, -1, w.D), np.concatenate(ks[(b, h)], axis=2),
                       np.concatenate(vs[(b, h)], axis=2) if want_v else None)
    return out


def _oracle_model_scores(step: Step, heads) -> np.ndarray:
    import oracle
    w = step.w
    heads = list(heads)
    blocks = oracle_blocks(step, [(b, h) for b in range(w.B) for h in heads], want_v=False)
    q = np.stack([np.stack([blocks[(b, h)][0][0, 0] for h in heads]) for b in range(w.B)])
    kc = np.stack([np.stack([blocks[(b, h)][1][0, 0, :step.n_hist] for h in heads])
                   for b in range(w.B)])
    valid = oracle_valid(step)
    B, Hs, R, D = q.shape
    qm = oracle.pool_blocks(q.reshape(B, Hs, step.n_own, BLK, D),
                            [int(v) for v in valid[step.own_first:step.own_first + step.n_own]])
    km = oracle.pool_blocks(kc, valid[:step.n_hist])
    return oracle.block_scores(qm, km, w.sm_scale)


def oracle_scores(step: Step, heads) -> np.ndarray:
    """Oracle fused scores s' [B, len(heads), n_own, n_hist]."""
    import oracle
    s = _oracle_model_scores(step, heads)
    return oracle.fuse_prior(s, step.g_np, step.w.lam, step.w.g_ref)


def oracle_scores_model(step: Step, heads) -> np.ndarray:
    """Oracle model scores s = sm_scale * <qmean, kmean> (no prior) [B, len(heads), n_own, n_hist]."""
    return _oracle_model_scores(step, heads)


def oracle_routes(step: Step, heads) -> dict:
    """The oracle's route of every query block of ``heads``: {(b, h, j): blocks}."""
    import oracle
    s = oracle_scores(step, heads)
    return {(b, h, j): oracle.top_k_with_own(s[b, hi, j], step.top_k, step.own_first, step.n_own)
            for b in range(step.w.B) for hi, h in enumerate(heads) for j in range(step.n_own)}


def attn_routes(step: Step, heads):
    """Routes for an attention parity test: (idx, cnt, routes).  The query
    blocks of ``heads`` get the oracle's route, so the library and the oracle
    attend over the same list, chosen by the oracle; the other heads keep the
    library's own route (their outputs are not compared)."""
    idx, cnt = route(step)
    routes = oracle_routes(step, heads)
    idx_h, cnt_h = idx.cpu(), cnt.cpu()
    for (b, h, j), r in routes.items():
        assert len(r) <= idx_h.shape[-1]
        idx_h[b, h, j] = -1
        idx_h[b, h, j, :len(r)] = torch.from_numpy(np.asarray(r, dtype=np.int32))
        cnt_h[b, h, j] = len(r)
    return idx_h.to(idx.device), cnt_h.to(cnt.device), routes


def check_route_rows(idx: np.ndarray, cnt: np.ndarray, scores: np.ndarray, top_k: int,
                     own_first: int, n_own: int, rel_tol: float = 1e-5) -> int:
    """Compare GPU routes with the oracle's, row by row.

    The route must equal the oracle's exactly, except that a block may be
    swapped with another whose oracle score lies within ``rel_tol`` (relative
    to max(|K-th score|, mean |score| of the row)) of the K-th score: fp32
    on the GPU and fp64 in the oracle may order such near-ties differently.
    Returns the number of rows that needed the near-tie rule.
    """
    import oracle
    n_hist = scores.shape[-1]
    K = min(top_k, n_hist)
    ties = 0
    B, Hs, J = cnt.shape
    for b in range(B):
        for h in range(Hs):
            for j in range(J):
                row = scores[b, h, j]
                want = oracle.top_k_with_own(row, top_k, own_first, n_own)
                assert int(cnt[b, h, j]) == K + n_own
                got = idx[b, h, j, :K + n_own]
                assert np.all(idx[b, h, j, K + n_own:] == -1)
                assert np.array_equal(got[K:], np.arange(own_first, own_first + n_own))
                assert np.all(np.diff(got[:K]) > 0), "route not sorted ascending"
                if np.array_equal(got, want):
                    continue
                kth = np.sort(row)[::-1][K - 1]
                tol = rel_tol * max(abs(kth), np.mean(np.abs(row)))
                diff = set(got[:K].tolist()) ^ set(want[:K].tolist())
                for n in diff:
                    assert abs(row[n] - kth) <= tol, (b, h, j, n, row[n], kth, tol)
                ties += 1
    return ties


def oracle_attn_items(step: Step, routes: dict, items, sm_scale=None):
    """Oracle O and LSE of the listed (b, h, j) items over ``routes[(b, h, j)]``,
    on the oracle's own cache and Q blocks."""
    import oracle
    sm = step.w.sm_scale if sm_scale is None else sm_scale
    valid = oracle_valid(step)
    blocks = oracle_blocks(step, [(b, h) for b, h, _ in items])
    out = []
    for (b, h, j) in items:
        q, kc, vc = blocks[(b, h)]
        sel = [int(x) for x in routes[(b, h, j)]]
        o, lse = oracle.attn_block(q[:, :, j * BLK:(j + 1) * BLK], kc, vc, valid,
                                   int(valid[step.own_first + j]), 0, 0, 0, sel, sm)
        out.append((o, lse))
    return out


def attn_errors(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray,
                q_valid: int):
    """(relative L2 of O, max |O| error, max |LSE| error) over the valid rows,
    after checking the pad rows are exactly O = 0 and LSE = -inf."""
    assert np.all(o_gpu[q_valid:] == 0)
    assert np.all(np.isneginf(lse_gpu[q_valid:]))
    ov, rv = o_gpu[:q_valid], o_ref[:q_valid]
    rel = float(np.linalg.norm(ov - rv) / max(np.linalg.norm(rv), 1e-30))
    mabs = float(np.max(np.abs(ov - rv))) if q_valid else 0.0
    lerr = float(np.max(np.abs(lse_gpu[:q_valid] - lse_ref[:q_valid]))) if q_valid else 0.0
    return rel, mabs, lerr


# Tolerances: O from bf16 inputs with fp32 accumulation against the fp64
# oracle: relative L2 <= 1e-2 and max abs <= 2e-2.  LSE is fp32 throughout
# apart from the bf16 inputs, and its error is dominated by fp32 rounding of
# the running sum and by ex2.approx (relative error ~2^-22 per term):
# |d LSE| <= 1e-3 leaves a wide margin.
O_REL_L2 = 1e-2
O_MAX_ABS = 2e-2
LSE_MAX_ABS = 1e-3
