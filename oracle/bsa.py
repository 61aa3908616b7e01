"""Oracle: the block-sparse KV attention path in plain fp64 numpy.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  It shares no
code with the CUDA library; the product path never calls it.

Every function writes out the plain definition of one step of the path in
"Velox: Spatial Memory Makes World Models Efficient" (Methodology Steps 4-6
and Key Contributions 2-3).  There is no tiling, fusion or reordering: loops
run over (batch, head, query block) and each step uses numpy's own
reductions in float64.

Shapes (BLK = 128 tokens per block):

* token layout   ``x_tok``  [B, T*H*W, Hh, D]   raster order (t, h, w)
* block layout   ``x_blk``  [B, Hh, n_blocks, BLK, D]
* ``valid``                 [n_blocks] valid rows per block (pads at the tail)
* ``g``                     [B, n_q_blocks, n_hist] overlap prior in [0, 1]

Readings of the page that are not spelled out there (each one is listed in
the design notes of the repository):

* pad rows are zero in the cache and are excluded from pooling and from the
  softmax; pad query rows give O = 0 and LSE = -inf;
* the block importance is s = sm_scale * <mean q, mean k> and the geometric
  prior is added as s' = s + lambda * min(g / g_ref, 1);
* the top-K candidates are the history blocks; the query block's own chunk is
  always added outside the budget; ties go to the lower block index; the
  list is sorted ascending;
* attention has no causal mask: every key of a selected block is visible;
  LSE uses the natural logarithm.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

from .gilbert import gilbert_perm

BLK = 128


def _f64(x) -> np.ndarray:
    """Upcast anything array-like (numpy or a CPU torch tensor) to float64."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


def n_blocks_for(T: int, H: int, W: int) -> int:
    """Number of 128-token blocks a T x H x W chunk occupies."""
    return -(-T * H * W // BLK)


def block_valid_for(T: int, H: int, W: int) -> np.ndarray:
    """Valid rows of each block of one chunk: 128 everywhere but the tail."""
    n = T * H * W
    nb = n_blocks_for(T, H, W)
    return np.array([min(BLK, n - k * BLK) for k in range(nb)], dtype=np.int64)


# ---------------------------------------------------------------------------
# Gilbert-ordered KV storage (Key Contributions 3; Methodology Step 6)
# ---------------------------------------------------------------------------

def tokens_to_blocks(x_tok, T: int, H: int, W: int) -> np.ndarray:
    """Scatter raster tokens to 128-token blocks in Gilbert order, zero pads.

    Token i (raster) goes to curve slot p = perm[i]: block p // 128, row
    p % 128.  Returns [B, Hh, nb, 128, D] float64.
    """
    x = _f64(x_tok)
    B, N, Hh, D = x.shape
    if N != T * H * W:
        raise ValueError("token count does not match the grid")
    perm = gilbert_perm(T, H, W)
    nb = n_blocks_for(T, H, W)
    out = np.zeros((B, Hh, nb * BLK, D), dtype=np.float64)
    for i in range(N):
        out[:, :, perm[i], :] = x[:, i, :, :]
    return out.reshape(B, Hh, nb, BLK, D)


def blocks_to_tokens(x_blk, T: int, H: int, W: int) -> np.ndarray:
    """Inverse of :func:`tokens_to_blocks`: gather raster tokens back out.

    ``x_blk`` may be [B, Hh, nb, 128, D] or [B, Hh, nb*128, D].
    Returns [B, T*H*W, Hh, D] float64.
    """
    x = _f64(x_blk)
    B, Hh = x.shape[0], x.shape[1]
    D = x.shape[-1]
    x = x.reshape(B, Hh, -1, D)
    N = T * H * W
    perm = gilbert_perm(T, H, W)
    out = np.zeros((B, N, Hh, D), dtype=np.float64)
    for i in range(N):
        out[:, i, :, :] = x[:, :, perm[i], :]
    return out


def kv_append(cache_k: np.ndarray, cache_v: np.ndarray, valid: np.ndarray,
              n_blocks: int, k_tok, v_tok, T: int, H: int, W: int) -> int:
    """Append one chunk to a block cache in place; return the new fill.

    ``cache_k``/``cache_v`` are float64 [B, Hh, max_blocks, 128, D];
    ``valid`` is int [max_blocks].  The chunk occupies blocks
    [n_blocks, n_blocks + nb).
    """
    kb = tokens_to_blocks(k_tok, T, H, W)
    vb = tokens_to_blocks(v_tok, T, H, W)
    nb = kb.shape[2]
    if n_blocks + nb > cache_k.shape[2]:
        raise ValueError("cache capacity exceeded")
    cache_k[:, :, n_blocks:n_blocks + nb] = kb
    cache_v[:, :, n_blocks:n_blocks + nb] = vb
    valid[n_blocks:n_blocks + nb] = block_valid_for(T, H, W)
    return n_blocks + nb


# ---------------------------------------------------------------------------
# Block importance from mean query and mean key (Methodology Step 4)
# ---------------------------------------------------------------------------

def pool_blocks(x_blk, valid: Sequence[int]) -> np.ndarray:
    """Mean of each block over its valid rows: [B, Hh, n, 128, D] -> [B, Hh, n, D]."""
    x = _f64(x_blk)
    B, Hh, n, blk, D = x.shape
    out = np.zeros((B, Hh, n, D), dtype=np.float64)
    for k in range(n):
        v = int(valid[k])
        if v <= 0:
            raise ValueError("a block with no valid rows has no mean")
        out[:, :, k, :] = x[:, :, k, :v, :].mean(axis=2)
    return out


def block_scores(q_mean: np.ndarray, k_mean: np.ndarray, sm_scale: float) -> np.ndarray:
    """s[b, h, j, n] = sm_scale * <q_mean[b, h, j], k_mean[b, h, n]>."""
    return sm_scale * np.einsum("bhjd,bhnd->bhjn", q_mean, k_mean)


def fuse_prior(s: np.ndarray, g: Optional[np.ndarray], lam: float, g_ref: float) -> np.ndarray:
    """s' = s + lambda * min(g / g_ref, 1); g is shared by all heads.

    With g absent the scores pass through unchanged.  A block with full
    overlap gains exactly lambda; a block with no overlap keeps its score.
    """
    if g is None:
        return s.copy()
    g = _f64(g)
    boost = lam * np.minimum(g / g_ref, 1.0)          # [B, J, N]
    return s + boost[:, None, :, :]


def top_k_with_own(scores_row: np.ndarray, top_k: int, own_first: int, n_own: int) -> np.ndarray:
    """Indices of one query block's route, sorted ascending.

    Budgeted part: the ``top_k`` largest history scores, ties to the lower
    index (all history blocks when top_k >= n_hist).  Reserved part: the
    own-chunk blocks [own_first, own_first + n_own), outside the budget.
    """
    n_hist = scores_row.shape[0]
    order = sorted(range(n_hist), key=lambda n: (-scores_row[n], n))
    chosen = sorted(order[:min(top_k, n_hist)])
    return np.array(chosen + list(range(own_first, own_first + n_own)), dtype=np.int64)


def route(q_blk, k_cache, valid, n_hist: int, own_first: int, n_own: int,
          g, lam: float, g_ref: float, sm_scale: float, top_k: int,
          q_valid: Optional[Sequence[int]] = None):
    """Route every (b, h, query block): returns (idx list of lists, fused scores).

    ``q_blk`` [B, Hh, n_own*128, D] (block order), ``k_cache``
    [B, Hh, >= n_hist, 128, D], ``valid`` valid rows per cache block,
    ``q_valid`` valid rows per query block (defaults to the cache's valid
    counts of the own-chunk blocks).
    """
    q = _f64(q_blk)
    B, Hh, nq_rows, D = q.shape
    if nq_rows != n_own * BLK:
        raise ValueError("query rows must be n_own * 128")
    if q_valid is None:
        q_valid = [int(valid[own_first + j]) for j in range(n_own)]
    q_mean = pool_blocks(q.reshape(B, Hh, n_own, BLK, D), q_valid)
    kc = _f64(k_cache)[:, :, :n_hist]
    k_mean = pool_blocks(kc, valid[:n_hist]) if n_hist > 0 else np.zeros((B, Hh, 0, D))
    s = block_scores(q_mean, k_mean, sm_scale)
    s = fuse_prior(s, g, lam, g_ref)
    idx = [[[top_k_with_own(s[b, h, j], top_k, own_first, n_own) for j in range(n_own)]
            for h in range(Hh)] for b in range(B)]
    return idx, s


# ---------------------------------------------------------------------------
# Indexed block-sparse attention (Methodology Step 6)
# ---------------------------------------------------------------------------

def attn_rows(q_rows: np.ndarray, keys: np.ndarray, vals: np.ndarray,
              sm_scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of some query rows over an explicit key set.

    O = softmax(sm_scale * q k^T) v, LSE = log sum exp(sm_scale * q k^T),
    with the maximum subtracted before exponentiation.
    """
    logits = sm_scale * (q_rows @ keys.T)             # [R, N]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ vals) / l
    lse = (m + np.log(l))[:, 0]
    return o, lse


def gather_keys(k_cache, v_cache, valid, b: int, h: int, sel: Sequence[int]):
    """Concatenate the valid rows of the selected blocks of head (b, h)."""
    kk = [np.asarray(k_cache[b, h, n, :int(valid[n])], dtype=np.float64) for n in sel]
    vv = [np.asarray(v_cache[b, h, n, :int(valid[n])], dtype=np.float64) for n in sel]
    return np.concatenate(kk, axis=0), np.concatenate(vv, axis=0)


def attn_block(q_blk, k_cache, v_cache, valid, q_valid_j: int,
               b: int, h: int, j: int, sel: Sequence[int], sm_scale: float):
    """O [128, D] and LSE [128] of query block j of head (b, h).

    Pad query rows (row >= q_valid_j) return O = 0 and LSE = -inf.
    """
    q = np.asarray(q_blk[b, h, j * BLK:(j + 1) * BLK], dtype=np.float64)
    D = q.shape[-1]
    o = np.zeros((BLK, D), dtype=np.float64)
    lse = np.full(BLK, -np.inf, dtype=np.float64)
    if len(sel) == 0 or q_valid_j == 0:
        return o, lse
    keys, vals = gather_keys(k_cache, v_cache, valid, b, h, sel)
    if keys.shape[0] == 0:
        return o, lse
    ov, lv = attn_rows(q[:q_valid_j], keys, vals, sm_scale)
    o[:q_valid_j] = ov
    lse[:q_valid_j] = lv
    return o, lse


def attn(q_blk, k_cache, v_cache, valid, q_valid, idx, cnt, sm_scale: float,
         items: Optional[Sequence[Tuple[int, int, int]]] = None):
    """Block-sparse attention for all (or the listed) (b, h, j) work items.

    ``idx`` [B, Hh, nQB, max_sel] and ``cnt`` [B, Hh, nQB] are the route.
    Returns O [B, Hh, nQB*128, D] and LSE [B, Hh, nQB*128] (float64); rows of
    items not listed stay NaN so a caller cannot mistake them for results.
    """
    q = _f64(q_blk)
    kc = _f64(k_cache)
    vc = _f64(v_cache)
    idx = np.asarray(idx)
    cnt = np.asarray(cnt)
    B, Hh, nrows, D = q.shape
    nqb = nrows // BLK
    o = np.full((B, Hh, nrows, D), np.nan)
    lse = np.full((B, Hh, nrows), np.nan)
    if items is None:
        items = [(b, h, j) for b in range(B) for h in range(Hh) for j in range(nqb)]
    for (b, h, j) in items:
        sel = [int(x) for x in idx[b, h, j, :int(cnt[b, h, j])]]
        ob, lb = attn_block(q, kc, vc, valid, int(q_valid[j]), b, h, j, sel, sm_scale)
        o[b, h, j * BLK:(j + 1) * BLK] = ob
        lse[b, h, j * BLK:(j + 1) * BLK] = lb
    return o, lse


def dense_masked_attn(q_rows, keys_all, vals_all, allowed: np.ndarray, sm_scale: float):
    """Brute force: full logit matrix, -inf where ``allowed`` is False.

    ``allowed`` is a boolean [R, N] mask over all keys.  Rows with no allowed
    key return O = 0 and LSE = -inf.
    """
    q = _f64(q_rows)
    k = _f64(keys_all)
    v = _f64(vals_all)
    logits = sm_scale * (q @ k.T)
    logits = np.where(allowed, logits, -np.inf)
    R, D = q.shape[0], v.shape[1]
    o = np.zeros((R, D))
    lse = np.full(R, -np.inf)
    for r in range(R):
        row = logits[r]
        if not np.any(allowed[r]):
            continue
        m = np.max(row)
        e = np.exp(row - m)
        o[r] = (e @ v) / e.sum()
        lse[r] = m + np.log(e.sum())
    return o, lse


# ---------------------------------------------------------------------------
# The page's full route (Methodology Steps 4-5)
# ---------------------------------------------------------------------------

def vetted_overlap(g: np.ndarray, tau: float, g_ref: float) -> np.ndarray:
    """g_hat: overlap above the noise threshold tau, rescaled by g_ref and
    clipped to 1; overlap at or below tau counts as none."""
    g = _f64(g)
    return np.where(g > tau, np.minimum(g / g_ref, 1.0), 0.0)


def velox_route_row(s_row: np.ndarray, g_row: Optional[np.ndarray], covered: bool,
                    j: int, lam: float, g_ref: float, tau: float, k_cov: int, k_unc: int,
                    mass: float, prev_first: int, n_prev: int, window_half: int,
                    ref_first: int, n_ref: int, own_first: int, n_own: int) -> np.ndarray:
    """Route of one query block j over history blocks [0, len(s_row)).

    Covered query block: the importance distribution softmax(s) is multiplied
    by (1 + lam * g_hat) and renormalised, which ranks blocks exactly like
    s + log(1 + lam * g_hat); the previous chunk's blocks are reserved first,
    then the best remaining blocks fill the budget up to k_cov in total.
    Uncovered query block: the unfused distribution softmax(s) is taken in
    decreasing order (ties to the lower index) up to the smallest prefix whose
    mass reaches `mass`, at most k_unc blocks.
    Both are joined with the window of previous-chunk blocks at Gilbert
    positions j - window_half .. j + window_half, the reference blocks and the
    query block's own chunk; the result is sorted ascending without repeats.
    """
    n_hist = s_row.shape[0]
    chosen = set()
    prev = [prev_first + p for p in range(n_prev) if 0 <= prev_first + p < n_hist]
    if covered:
        f = s_row.copy()
        if g_row is not None:
            f = f + np.log1p(lam * vetted_overlap(g_row, tau, g_ref))
        reserved = set(prev)
        chosen |= reserved
        budget = max(k_cov - len(reserved), 0)
        rest = sorted((n for n in range(n_hist) if n not in reserved), key=lambda n: (-f[n], n))
        chosen |= set(rest[:budget])
    elif n_hist > 0:
        m = s_row.max()
        p = np.exp(s_row - m)
        p = p / p.sum()
        order = sorted(range(n_hist), key=lambda n: (-s_row[n], n))
        acc = 0.0
        for r, n in enumerate(order[:k_unc]):
            chosen.add(n)
            acc += p[n]
            if acc >= mass:
                break
    for pos in range(j - window_half, j + window_half + 1):
        if 0 <= pos < n_prev and 0 <= prev_first + pos < n_hist:
            chosen.add(prev_first + pos)
    for r in range(n_ref):
        if 0 <= ref_first + r < n_hist:
            chosen.add(ref_first + r)
    return np.array(sorted(chosen) + list(range(own_first, own_first + n_own)), dtype=np.int64)


def velox_route(q_blk, k_cache, valid, n_hist: int, own_first: int, n_own: int, g,
                coverage, lam: float, g_ref: float, sm_scale: float, tau: float,
                eta_cov: float, k_cov: int, k_unc: int, mass: float, prev_first: int,
                n_prev: int, window_half: int, ref_first: int = 0, n_ref: int = 0,
                q_valid: Optional[Sequence[int]] = None):
    """The page's route for every (b, h, query block); returns (idx lists, model scores).

    ``coverage`` is [B, n_own] (fraction of a query block's tokens inside a
    valid historical slab) or None (no query block is covered).
    """
    q = _f64(q_blk)
    B, Hh, nq_rows, D = q.shape
    if q_valid is None:
        q_valid = [int(valid[own_first + j]) for j in range(n_own)]
    q_mean = pool_blocks(q.reshape(B, Hh, n_own, BLK, D), q_valid)
    kc = _f64(k_cache)[:, :, :n_hist]
    k_mean = pool_blocks(kc, valid[:n_hist]) if n_hist > 0 else np.zeros((B, Hh, 0, D))
    s = block_scores(q_mean, k_mean, sm_scale)
    g = None if g is None else _f64(g)
    cov = None if coverage is None else _f64(coverage)
    idx = [[[velox_route_row(s[b, h, j], None if g is None else g[b, j],
                             cov is not None and cov[b, j] >= eta_cov, j, lam, g_ref, tau,
                             k_cov, k_unc, mass, prev_first, n_prev, window_half, ref_first,
                             n_ref, own_first, n_own)
             for j in range(n_own)] for h in range(Hh)] for b in range(B)]
    return idx, s
