"""CPU models of the selection steps in csrc/route.cu, checked against a
plain stable sort.

* topk_row_kernel: the K-th largest key found bit by bit from the top (the
  largest t with #{key >= t} >= K), stopping early once a count is exactly
  K; then the keys above t and the lowest-indexed keys equal to t.  Thread
  t of 128 holds blocks c*128 + t; padding keys are 0.
* velox_select_kernel: the budget's blocks put in (score descending, index
  ascending) order by counting, for each packed 64-bit sort value, the
  values below it; and compactions where thread t owns the contiguous
  blocks [t*run, (t+1)*run) and a scan over the per-thread counts gives
  every thread its output offset.

The selection a route needs is "the K best, ties to the lowest index" (the
top-K of the pages' routing, with the tie rule the oracle states); these
models must give exactly that on keys with heavy ties.
"""
import numpy as np
import pytest

THREADS = 128


def _reference_topk(keys, K):
    order = sorted(range(len(keys)), key=lambda n: (-int(keys[n]), n))
    return sorted(order[:K])


def _register_topk(keys, K, kpl):
    nh = len(keys)
    held = np.zeros(kpl * THREADS, dtype=np.uint64)      # block c*128 + t, padding 0
    held[:nh] = keys
    thr, exact = 0, False
    for bit in range(31, -1, -1):
        cand = thr | (1 << bit)
        cnt = int((held >= cand).sum())
        if cnt >= K:
            thr = cand
            if cnt == K:
                exact = True
                break
    need_eq = 0 if exact else K - int((held > thr).sum())
    out, eq_seen = [], 0
    for c in range(kpl):                                  # group c, threads in order
        for t in range(THREADS):
            n = c * THREADS + t
            if n >= nh:
                continue
            k = int(held[n])
            if exact:
                if k >= thr:
                    out.append(n)
            elif k > thr:
                out.append(n)
            elif k == thr:
                if eq_seen < need_eq:
                    out.append(n)
                eq_seen += 1
    return out


def _keys(rng, kind, n):
    if kind == "distinct":
        return rng.integers(1, 2 ** 32, n, dtype=np.uint64)
    if kind == "few values":
        return rng.integers(1, 5, n, dtype=np.uint64)
    if kind == "all equal":
        return np.full(n, 7, dtype=np.uint64)
    # order-preserving keys of normal fp32 scores, as score_key makes them
    u = rng.normal(0, 1, n).astype(np.float32).view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


@pytest.mark.parametrize("kind", ["distinct", "few values", "all equal", "fp32 scores"])
def test_register_topk_equals_stable_sort(kind):
    rng = np.random.default_rng(11)
    for _ in range(60):
        nh = int(rng.integers(2, 3073))
        K = int(rng.integers(1, nh))
        kpl = 4 if nh <= 512 else 10 if nh <= 1280 else 18 if nh <= 2304 else 24
        keys = _keys(rng, kind, nh)
        assert _register_topk(keys, K, kpl) == _reference_topk(keys, K), (kind, nh, K)


def test_register_topk_stops_early_on_distinct_scores():
    # With distinct fp32 scores the count hits K exactly long before the
    # last bit; with all keys equal it never does.
    def passes(keys, K=64):
        thr, n = 0, 0
        for bit in range(31, -1, -1):
            n += 1
            cand = thr | (1 << bit)
            cnt = int((keys >= cand).sum())
            if cnt >= K:
                thr = cand
                if cnt == K:
                    break
        return n
    rng = np.random.default_rng(3)
    assert passes(_keys(rng, "fp32 scores", 2303)) < 32
    assert passes(_keys(rng, "all equal", 2303)) == 32


def _pack(key, n):
    # ascending order of ~((key << 32) | ~n) = descending key, ascending n
    return (~((int(key) << 32) | (0xFFFFFFFF - n))) & 0xFFFFFFFFFFFFFFFF


def test_rank_by_counting_is_the_sorted_order():
    rng = np.random.default_rng(5)
    for kind in ("distinct", "few values", "fp32 scores"):
        keys = _keys(rng, kind, 400)
        chosen = sorted(rng.choice(400, size=150, replace=False).tolist())
        vals = [_pack(keys[n], n) for n in chosen]
        order = [None] * len(vals)
        for x, n in zip(vals, chosen):
            rank = sum(1 for y in vals if y < x)
            order[rank] = n
        assert order == sorted(chosen, key=lambda n: (-int(keys[n]), n))


def test_contiguous_runs_compact_in_block_order():
    rng = np.random.default_rng(9)
    threads = 256
    for nh in (1, 255, 256, 257, 2303, 4097):
        flags = rng.random(nh) < 0.3
        run = -(-nh // threads)
        counts = [int(flags[min(t * run, nh):min(t * run + run, nh)].sum()) for t in range(threads)]
        offsets = np.concatenate([[0], np.cumsum(counts)[:-1]])
        out = [None] * int(flags.sum())
        for t in range(threads):
            at = int(offsets[t])
            for n in range(min(t * run, nh), min(t * run + run, nh)):
                if flags[n]:
                    out[at] = n
                    at += 1
        assert out == [n for n in range(nh) if flags[n]]
