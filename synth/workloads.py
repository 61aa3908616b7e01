"""Seeded synthetic workloads for the block-sparse KV attention path.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic (no curve, pooling, scoring, routing or attention).
Both the CUDA path and the oracle consume the exact bf16 tensors made here.

The five workloads mirror the shapes the Velox page's setting implies
(chunked latent video, 128-token blocks, head_dim 128, a KV cache that grows
by one chunk at a time) at the sizes listed in :data:`CONFIGS`.  The page's
own model (LingBot-Fast-Cam) and benchmark (WBench) are not available; these
synthetic tensors stand in for them.

Recipe
------
* Q, K, V ~ N(0, 1), drawn in fp32 by a seeded ``torch.Generator`` on the
  requested device, then rounded to bf16 (round to nearest even).
* ``offset_std > 0``: every (batch, head, spatial tile) gets one offset vector
  ~ N(0, offset_std^2) added to all its Q and K tokens, so block means differ
  and routing is not a coin toss.  Tiles are ``tile`` = (tt, th, tw) latent
  cells (about 128 tokens each).
* ``dist == "scaled"``: Q, K ~ N(0, 1) / sqrt(D) and V ~ U(-1, 1).
* geometric prior g ~ Beta(0.5, 2) per (batch, query block, history block),
  30% of the entries set to 0, from numpy's PCG64.
* seeds: chunk c (1-based; the query chunk is the last one) of workload k
  uses seed 1000*k + c; the prior of chunk c uses 1000*k + 500 + c; blocks
  written straight into the cache use 1000*k + 900.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Tuple

import numpy as np
import torch

BLK = 128


@dataclass(frozen=True)
class Workload:
    key: int
    name: str
    B: int
    Hh: int
    D: int
    grid: Tuple[int, int, int]          # (T, H, W) of every chunk
    hist_chunks: int = 0                # history chunks built by appending
    hist_direct: int = 0                # history blocks written straight into the cache
    top_k: Tuple[int, ...] = (0,)
    prior: bool = False
    offset_std: float = 0.0
    tile: Tuple[int, int, int] = (1, 1, 1)
    dist: str = "normal"
    lam: float = 2.0
    g_ref: float = 0.2
    notes: str = field(default="", compare=False)

    @property
    def tokens(self) -> int:
        T, H, W = self.grid
        return T * H * W

    @property
    def blocks_per_chunk(self) -> int:
        return -(-self.tokens // BLK)

    @property
    def n_hist(self) -> int:
        return self.hist_direct + self.hist_chunks * self.blocks_per_chunk

    @property
    def max_blocks(self) -> int:
        return self.n_hist + self.blocks_per_chunk

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


CONFIGS = {
    1: Workload(1, "tiny", B=1, Hh=2, D=64, grid=(2, 8, 16), hist_chunks=4, top_k=(3,)),
    2: Workload(2, "block-offsets", B=1, Hh=12, D=128, grid=(4, 16, 32), hist_chunks=4,
                top_k=(16,), offset_std=0.5, tile=(1, 8, 16)),
    3: Workload(3, "velox-budget", B=1, Hh=24, D=128, grid=(5, 30, 52), hist_direct=143,
                top_k=(50,), prior=True, offset_std=0.5, tile=(1, 10, 13)),
    # 48-chunk sweep: chunk c has 49*(c-1) history blocks; chunk 48 is the headline.
    4: Workload(4, "sweep-48-chunks", B=1, Hh=24, D=128, grid=(4, 30, 52), hist_chunks=47,
                top_k=(64,), prior=True, offset_std=0.5, tile=(1, 10, 13)),
    5: Workload(5, "dense-equivalence", B=2, Hh=40, D=128, grid=(4, 32, 32), hist_chunks=8,
                top_k=(256, 32), dist="scaled"),
}


def chunk_seed(w: Workload, c: int) -> int:
    return 1000 * w.key + c


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(int(seed))
    return g


def chunk_tokens(w: Workload, c: int, device="cpu",
                 want=("q", "k", "v")) -> dict:
    """Raster-order tokens of chunk ``c`` (1-based): bf16 [B, T*H*W, Hh, D].

    The draws happen in a fixed order (q, k, v, q-offsets, k-offsets) whatever
    ``want`` asks for, so a tensor is the same whether or not the others are
    kept.
    """
    gen = _gen(chunk_seed(w, c), device)
    shape = (w.B, w.tokens, w.Hh, w.D)
    dev = torch.device(device)
    if w.dist == "scaled":
        s = 1.0 / math.sqrt(w.D)
        q = torch.randn(shape, generator=gen, device=dev) * s
        k = torch.randn(shape, generator=gen, device=dev) * s
        v = torch.rand(shape, generator=gen, device=dev) * 2.0 - 1.0
    else:
        q = torch.randn(shape, generator=gen, device=dev)
        k = torch.randn(shape, generator=gen, device=dev)
        v = torch.randn(shape, generator=gen, device=dev)
    if w.offset_std > 0:
        tile_of = _tile_index(w, dev)
        n_tiles = int(tile_of.max().item()) + 1
        oq = torch.randn((w.B, n_tiles, w.Hh, w.D), generator=gen, device=dev) * w.offset_std
        ok = torch.randn((w.B, n_tiles, w.Hh, w.D), generator=gen, device=dev) * w.offset_std
        q = q + oq[:, tile_of]
        k = k + ok[:, tile_of]
    out = {"q": q, "k": k, "v": v}
    return {n: out[n].to(torch.bfloat16).contiguous() for n in want}


def _tile_index(w: Workload, dev) -> torch.Tensor:
    """Spatial tile id of every raster token (tiles of ``w.tile`` cells)."""
    T, H, W = w.grid
    tt, th, tw = w.tile
    t = torch.arange(T, device=dev).view(T, 1, 1) // tt
    h = torch.arange(H, device=dev).view(1, H, 1) // th
    x = torch.arange(W, device=dev).view(1, 1, W) // tw
    nh, nw = -(-H // th), -(-W // tw)
    return ((t * nh + h) * nw + x).reshape(-1)


def direct_blocks(w: Workload, n_blocks: int, device="cpu"):
    """History blocks written straight into the cache (all rows valid):
    bf16 [B, Hh, n_blocks, 128, D] for K and V, with per-block offsets on K."""
    gen = _gen(1000 * w.key + 900, device)
    dev = torch.device(device)
    shape = (w.B, w.Hh, n_blocks, BLK, w.D)
    k = torch.randn(shape, generator=gen, device=dev)
    v = torch.randn(shape, generator=gen, device=dev)
    if w.offset_std > 0:
        ok = torch.randn((w.B, w.Hh, n_blocks, 1, w.D), generator=gen, device=dev) * w.offset_std
        k = k + ok
    return k.to(torch.bfloat16).contiguous(), v.to(torch.bfloat16).contiguous()


def prior(w: Workload, c: int, n_q_blocks: int, n_hist: int) -> Optional[np.ndarray]:
    """Geometric overlap prior g (float32 [B, n_q_blocks, n_hist]) or None."""
    if not w.prior:
        return None
    rng = np.random.Generator(np.random.PCG64(1000 * w.key + 500 + c))
    g = rng.beta(0.5, 2.0, size=(w.B, n_q_blocks, n_hist))
    zero = rng.random(size=g.shape) < 0.3
    g[zero] = 0.0
    return g.astype(np.float32)


def coverage(w: Workload, c: int, n_q_blocks: int) -> np.ndarray:
    """Synthetic coverage of each query block (fraction of its tokens inside a
    valid historical slab): float32 [B, n_q_blocks] ~ U(0.5, 1), so that about
    one query block in five is well covered at eta_cov = 0.9."""
    rng = np.random.Generator(np.random.PCG64(1000 * w.key + 700 + c))
    return rng.uniform(0.5, 1.0, size=(w.B, n_q_blocks)).astype(np.float32)


def random_bf16(shape, seed: int, device="cpu", scale: float = 1.0) -> torch.Tensor:
    """Plain N(0, scale^2) bf16 tensor for edge-case tests."""
    gen = _gen(seed, device)
    return (torch.randn(shape, generator=gen, device=torch.device(device)) * scale).to(torch.bfloat16)
