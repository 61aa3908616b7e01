"""Seeded synthetic geometry for the overlap prior: cameras, slabs, tokens.

The pages build slabs with a reconstruction backend (depth, poses, masks)
that is not available here, so this module draws them from a small
analytic scene instead.  It holds none of the method's arithmetic (no boxes,
no overlap, no coverage).

Recipe (all float32, seeded):

* one pinhole camera per latent frame, shared intrinsics fx = fy = W/2,
  cx = W/2, cy = H/2 (a 90-degree horizontal field of view on the latent
  grid); frame f sits at (0.35 sin(0.03 f), 0.05 sin(0.05 f), 0.04 f) and
  turns about the vertical axis by 0.15 sin(0.02 f) radians;
* the scene is a wall at world z = 14; a ray's depth is the camera-z
  distance to it;
* block b of a chunk covers, in frame min(b // tiles_per_frame, T - 1), the
  latent tile (b mod tiles_per_frame) of size th x tw (the tiles of a
  chunk's block grid); its first slab is that tile with the wall's depth
  range over the tile's corners widened by 3 % on each side; 10 % of first
  slabs are invalid (camera -1), as validity gates would drop them;
* a second slab exists for 25 % of blocks: a foreground object on a random
  half-size sub-rectangle of the tile with a depth interval [d, d + 0.4],
  d ~ U(3, 8);
* the query chunk's 128 tokens per block are the first 128 cells of the
  block's tile (row-major), at cell centres, with the wall depth times
  (1 + N(0, 0.01^2)); 8 % of tokens have no depth (camera -1).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

WALL_Z = 14.0


@dataclass
class SlabScene:
    intr: tuple            # (fx, fy, cx, cy)
    cams: np.ndarray       # float32 [n_frames, 12]: R (row-major), centre
    h_cam: np.ndarray      # int32 [n_hist, 2]
    h_rect: np.ndarray     # float32 [n_hist, 2, 6]: u0, u1, v0, v1, d0, d1
    q_cam: np.ndarray      # int32 [n_q, 2]
    q_rect: np.ndarray     # float32 [n_q, 2, 6]
    tok_cam: np.ndarray    # int32 [n_q, 128]
    tok_uvd: np.ndarray    # float32 [n_q, 128, 3]


def _camera(f: int):
    yaw = 0.15 * np.sin(0.02 * f)
    cy, sy = np.cos(yaw), np.sin(yaw)
    R = np.array([[cy, 0.0, sy], [0.0, 1.0, 0.0], [-sy, 0.0, cy]])
    c = np.array([0.35 * np.sin(0.03 * f), 0.05 * np.sin(0.05 * f), 0.04 * f])
    return R, c


def _wall_depth(R, c, intr, u, v):
    fx, fy, cx, cy = intr
    ray = R @ np.array([(u - cx) / fx, (v - cy) / fy, 1.0])
    return (WALL_Z - c[2]) / ray[2]


def slab_scene(grid, n_hist_chunks: int, blocks_per_chunk: int, seed: int,
               tile=(10, 13)) -> SlabScene:
    """Scene for a query chunk that follows ``n_hist_chunks`` history chunks of
    ``blocks_per_chunk`` blocks each (history block index = chunk * bpc + b)."""
    T, H, W = grid
    th, tw = tile
    ty_n, tx_n = -(-H // th), -(-W // tw)
    tiles = ty_n * tx_n
    intr = (W / 2.0, W / 2.0, W / 2.0, H / 2.0)
    n_frames = (n_hist_chunks + 1) * T
    cams = np.zeros((n_frames, 12), np.float64)
    for f in range(n_frames):
        R, c = _camera(f)
        cams[f, :9] = R.ravel()
        cams[f, 9:] = c
    rng = np.random.default_rng(seed)

    def block_slabs(chunk: int, b: int):
        t = min(b // tiles, T - 1)
        k = b % tiles
        ty, tx = k // tx_n, k % tx_n
        u0, u1 = float(tx * tw), float(min((tx + 1) * tw, W))
        v0, v1 = float(ty * th), float(min((ty + 1) * th, H))
        f = chunk * T + t
        R, c = _camera(f)
        ds = [_wall_depth(R, c, intr, u, v) for u in (u0, u1) for v in (v0, v1)]
        cam = np.full(2, -1, np.int32)
        rect = np.zeros((2, 6), np.float64)
        rect[0] = (u0, u1, v0, v1, min(ds) * 0.97, max(ds) * 1.03)
        if rng.random() >= 0.10:
            cam[0] = f
        su, sv = (u1 - u0) / 2, (v1 - v0) / 2
        ou, ov = rng.uniform(0, su), rng.uniform(0, sv)
        d = rng.uniform(3.0, 8.0)
        rect[1] = (u0 + ou, u0 + ou + su, v0 + ov, v0 + ov + sv, d, d + 0.4)
        if rng.random() < 0.25:
            cam[1] = f
        return cam, rect, (t, ty, tx, f)

    n_hist = n_hist_chunks * blocks_per_chunk
    h_cam = np.zeros((n_hist, 2), np.int32)
    h_rect = np.zeros((n_hist, 2, 6), np.float64)
    for ch in range(n_hist_chunks):
        for b in range(blocks_per_chunk):
            h_cam[ch * blocks_per_chunk + b], h_rect[ch * blocks_per_chunk + b], _ = block_slabs(ch, b)
    q_cam = np.zeros((blocks_per_chunk, 2), np.int32)
    q_rect = np.zeros((blocks_per_chunk, 2, 6), np.float64)
    tok_cam = np.full((blocks_per_chunk, 128), -1, np.int32)
    tok_uvd = np.zeros((blocks_per_chunk, 128, 3), np.float64)
    for b in range(blocks_per_chunk):
        q_cam[b], q_rect[b], (t, ty, tx, f) = block_slabs(n_hist_chunks, b)
        R, c = _camera(f)
        cells = [(h, w) for h in range(ty * th, min((ty + 1) * th, H))
                 for w in range(tx * tw, min((tx + 1) * tw, W))][:128]
        for r, (h, w) in enumerate(cells):
            u, v = w + 0.5, h + 0.5
            d = _wall_depth(R, c, intr, u, v) * (1.0 + 0.01 * rng.standard_normal())
            tok_uvd[b, r] = (u, v, d)
            if rng.random() >= 0.08:
                tok_cam[b, r] = f
    f32 = np.float32
    return SlabScene(tuple(float(f32(x)) for x in intr), cams.astype(f32), h_cam, h_rect.astype(f32),
                     q_cam, q_rect.astype(f32), tok_cam, tok_uvd.astype(f32))
