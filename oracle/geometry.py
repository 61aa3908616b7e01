"""Oracle: the geometric overlap prior g and the coverage score, plain numpy.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this module.  It shares no
code with the CUDA library; the product path never calls it.

"Velox: Spatial Memory Makes World Models Efficient", Methodology Step 3:
each query slab and each historical slab is approximated by a camera-facing
oriented bounding box (OBB); the geometric score of a (query block, KV block)
pair is the intersection-over-union of the query box with the best-matching
historical box, estimated on a deterministic grid after a separating-axis
test; the coverage of a query block is the fraction of its tokens that fall
inside a valid historical slab both spatially and in depth.  Slabs
themselves (Step 1: a source-camera token rectangle and a depth interval)
come from a reconstruction backend the pages describe but do not specify;
here they are inputs.

Readings of the page (each one is listed in the design notes):

* camera model: pinhole, shared intrinsics (fx, fy, cx, cy) in latent-token
  pixels; a camera is (R, c) with X_world = c + R @ X_cam, camera axes
  x right, y down, z forward;
* a slab is (camera, token rectangle [u0, u1] x [v0, v1] in pixel-edge
  coordinates, depth interval [d0, d1]); its camera-facing OBB is the
  smallest box with the camera's axes that contains the slab's frustum
  segment;
* "deterministic OBB grid": n^3 cell centres of the query box, counted
  inside the historical box; intersection I = min(vol(query box) * count /
  n^3, vol(historical box)); IoU = I / (vol_q + vol_h - I), so IoU is in
  [0, 1].  A pair the separating-axis test separates has IoU 0;
* g is the largest IoU over the valid slabs of the two blocks (0 when there
  is none); coverage counts a token when its back-projected point lies in
  some valid slab of any history block (its depth in the slab's camera in
  [d0, d1] and its projection in the rectangle); tokens without depth count
  as uncovered; the denominator is the query block's valid token count.

Precision: the boxes, the separating-axis test, the grid count and the
coverage test decide integers (inside or not), so they are evaluated in
float32, one rounding per operation, in exactly the order written below; the
CUDA kernel takes the same decisions in the same precision and order.
"""
from __future__ import annotations

import numpy as np

F = np.float32
SAT_EPS = F(1e-6)   # added to |R_ij| in the edge-edge tests (near-parallel axes)


def _f(x):
    return np.asarray(x, dtype=np.float32)


def dot3(x, y):
    """(x0*y0 + x1*y1) + x2*y2, float32, one rounding per operation."""
    x = _f(x)
    y = _f(y)
    return (x[..., 0] * y[..., 0] + x[..., 1] * y[..., 1]) + x[..., 2] * y[..., 2]


def slab_box(R, c, intr, rect):
    """Camera-facing OBB of a slab.

    R: [3, 3] world-from-camera rotation, c: [3] camera centre,
    intr: (fx, fy, cx, cy), rect: (u0, u1, v0, v1, d0, d1).
    Returns (centre [3], axes [3, 3] with axis k in column k, half [3]).
    """
    R = _f(R)
    c = _f(c)
    fx, fy, cx, cy = (F(v) for v in intr)
    u0, u1, v0, v1, d0, d1 = (F(v) for v in rect)
    ax0 = (u0 - cx) / fx
    ax1 = (u1 - cx) / fx
    ay0 = (v0 - cy) / fy
    ay1 = (v1 - cy) / fy
    x_lo = min(ax0 * d0, ax0 * d1)
    x_hi = max(ax1 * d0, ax1 * d1)
    y_lo = min(ay0 * d0, ay0 * d1)
    y_hi = max(ay1 * d0, ay1 * d1)
    half_c = F(0.5)
    lc = _f([(x_lo + x_hi) * half_c, (y_lo + y_hi) * half_c, (d0 + d1) * half_c])
    half = _f([(x_hi - x_lo) * half_c, (y_hi - y_lo) * half_c, (d1 - d0) * half_c])
    centre = _f([c[i] + ((R[i, 0] * lc[0] + R[i, 1] * lc[1]) + R[i, 2] * lc[2]) for i in range(3)])
    return centre, R.copy(), half


def sat_separated(box_a, box_b) -> bool:
    """Separating-axis test of two OBBs over the 15 candidate axes (the 3 face
    normals of each box and the 9 edge-edge cross products), written in box
    A's frame: M[i, j] = a_i . b_j, t = A^T (C_b - C_a)."""
    ca, A, e = box_a
    cb, B, f = box_b
    T = _f(cb) - _f(ca)
    t = _f([dot3(A[:, i], T) for i in range(3)])
    M = _f([[dot3(A[:, i], B[:, j]) for j in range(3)] for i in range(3)])
    aM = np.abs(M)
    for i in range(3):          # axes of A
        rb = (f[0] * aM[i, 0] + f[1] * aM[i, 1]) + f[2] * aM[i, 2]
        if abs(t[i]) > e[i] + rb:
            return True
    for j in range(3):          # axes of B
        ra = (e[0] * aM[0, j] + e[1] * aM[1, j]) + e[2] * aM[2, j]
        tj = (t[0] * M[0, j] + t[1] * M[1, j]) + t[2] * M[2, j]
        if abs(tj) > ra + f[j]:
            return True
    aE = aM + SAT_EPS
    for i in range(3):          # a_i x b_j
        i1, i2 = (i + 1) % 3, (i + 2) % 3
        for j in range(3):
            j1, j2 = (j + 1) % 3, (j + 2) % 3
            lhs = abs(t[i2] * M[i1, j] - t[i1] * M[i2, j])
            ra = e[i1] * aE[i2, j] + e[i2] * aE[i1, j]
            rb = f[j1] * aE[i, j2] + f[j2] * aE[i, j1]
            if lhs > ra + rb:
                return True
    return False


def grid_points(n: int) -> np.ndarray:
    """Cell-centre coordinates s_i = (2i+1)/n - 1 in [-1, 1], float32."""
    i = np.arange(n, dtype=np.float32)
    return (F(2) * i + F(1)) / F(n) - F(1)


def grid_count(box_a, box_b, n: int) -> int:
    """Number of the n^3 cell centres of box A that lie inside box B.  A's
    point (x, y, z) (local, scaled by A's half-extents) has coordinates
    q_k = ((t_k + N_k0 x) + N_k1 y) + N_k2 z in B's frame, with
    t = B^T (C_a - C_b) and N[k, l] = b_k . a_l."""
    ca, A, e = box_a
    cb, B, f = box_b
    Dv = _f(ca) - _f(cb)
    t = _f([dot3(B[:, k], Dv) for k in range(3)])
    N = _f([[dot3(B[:, k], A[:, l]) for l in range(3)] for k in range(3)])
    s = grid_points(n)
    x = s * e[0]
    y = s * e[1]
    z = s * e[2]
    inside = np.ones((n, n, n), dtype=bool)
    for k in range(3):
        q = ((t[k] + N[k, 0] * x[:, None, None]) + N[k, 1] * y[None, :, None]) + N[k, 2] * z[None, None, :]
        inside &= np.abs(q) <= f[k]
    return int(inside.sum())


def box_iou(box_a, box_b, n: int) -> np.float32:
    """Grid estimate of IoU(A, B), 0 when the separating-axis test separates
    them or when the union volume is not positive."""
    if sat_separated(box_a, box_b):
        return F(0)
    cnt = grid_count(box_a, box_b, n)
    e = box_a[2]
    f = box_b[2]
    va = ((F(8) * e[0]) * e[1]) * e[2]
    vb = ((F(8) * f[0]) * f[1]) * f[2]
    # The grid count can credit A's cells to a B that is slightly smaller
    # than A; no intersection exceeds either volume.
    inter = min(va * (F(cnt) / F(n * n * n)), vb)
    union = (va + vb) - inter
    if not union > 0:
        return F(0)
    return F(inter / union)


def _cam(cams, i):
    cams = _f(cams)
    return cams[i, :9].reshape(3, 3), cams[i, 9:12]


def prior_g(cams, intr, q_cam, q_rect, h_cam, h_rect, n: int) -> np.ndarray:
    """g[j, m] = max over valid slabs (a of query block j, b of history
    block m) of box_iou(box(a), box(b)); slabs with camera < 0 are absent.

    q_cam: int [nq, S], q_rect: float [nq, S, 6]; h_cam, h_rect likewise for
    the history blocks.  Returns float32 [nq, n_hist]."""
    nq, nh = q_cam.shape[0], h_cam.shape[0]
    qbox = [[slab_box(*_cam(cams, q_cam[j, s]), intr, q_rect[j, s]) if q_cam[j, s] >= 0 else None
             for s in range(q_cam.shape[1])] for j in range(nq)]
    hbox = [[slab_box(*_cam(cams, h_cam[m, s]), intr, h_rect[m, s]) if h_cam[m, s] >= 0 else None
             for s in range(h_cam.shape[1])] for m in range(nh)]
    g = np.zeros((nq, nh), dtype=np.float32)
    for j in range(nq):
        for m in range(nh):
            best = F(0)
            for a in qbox[j]:
                if a is None:
                    continue
                for b in hbox[m]:
                    if b is None:
                        continue
                    v = box_iou(a, b, n)
                    if v > best:
                        best = v
            g[j, m] = best
    return g


def token_point(R, c, intr, u, v, d):
    """World point of the token at pixel (u, v) with depth d (float32)."""
    R = _f(R)
    c = _f(c)
    fx, fy, cx, cy = (F(x) for x in intr)
    u, v, d = F(u), F(v), F(d)
    x = ((u - cx) / fx) * d
    y = ((v - cy) / fy) * d
    return _f([c[i] + ((R[i, 0] * x + R[i, 1] * y) + R[i, 2] * d) for i in range(3)])


def in_slab(X, R, c, intr, rect) -> bool:
    """Does world point X fall inside the slab: depth in the slab's camera
    within [d0, d1] (and positive), projection within the rectangle."""
    R = _f(R)
    c = _f(c)
    fx, fy, cx, cy = (F(x) for x in intr)
    u0, u1, v0, v1, d0, d1 = (F(x) for x in rect)
    Dv = _f(X) - c
    xs = dot3(R[:, 0], Dv)
    ys = dot3(R[:, 1], Dv)
    zs = dot3(R[:, 2], Dv)
    if not (zs > 0 and zs >= d0 and zs <= d1):
        return False
    us = (fx * xs) / zs + cx
    vs = (fy * ys) / zs + cy
    return bool(us >= u0 and us <= u1 and vs >= v0 and vs <= v1)


def coverage(cams, intr, tok_cam, tok_uvd, q_valid, h_cam, h_rect) -> np.ndarray:
    """Fraction of each query block's valid tokens (the first q_valid[j] of
    its 128) that fall inside some valid slab of any history block.
    tok_cam: int [nq, 128] (-1 = no depth), tok_uvd: float [nq, 128, 3]."""
    nq = tok_cam.shape[0]
    slabs = [(_cam(cams, h_cam[m, s]), h_rect[m, s])
             for m in range(h_cam.shape[0]) for s in range(h_cam.shape[1]) if h_cam[m, s] >= 0]
    cov = np.zeros(nq, dtype=np.float32)
    for j in range(nq):
        nv = int(q_valid[j])
        hit = 0
        for r in range(nv):
            if tok_cam[j, r] < 0:
                continue
            X = token_point(*_cam(cams, tok_cam[j, r]), intr, *tok_uvd[j, r])
            if any(in_slab(X, Rc[0], Rc[1], intr, rect) for Rc, rect in slabs):
                hit += 1
        cov[j] = F(hit) / F(nv) if nv > 0 else F(0)
    return cov
