"""Pins of the geometric-prior oracle ("Velox: Spatial Memory Makes World
Models Efficient", Methodology Step 3) against closed forms, exact special
cases and brute force on small inputs.  CPU only."""
import math

import numpy as np
import pytest

from oracle import geometry as geo

F = np.float32


def rot(yaw=0.0, pitch=0.0, roll=0.0):
    """World-from-camera rotation from three angles (radians), float32."""
    cy, sy = math.cos(yaw), math.sin(yaw)
    cp, sp = math.cos(pitch), math.sin(pitch)
    cr, sr = math.cos(roll), math.sin(roll)
    Ry = np.array([[cy, 0, sy], [0, 1, 0], [-sy, 0, cy]])
    Rx = np.array([[1, 0, 0], [0, cp, -sp], [0, sp, cp]])
    Rz = np.array([[cr, -sr, 0], [sr, cr, 0], [0, 0, 1]])
    return (Ry @ Rx @ Rz).astype(np.float32)


def box(centre, R, half):
    return (np.asarray(centre, np.float32), np.asarray(R, np.float32), np.asarray(half, np.float32))


def random_rot(rng):
    return rot(*rng.uniform(-math.pi, math.pi, size=3))


def test_slab_box_closed_form():
    # Rectangle symmetric about the principal point, depths [2, 4]: the
    # frustum segment's camera-aligned box is centred on the axis at depth 3,
    # with lateral half-extents set by the far plane (0.2 * 4) and depth
    # half-extent 1.
    intr = (10.0, 10.0, 5.0, 4.0)
    c, A, h = geo.slab_box(np.eye(3), np.zeros(3), intr, (3.0, 7.0, 2.0, 6.0, 2.0, 4.0))
    np.testing.assert_allclose(c, [0, 0, 3], atol=1e-6)
    np.testing.assert_allclose(h, [0.8, 0.8, 1.0], rtol=1e-6)
    assert np.array_equal(A, np.eye(3, dtype=np.float32))
    # Off-axis rectangle: x in tan space [0.1, 0.3] -> box x in [0.2, 1.2].
    c, A, h = geo.slab_box(np.eye(3), np.zeros(3), intr, (6.0, 8.0, 4.0, 4.0, 2.0, 4.0))
    np.testing.assert_allclose([c[0], h[0]], [0.7, 0.5], rtol=1e-6)
    # A moved and turned camera moves and turns the box rigidly.
    R = rot(0.3, -0.2, 0.1)
    t = np.array([1.0, -2.0, 0.5], np.float32)
    c2, A2, h2 = geo.slab_box(R, t, intr, (3.0, 7.0, 2.0, 6.0, 2.0, 4.0))
    np.testing.assert_allclose(c2, t + R @ np.array([0, 0, 3], np.float32), atol=1e-5)
    np.testing.assert_allclose(h2, [0.8, 0.8, 1.0], rtol=1e-6)
    assert np.array_equal(A2, R)


def test_iou_of_a_box_with_itself_is_one():
    rng = np.random.default_rng(1)
    for _ in range(20):
        b = box(rng.normal(size=3), random_rot(rng), rng.uniform(0.1, 2.0, size=3))
        assert geo.grid_count(b, b, 8) == 512
        assert geo.box_iou(b, b, 8) == F(1)


def test_iou_of_shifted_cubes_exact():
    # Unit cubes (half-extent 1) offset by 0.5 along x: 6 of the 8 grid
    # columns fall inside, intersection 6 of volume 8 each, IoU 6/10 -- the
    # analytic value.
    a = box([0, 0, 0], np.eye(3), [1, 1, 1])
    b = box([0.5, 0, 0], np.eye(3), [1, 1, 1])
    assert geo.grid_count(a, b, 8) == 6 * 64
    assert geo.box_iou(a, b, 8) == F(6) / F(10)
    assert geo.box_iou(b, a, 8) == F(6) / F(10)


def test_iou_is_a_fraction():
    # Random pairs, including a box just smaller than one that contains
    # every cell centre of the other: the estimate stays in [0, 1].
    rng = np.random.default_rng(5)
    a = box([0, 0, 0], np.eye(3), [1, 1, 1])
    b = box([0, 0, 0], np.eye(3), [0.9, 0.9, 0.9])       # holds all 8^3 centres
    assert geo.grid_count(a, b, 8) == 512
    # B inside A: the IoU is vol(B) / vol(A) = 0.729, exactly what the cap
    # on the intersection gives (the uncapped count would say 1/0.729).
    assert abs(float(geo.box_iou(a, b, 8)) - 0.729) < 1e-6
    for _ in range(200):
        p = box(rng.normal(scale=0.5, size=3), random_rot(rng), rng.uniform(0.2, 1.0, size=3))
        q = box(rng.normal(scale=0.5, size=3), random_rot(rng), rng.uniform(0.2, 1.0, size=3))
        assert 0 <= geo.box_iou(p, q, 8) <= 1


def test_grid_count_axis_aligned_is_separable():
    # With both boxes axis-aligned the 3-D count is the product of three 1-D
    # counts of grid points inside an interval (written here independently).
    rng = np.random.default_rng(2)
    n = 8
    s = [(2 * i + 1) / n - 1 for i in range(n)]
    for _ in range(50):
        ca, cb = rng.normal(size=3), rng.normal(size=3)
        e, f = rng.uniform(0.2, 1.5, size=3), rng.uniform(0.2, 1.5, size=3)
        a, b = box(ca, np.eye(3), e), box(cb, np.eye(3), f)
        exp = 1
        for k in range(3):
            exp *= sum(1 for si in s if abs(F(F(ca[k]) - F(cb[k])) + F(F(si) * F(e[k]))) <= F(f[k]))
        assert geo.grid_count(a, b, n) == exp


def test_grid_iou_converges_to_analytic_axis_aligned():
    # For axis-aligned boxes the IoU is a product of interval overlaps; the
    # grid estimate is within its discretisation error (one cell per axis).
    rng = np.random.default_rng(3)
    n = 32
    for _ in range(30):
        ca, cb = rng.normal(scale=0.5, size=3), rng.normal(scale=0.5, size=3)
        e, f = rng.uniform(0.3, 1.5, size=3), rng.uniform(0.3, 1.5, size=3)
        ov = [max(0.0, min(ca[k] + e[k], cb[k] + f[k]) - max(ca[k] - e[k], cb[k] - f[k])) for k in range(3)]
        inter = ov[0] * ov[1] * ov[2]
        va, vb = 8 * np.prod(e), 8 * np.prod(f)
        exact = inter / (va + vb - inter)
        got = float(geo.box_iou(box(ca, np.eye(3), e), box(cb, np.eye(3), f), n))
        assert abs(got - exact) <= 4.0 / n


def _sample_inside(bx, m):
    c, A, h = bx
    g = (np.arange(m) + 0.5) / m * 2 - 1
    pts = np.stack(np.meshgrid(g, g, g, indexing="ij"), -1).reshape(-1, 3) * h
    corners = np.array([[sx, sy, sz] for sx in (-1, 1) for sy in (-1, 1) for sz in (-1, 1)]) * h
    return np.concatenate([pts, corners]) @ A.T.astype(np.float64) + c


def _inside(bx, pts):
    c, A, h = bx
    q = (pts - c) @ A.astype(np.float64)
    return np.all(np.abs(q) <= h * (1 + 1e-9), axis=1)


def test_sat_never_separates_intersecting_boxes():
    # Brute force: whenever a dense sample of one box has a point inside the
    # other, the boxes intersect and the test must not separate them; and a
    # separated pair shares no sampled point.  The sample includes pairs that
    # only an edge-edge axis separates.
    rng = np.random.default_rng(4)
    edge_only = 0
    for _ in range(400):
        a = box(rng.normal(scale=0.3, size=3), random_rot(rng), rng.uniform(0.2, 1.0, size=3))
        b = box(rng.normal(scale=1.2, size=3), random_rot(rng), rng.uniform(0.2, 1.0, size=3))
        sep = geo.sat_separated(a, b)
        touch = _inside(b, _sample_inside(a, 12)).any() or _inside(a, _sample_inside(b, 12)).any()
        if touch:
            assert not sep
        if sep:
            assert not touch
            assert geo.grid_count(a, b, 8) == 0
            # Face axes alone would not have separated it?
            ca, A, e = a
            cb, B, f = b
            t = A.T @ (cb - ca)
            M = A.T @ B
            face = any(abs(t[i]) > e[i] + np.abs(M[i]) @ f for i in range(3)) or \
                any(abs(t @ M[:, j]) > np.abs(M[:, j]) @ e + f[j] for j in range(3))
            edge_only += not face
    assert edge_only > 0


def test_prior_g_definition():
    intr = (20.0, 20.0, 13.0, 10.0)
    cams = np.zeros((2, 12), np.float32)
    cams[0, :9] = np.eye(3).ravel()
    cams[1, :9] = rot(0.05, 0.0, 0.0).ravel()
    cams[1, 9:] = [0.2, 0.0, 0.1]
    rect = np.array([0.0, 13.0, 0.0, 10.0, 3.0, 3.5], np.float32)
    far = np.array([0.0, 13.0, 0.0, 10.0, 30.0, 31.0], np.float32)
    q_cam = np.array([[0, -1], [-1, -1]], np.int32)
    q_rect = np.stack([np.stack([rect, rect]), np.stack([rect, rect])])
    h_cam = np.array([[0, -1], [1, 1], [-1, -1]], np.int32)
    h_rect = np.stack([np.stack([rect, rect]), np.stack([far, rect]), np.stack([rect, rect])])
    g = geo.prior_g(cams, intr, q_cam, q_rect, h_cam, h_rect, 8)
    assert g[0, 0] == F(1)                         # the same slab
    a = geo.slab_box(np.eye(3), np.zeros(3), intr, rect)
    b = geo.slab_box(cams[1, :9].reshape(3, 3), cams[1, 9:], intr, rect)
    assert g[0, 1] == geo.box_iou(a, b, 8) > 0     # best of its two slabs
    assert g[0, 2] == 0 and np.all(g[1] == 0)      # no valid slab


def test_coverage_definition():
    intr = (20.0, 20.0, 13.0, 10.0)
    cams = np.zeros((2, 12), np.float32)
    cams[0, :9] = np.eye(3).ravel()
    R1 = rot(0.1, 0.05, 0.0)
    cams[1, :9] = R1.ravel()
    cams[1, 9:] = [0.4, -0.1, -0.3]
    h_cam = np.array([[0]], np.int32)
    h_rect = np.array([[[4.0, 9.0, 3.0, 7.0, 2.0, 3.0]]], np.float32)
    # Tokens of camera 0: inside, depth too small, outside the rectangle,
    # no depth; then a token of camera 1 that sees a point inside the slab.
    X = geo.token_point(np.eye(3), np.zeros(3), intr, 6.5, 5.0, 2.5)
    Xc1 = R1.T.astype(np.float64) @ (X.astype(np.float64) - cams[1, 9:])
    u1 = 20.0 * Xc1[0] / Xc1[2] + 13.0
    v1 = 20.0 * Xc1[1] / Xc1[2] + 10.0
    tok_cam = np.array([[0, 0, 0, -1, 1]], np.int32)
    tok_uvd = np.array([[[6.5, 5.0, 2.5], [6.5, 5.0, 1.5], [11.0, 5.0, 2.5], [6.5, 5.0, 2.5],
                         [u1, v1, Xc1[2]]]], np.float32)
    cov = geo.coverage(cams, intr, tok_cam, tok_uvd, np.array([5]), h_cam, h_rect)
    assert cov[0] == F(2) / F(5)
    cov4 = geo.coverage(cams, intr, tok_cam, tok_uvd, np.array([4]), h_cam, h_rect)
    assert cov4[0] == F(1) / F(4)                  # only the first 4 tokens count
    none = geo.coverage(cams, intr, tok_cam, tok_uvd, np.array([5]), np.array([[-1]], np.int32), h_rect)
    assert none[0] == 0
