"""GPU parity: the geometric overlap prior g and the coverage score
("Velox: Spatial Memory Makes World Models Efficient", Methodology Step 3)
against the oracle, on synthetic slabs.

Both sides take every inside / outside decision in float32 with one rounding
per operation in the same order, so the grid counts, the IoUs and the
coverage fractions must agree exactly.
"""
import numpy as np
import pytest
import torch

import block_sparse_kv_bsa_b200 as bsa
from oracle import geometry as geo
from synth.geometry import slab_scene

pytestmark = pytest.mark.gpu
DEV = "cuda"


def to_dev(scenes, S=2):
    """Stack scenes (one per batch element) into device tensors."""
    def st(name, dtype):
        return torch.from_numpy(np.stack([getattr(sc, name) for sc in scenes])).to(DEV, dtype)
    t = {k: st(k, torch.float32) for k in ("cams", "h_rect", "q_rect", "tok_uvd")}
    t.update({k: st(k, torch.int32) for k in ("h_cam", "q_cam", "tok_cam")})
    t["h_cam"] = t["h_cam"][:, :, :S].contiguous()
    t["q_cam"] = t["q_cam"][:, :, :S].contiguous()
    t["h_rect"] = t["h_rect"][:, :, :S].contiguous()
    t["q_rect"] = t["q_rect"][:, :, :S].contiguous()
    return t


def run(t, intr, n, q_valid=None):
    g, cov = bsa.bsa_geometry_prior(t["cams"], intr, t["h_cam"], t["h_rect"], t["q_cam"],
                                    t["q_rect"], t["tok_cam"], t["tok_uvd"], q_valid=q_valid,
                                    grid_n=n)
    bsa.raise_on_device_error(DEV)
    return g.cpu().numpy(), cov.cpu().numpy()


@pytest.mark.parametrize("n,S", [(8, 2), (5, 2), (16, 1), (1, 2)])
def test_prior_and_coverage_match_oracle(n, S):
    sc = slab_scene((4, 30, 52), 3, 49, seed=4700 + n)
    t = to_dev([sc], S)
    qv = np.full(49, 128, np.int32)
    qv[-1] = 96                                       # the chunk's tail block
    g, cov = run(t, sc.intr, n, torch.from_numpy(qv).to(DEV))
    exp_g = geo.prior_g(sc.cams, sc.intr, sc.q_cam[:, :S], sc.q_rect[:, :S], sc.h_cam[:, :S],
                        sc.h_rect[:, :S], n)
    assert np.array_equal(g[0], exp_g)
    exp_c = geo.coverage(sc.cams, sc.intr, sc.tok_cam, sc.tok_uvd, qv, sc.h_cam[:, :S],
                         sc.h_rect[:, :S])
    assert np.array_equal(cov[0], exp_c)
    assert (g > 0).mean() > 0.05 and 0 < cov.min()       # the case is not trivial


def test_batch_elements_are_independent():
    scs = [slab_scene((4, 16, 32), 2, 16, seed=s, tile=(8, 8)) for s in (11, 12)]
    t = to_dev(scs)
    g, cov = run(t, scs[0].intr, 8)
    for b, sc in enumerate(scs):
        assert np.array_equal(g[b], geo.prior_g(sc.cams, sc.intr, sc.q_cam, sc.q_rect, sc.h_cam,
                                                sc.h_rect, 8))
        assert np.array_equal(cov[b], geo.coverage(sc.cams, sc.intr, sc.tok_cam, sc.tok_uvd,
                                                   np.full(16, 128), sc.h_cam, sc.h_rect))


def test_full_size_sampled_rows():
    # The 48-chunk sweep workload at chunk 48: 49 query blocks against 2303
    # history blocks; the oracle checks three rows of g and one coverage.
    sc = slab_scene((4, 30, 52), 47, 49, seed=4800)
    t = to_dev([sc])
    g, cov = run(t, sc.intr, 8)
    for j in (0, 24, 48):
        exp = geo.prior_g(sc.cams, sc.intr, sc.q_cam[j:j + 1], sc.q_rect[j:j + 1], sc.h_cam,
                          sc.h_rect, 8)
        assert np.array_equal(g[0, j], exp[0])
    j = 17
    exp_c = geo.coverage(sc.cams, sc.intr, sc.tok_cam[j:j + 1], sc.tok_uvd[j:j + 1],
                         np.array([128]), sc.h_cam, sc.h_rect)
    assert cov[0, j] == exp_c[0]


def test_bad_camera_index_is_reported_and_absent():
    sc = slab_scene((4, 16, 32), 2, 16, seed=13, tile=(8, 8))
    t = to_dev([sc])
    t["h_cam"][0, 3, 0] = 10 ** 6
    g, cov = bsa.bsa_geometry_prior(t["cams"], sc.intr, t["h_cam"], t["h_rect"], t["q_cam"],
                                    t["q_rect"], t["tok_cam"], t["tok_uvd"], grid_n=8)
    status, code = bsa.bsa_check_device_error(DEV)
    assert status == 6 and code == 1
    h_cam = sc.h_cam.copy()
    h_cam[3, 0] = -1
    exp = geo.prior_g(sc.cams, sc.intr, sc.q_cam, sc.q_rect, h_cam, sc.h_rect, 8)
    assert np.array_equal(g[0].cpu().numpy(), exp)


def test_argument_checks():
    sc = slab_scene((4, 16, 32), 1, 16, seed=14, tile=(8, 8))
    t = to_dev([sc])
    with pytest.raises(bsa.BsaError):
        bsa.bsa_geometry_prior(t["cams"], sc.intr, t["h_cam"], t["h_rect"], t["q_cam"],
                               t["q_rect"], t["tok_cam"], t["tok_uvd"], grid_n=17)
    with pytest.raises(bsa.BsaError):
        bsa.bsa_geometry_prior(t["cams"], (0.0, 1.0, 0.0, 0.0), t["h_cam"], t["h_rect"],
                               t["q_cam"], t["q_rect"], t["tok_cam"], t["tok_uvd"])
    # Coverage alone, with no history slab at all: every block is uncovered.
    none = torch.full_like(t["h_cam"], -1)
    _, cov = bsa.bsa_geometry_prior(t["cams"], sc.intr, none, t["h_rect"], tok_cam=t["tok_cam"],
                                    tok_uvd=t["tok_uvd"], want_g=False)
    bsa.raise_on_device_error(DEV)
    assert torch.count_nonzero(cov).item() == 0
