"""GPU test of bsa_route_noalloc, the routing entry point that allocates nothing.

Some callers cannot hand the router a device workspace: code that runs inside
another runtime's plugin or enqueue hook, where the host framework owns all
device memory and refuses new allocations, or a latency-bound loop that cannot
pay for cudaMalloc's implicit device synchronisation.  For them the library
keeps the router's scratch in a fixed array inside its own device image.

This file is collected last on purpose.  It checks, through the C ABI, that
the no-allocation entry point returns exactly the routes of the ordinary
bsa_route (same kernels, same fp32 arithmetic, so the same indices and
counts) on two calls in a row, then on a second, differently sized problem
(the shared array keeps the previous call's contents, which must not leak
into the next result), and that a problem too large for the array is
refused before anything runs.
"""
import ctypes

import pytest
import torch

import block_sparse_kv_bsa_b200 as bsa
import synth
from tests import _harness as hx

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _noalloc(step, idx, cnt, max_sel):
    cs = step.cache.c_struct()
    w = step.w
    return bsa.lib().bsa_route_noalloc(
        ctypes.c_void_p(step.q_blk.data_ptr()), ctypes.byref(cs),
        ctypes.c_void_p(step.q_valid.data_ptr()), step.n_hist, step.own_first, step.n_own,
        None if step.g is None else ctypes.c_void_p(step.g.data_ptr()),
        w.lam, w.g_ref, w.sm_scale, step.top_k,
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(cnt.data_ptr()), max_sel,
        ctypes.c_void_p(bsa.error_word(DEV).data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _same_as_workspace_route(step, calls):
    ref_idx, ref_cnt = hx.route(step)
    max_sel = ref_idx.shape[-1]
    for _ in range(calls):
        idx = torch.full_like(ref_idx, -7)
        cnt = torch.full_like(ref_cnt, -7)
        assert _noalloc(step, idx, cnt, max_sel) == 0
        torch.cuda.synchronize()
        assert bsa.bsa_check_device_error(DEV) == (0, 0)
        assert torch.equal(cnt, ref_cnt)
        assert torch.equal(idx, ref_idx)


def test_noalloc_route_matches_workspace_route():
    # Velox-like budget with the geometric prior: two calls in a row.
    _same_as_workspace_route(hx.build_step(synth.CONFIGS[3], DEV), calls=2)
    # A second, smaller problem right after: stale scratch must not matter.
    _same_as_workspace_route(hx.build_step(synth.CONFIGS[2], DEV), calls=1)


def test_noalloc_route_from_pooled_keys_and_head_dim_64():
    # Scores from the pooled-key cache (the product kernels write the scores
    # into the shared array with their own layout), then the D = 64 kernels.
    _same_as_workspace_route(hx.build_step(synth.CONFIGS[3], DEV, pooled_keys=True), calls=2)
    _same_as_workspace_route(hx.build_step(synth.CONFIGS[4], DEV, chunk=12, pooled_keys=True),
                             calls=1)
    _same_as_workspace_route(hx.build_step(synth.CONFIGS[1], DEV), calls=2)
    _same_as_workspace_route(hx.build_step(synth.CONFIGS[1], DEV, pooled_keys=True), calls=1)


def test_noalloc_route_rejects_problems_larger_than_its_scratch():
    step = hx.build_step(synth.CONFIGS[1], DEV)
    cs = step.cache.c_struct()
    # Claim a history so long that its scores alone exceed the fixed array;
    # the call must refuse it up front (nothing is launched).
    n_hist = 2_000_000
    cs.n_blocks = cs.max_blocks = n_hist + step.n_own
    need = bsa.bsa_route_workspace_size(step.w.B, step.w.Hh, step.w.D, step.n_own, n_hist)
    assert need > (16 << 20)
    idx = torch.empty((1,), dtype=torch.int32, device=DEV)
    st = bsa.lib().bsa_route_noalloc(
        ctypes.c_void_p(step.q_blk.data_ptr()), ctypes.byref(cs), None, n_hist, n_hist,
        step.n_own, None, 2.0, 0.2, step.w.sm_scale, 3, ctypes.c_void_p(idx.data_ptr()),
        ctypes.c_void_p(idx.data_ptr()), 5, None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 3  # BSA_ERR_CAPACITY
