"""GPU test of the bounded-wait failure path (no fault, no hang).

Every pipeline wait in the library gives up after a bounded number of SM
clocks, records BSA_DEV_WAIT_TIMEOUT in the caller's error word and lets the
kernel return.  The self-test entry waits on an mbarrier that nothing ever
arrives on, with a limit of about a millisecond, and the host must then read
the timeout and find the CUDA context still usable.
"""
import pytest
import torch

import block_sparse_kv_bsa_b200 as bsa
import synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_wait_that_never_completes_times_out_and_reports():
    assert bsa.bsa_check_device_error(DEV) == (0, 0)
    status, code = bsa.bsa_selftest_bounded_wait(DEV, limit_cycles=2_000_000)
    assert status == 7 and code == 5            # BSA_ERR_TIMEOUT, BSA_DEV_WAIT_TIMEOUT
    assert bsa.bsa_check_device_error(DEV) == (0, 0)   # read clears the word
    # The context is still usable: a library call and a torch op both run.
    x = synth.random_bf16((1, 2 * 8 * 16, 2, 64), seed=3, device=DEV)
    blk = bsa.bsa_tokens_to_blocks(x, 2, 8, 16)
    back = bsa.bsa_blocks_to_tokens(blk, 2, 8, 16)
    torch.cuda.synchronize()
    assert torch.equal(back, x)


def test_selftest_rejects_bad_limits():
    with pytest.raises(bsa.BsaError):
        bsa.bsa_selftest_bounded_wait(DEV, limit_cycles=0)
