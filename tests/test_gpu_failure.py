"""Failure handling on the GPU without a fault: the bounded device-side wait.

Every tcgen05 kernel waits on mbarriers with a time limit; on expiry it sets
LSA_ERR_TIMEOUT in the caller's error word and returns.  Here that path runs
on a barrier nothing arrives at (lsa_selftest_bounded_wait), with a 1 ms limit,
and the context must stay usable afterwards.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_cases import Z_TOL, gpu_full_scores, lsa_mod

pytestmark = pytest.mark.gpu

LSA_ERR_TIMEOUT = 4


@pytest.fixture(scope="module")
def lsa():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return lsa_mod()


def test_bounded_wait_expires_and_reports_timeout(lsa):
    limit = 1_000_000   # 1 ms
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.full((3,), -1, dtype=torch.int64, device="cuda")
    lsa.selftest_bounded_wait(limit, err, waited)
    torch.cuda.synchronize()   # the kernel returned: no hang, no fault
    w = waited.cpu().tolist()
    assert int(err.item()) == LSA_ERR_TIMEOUT
    assert limit <= w[0] < 100 * limit          # gave up after its limit, not much later
    assert w[1] < 3 * limit                      # the second waiter left on the abort flag, not its 4 ms limit
    assert w[2] == 0                             # and did not report success


def test_error_word_keeps_first_error(lsa):
    err = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    waited = torch.zeros(3, dtype=torch.int64, device="cuda")
    lsa.selftest_bounded_wait(10_000, err, waited)
    torch.cuda.synchronize()
    assert int(err.item()) == 7


def test_context_usable_after_timeout(lsa):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(3, dtype=torch.int64, device="cuda")
    lsa.selftest_bounded_wait(100_000, err, waited)
    torch.cuda.synchronize()
    assert int(err.item()) == LSA_ERR_TIMEOUT
    # a real kernel right after, on the same context, still matches the oracle
    wl = synth.small_ragged(key_dtype="e4m3")
    dev = synth.to_torch(wl, pin_cold=False)
    z, _ = gpu_full_scores(wl, dev, lsa, tc=True)   # asserts the scan's own error word is 0
    z_ref, _ = oracle.index_score(wl.q, wl.q_dtype, wl.w, wl.keys, wl.key_dtype, wl.k_scale, wl.seq_off,
                                  wl.H, wl.d)
    assert np.abs(z - z_ref).max() <= Z_TOL
