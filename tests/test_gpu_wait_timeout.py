"""Failure detection on the device, without a fault: a bounded wait that nobody
completes expires after its budget, records DSA_ERR_TIMEOUT in the sticky
device word and returns normally; the context stays usable afterwards.

The wait runs through the same routine every kernel of the library uses for
its barriers (TMA loads, tensor-core commits, peer CTAs), with the budget as a
kernel argument so that it can be made short here (1e5 SM cycles, tens of
microseconds) instead of the kernels' second."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

BUDGET = 100_000        # SM clock cycles


@pytest.fixture(scope="module")
def dsa():
    import top_kv_selection_b200 as m
    return m


def _timed(fn):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fn()
    e1.record()
    e1.synchronize()
    return e0.elapsed_time(e1)          # ms


def test_expired_wait_records_timeout(dsa):
    torch.cuda.synchronize()
    dsa.dsa_get_device_error()                       # start from a clear word
    ms = _timed(lambda: dsa.dsa_wait_selftest(BUDGET, complete=False))
    assert dsa.dsa_get_device_error() == dsa.DSA_ERR_TIMEOUT
    # it waited for its budget (1e5 cycles is 50 us at 2 GHz) and no longer
    # than a generous bound: the wait is bounded, not a hang
    assert 0.02 < ms < 50.0
    # the read cleared the sticky word
    assert dsa.dsa_get_device_error() == dsa.DSA_OK


def test_completed_wait_records_nothing(dsa):
    dsa.dsa_get_device_error()
    ms = _timed(lambda: dsa.dsa_wait_selftest(BUDGET, complete=True))
    assert dsa.dsa_get_device_error() == dsa.DSA_OK
    assert ms < 50.0


def test_context_usable_after_expired_wait(dsa):
    dsa.dsa_wait_selftest(BUDGET, complete=False)
    assert dsa.dsa_get_device_error() == dsa.DSA_ERR_TIMEOUT
    # the next kernels run and give the oracle's answer
    B, T, k = 2, 5003, 2048
    sc = workloads.score_rows(B, T, seed=17).numpy().reshape(B, 1, T)
    idx = torch.empty(B, 1, k, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(dsa.dsa_topk_select_workspace_size(B, 1, T, k), 1), dtype=torch.uint8,
                     device="cuda")
    dsa.dsa_topk_select(torch.from_numpy(np.ascontiguousarray(sc)).cuda(), T - 1, k, idx, ws)
    assert np.array_equal(idx.cpu().numpy(), oracle.topk_select(sc, T - 1, k))
    assert dsa.dsa_get_device_error() == dsa.DSA_OK
