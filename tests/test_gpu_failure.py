"""Failure detection on the GPU without a fault: the bounded waits.

Every pipeline of the library waits on mbarriers through one bounded wait
that gives up after a time limit, records QSA_DEV_TIMEOUT (status bit 4) and
lets the kernel release its tensor memory and return.  The self-test entry
point runs that wait on an mbarrier nothing arrives on, with a short limit:
the call must come back, the status word must report the timeout once, and
the library must keep working afterwards (its tensor-core kernels can still
allocate TMEM)."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads
from qsa_testlib import np32

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def qsa():
    import block_sparse_attention_11_b200 as m
    return m


@pytest.mark.parametrize("limit_ns", [50_000, 2_000_000, 100_000_000])
def test_bounded_wait_gives_up_reports_and_recovers(qsa, limit_ns):
    assert qsa.qsa_check_status() == 0      # clean before
    res = torch.full((1,), 7, dtype=torch.int32, device=DEV)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    qsa.qsa_selftest_wait_timeout(limit_ns, res)
    with pytest.raises(qsa.QSAError) as ei:
        qsa.qsa_check_status()
    elapsed = time.perf_counter() - t0
    assert ei.value.status == qsa.QSA_ERR_DEVICE
    assert "0x4" in str(ei.value)           # QSA_DEV_TIMEOUT and nothing else
    assert int(res.item()) == 0             # the wait gave up
    assert elapsed >= limit_ns * 1e-9       # it waited at least its limit
    assert elapsed < 10.0                   # and did not hang
    assert qsa.qsa_check_status() == 0      # read-and-clear: clean again


def test_library_works_after_a_timeout(qsa):
    """After the timed-out self-test (which freed its TMEM), the tcgen05
    prefill indexer and the attention still run and match the oracle."""
    res = torch.zeros(1, dtype=torch.int32, device=DEV)
    for _ in range(3):
        qsa.qsa_selftest_wait_timeout(10_000, res)
    with pytest.raises(qsa.QSAError):
        qsa.qsa_check_status()
    w = workloads.Workload("after_timeout", "prefill", 1, 3001, 64, 16, 2, 128, "bf16", 77)
    x = workloads.make_prefill(w, device=DEV)
    T = w.T
    k_pool = torch.zeros(1, T // 4, 128, dtype=torch.bfloat16, device=DEV)
    qsa.qsa_pool_keys_prefill(x["k_idx"], k_pool)
    sel = torch.empty(1, T, w.top_k, dtype=torch.int32, device=DEV)
    nsel = torch.empty(1, T, dtype=torch.int32, device=DEV)
    qsa.qsa_index_topk_prefill(x["q_idx"], k_pool, sel, nsel, top_k=w.top_k)
    assert qsa.qsa_check_status() == 0
    rows = np.array([0, 5, 1000, 2047, T - 1])
    ref = oracle.prefill_rows(rows, q_idx=np32(x["q_idx"][0]), k_pool=oracle.pool_keys(np32(x["k_idx"][0])),
                              top_k=w.top_k)
    g = sel[0].cpu().numpy()[rows]
    gap = (ref["kth"] - ref["next"]) / np.maximum(np.abs(ref["kth"]), 1e-30)
    assert np.all(np.all(g == ref["sel"], axis=1) | (gap < 1e-4))
