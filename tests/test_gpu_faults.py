"""Failure detection on the GPU without a GPU fault: a wait that runs out and a routing
entry outside the sample both come back as a device status, and the context stays
usable for the next call."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, output_errors, to_device
from workloads import make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def test_wait_limit_expiry_reports_timeout(sba, oracle_mod):
    w = make_workload("tiny")
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    assert sba.device_status() == 0
    sba.set_wait_limit(1)            # every wait that is not already satisfied gives up
    try:
        sba.attention(q, k, v, idx, cnt, vl)
        assert sba.device_status() == 5   # SBA_ERR_TIMEOUT
    finally:
        sba.set_wait_limit(0)        # default limit
    # the context is intact: the same call now succeeds and is correct
    o, _ = sba.attention(q, k, v, idx, cnt, vl)
    assert sba.device_status() == 0
    o_ref, _ = oracle_mod.attention(w.q, w.k, w.v, idx.cpu().numpy(), cnt.cpu().numpy(), w.valid_len)
    mx, mean = output_errors(o.float().cpu().numpy(), o_ref)
    assert mx <= MAX_ABS and mean <= MEAN_ABS


def test_routing_wait_limit_expiry_reports_timeout(sba):
    """A wait of the fused screen that runs out: status 5, and the next routing call on
    the same context gives the same lists as before."""
    w = make_workload("tiny")
    q, k, v, vl = to_device(w, DEV)
    idx0, cnt0 = sba.pool_select(q, k, vl, w.sparsity)
    assert sba.device_status() == 0
    sba.set_wait_limit(1)
    try:
        sba.pool_select(q, k, vl, w.sparsity)
        assert sba.device_status() == 5
    finally:
        sba.set_wait_limit(0)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    assert sba.device_status() == 0
    assert torch.equal(cnt, cnt0)
    for r in np.ndindex(tuple(cnt.shape)):
        c = int(cnt[r])
        assert torch.equal(idx[r][:c], idx0[r][:c])


def test_bad_routing_entry_is_flagged_and_skipped(sba):
    w = make_workload("tiny")
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    bad = idx.clone()
    bad[0, 0, 3, 0] = 10_000           # outside [0, nB)
    bad[0, 1, 5, 1] = -2
    sba.attention(q, k, v, bad, cnt, vl)
    assert sba.device_status() == 6    # SBA_ERR_DEVICE_FLAG
    cnt_bad = cnt.clone()
    cnt_bad[0, 0, 0] = 1_000_000       # more than kmax entries
    sba.attention(q, k, v, idx, cnt_bad, vl)
    assert sba.device_status() == 6
    sba.attention(q, k, v, idx, cnt, vl)
    assert sba.device_status() == 0
