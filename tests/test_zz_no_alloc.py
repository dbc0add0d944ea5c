"""The routing entry point for callers that cannot allocate device memory.

sba_pool_select_noalloc works from a fixed scratch array inside the library instead
of a caller-provided workspace (for callers that may not call cudaMalloc, e.g. code
running inside a framework that owns all device memory and hands out no workspace).
These tests call it through the C ABI and require its routing to equal that of
sba_pool_select with a caller-allocated workspace, exactly (routing is compared bit
for bit everywhere in this suite), on two calls in a row with different problems,
so the second call also shows that what the first left in the array does not leak
into the result.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import to_device
from workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _route_both(lib, sba, w):
    q, k, _, vl = to_device(w, DEV)
    B, H, Npad, D = q.shape
    nB = Npad // 64
    kmax = sba.kmax_for(Npad, w.sparsity)
    # existing entry point, caller-allocated workspace
    ws = torch.empty(sba.workspace_size(B, H, Npad, D), dtype=torch.uint8, device=DEV)
    idx_a = torch.full((B, H, nB, kmax), -7, dtype=torch.int32, device=DEV)
    cnt_a = torch.full((B, H, nB), -7, dtype=torch.int32, device=DEV)
    st = lib.sba_pool_select(_p(q), _p(k), B, H, Npad, D, _p(vl), 64, w.sparsity, kmax, _p(idx_a),
                             _p(cnt_a), _p(ws), ws.numel(), _stream())
    assert st == 0
    # no-allocation entry point
    idx_b = torch.full((B, H, nB, kmax), -9, dtype=torch.int32, device=DEV)
    cnt_b = torch.full((B, H, nB), -9, dtype=torch.int32, device=DEV)
    st = lib.sba_pool_select_noalloc(_p(q), _p(k), B, H, Npad, D, _p(vl), 64, w.sparsity, kmax,
                                     _p(idx_b), _p(cnt_b), _stream())
    assert st == 0
    assert lib.sba_get_device_status(_stream()) == 0
    ca, cb = cnt_a.cpu().numpy(), cnt_b.cpu().numpy()
    ia, ib = idx_a.cpu().numpy(), idx_b.cpu().numpy()
    np.testing.assert_array_equal(ca, cb)
    for r in np.ndindex(ca.shape):
        c = int(ca[r])
        np.testing.assert_array_equal(ia[r][:c], ib[r][:c])
    return ca


def test_noalloc_routing_matches_workspace_routing_twice():
    import video_dit_block_b200 as sba
    lib = sba.lib()
    # two different problems back to back; the second sees the first's leftovers
    first = make_custom(2, 3, 128, (3, 10, 50), 0.75, drop_rate=0.15, seed=101)
    second = make_workload("tiny")
    assert sba.workspace_size(first.B, first.H, first.Npad, first.D) <= lib.sba_noalloc_scratch_bytes()
    c1 = _route_both(lib, sba, first)
    c2 = _route_both(lib, sba, second)
    assert c1.sum() > 0 and c2.sum() > 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    import video_dit_block_b200 as sba
    lib = sba.lib()
    cap = lib.sba_noalloc_scratch_bytes()
    # 720p-sized routing of 40 heads needs far more than the fixed scratch
    assert sba.workspace_size(1, 40, 75648, 128) > cap
    A = ctypes.c_void_p(0x10000)   # never dereferenced: the size check comes first
    st = lib.sba_pool_select_noalloc(A, A, 1, 40, 75648, 128, None, 64, 0.8, 237, A, A, _stream())
    assert st == 7   # SBA_ERR_SCRATCH_TOO_SMALL
    assert b"scratch" in lib.sba_strerror(7)
