"""The routing entry point for callers that cannot allocate device memory.

sba_pool_select_noalloc works from a fixed scratch array inside the library instead
of a caller-provided workspace (for callers that may not call cudaMalloc, e.g. code
running inside a framework that owns all device memory and hands out no workspace).
These tests call it through the C ABI and require its routing to equal that of
sba_pool_select with a caller-allocated workspace, exactly (routing is compared bit
for bit everywhere in this suite), and the fp64 oracle's, with score ties counted and
reported.  Problems run back to back with different shapes, so every call after the
first finds the array full of another problem's values: what a call leaves there
must not leak into the next result.  The cases cover a sparse and a dense (s = 0)
routing and a problem whose workspace fills the scratch almost exactly.  The file is
named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import compare_routing, to_device
from workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _route_both(lib, sba, oracle_mod, w):
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
    # and against the oracle directly
    io, co, _, _, S = oracle_mod.select(w.q, w.k, w.valid_len, w.sparsity, kmax=kmax, return_intermediates=True)
    bad, excused = compare_routing(ib, cb, io, co, S)
    assert not bad, bad[:3]
    print(f"no-alloc routing {w.name}: {cb.size} rows, {len(excused)} excused ties")
    return cb


def _at_limit_problem(lib, sba):
    """The most heads of a 32768-token D = 128 problem whose workspace fits the scratch."""
    cap = lib.sba_noalloc_scratch_bytes()
    H = 1
    while sba.workspace_size(1, H + 1, 32768, 128) <= cap:
        H += 1
    assert sba.workspace_size(1, H, 32768, 128) <= cap < sba.workspace_size(1, H + 1, 32768, 128)
    return make_custom(1, H, 128, (8, 64, 64), 0.75, seed=17)


def test_noalloc_routing_matches_workspace_routing_and_oracle(oracle_mod):
    import video_dit_block_b200 as sba
    lib = sba.lib()
    cap = lib.sba_noalloc_scratch_bytes()
    ragged = make_custom(2, 3, 128, (3, 10, 50), 0.75, drop_rate=0.15, seed=101)
    dense = make_custom(1, 2, 64, (2, 16, 24), 0.0, seed=103)        # s = 0: no scores
    tiny = make_workload("tiny")
    full = _at_limit_problem(lib, sba)
    # at the limit: one more head would not fit the scratch
    assert sba.workspace_size(full.B, full.H, full.Npad, full.D) <= cap < \
        sba.workspace_size(full.B, full.H + 1, full.Npad, full.D)
    counts = [_route_both(lib, sba, oracle_mod, w) for w in (ragged, dense, tiny, full, ragged)]
    assert all(c.sum() > 0 for c in counts)
    # the dense routing keeps every block of its sample
    nB = (int(dense.valid_len[0]) + 63) // 64
    assert np.all(counts[1][0, :, :nB] == nB)
    # the same problem routed again after three others gives the same counts
    np.testing.assert_array_equal(counts[0], counts[4])


def test_noalloc_rejects_problems_beyond_its_scratch():
    import video_dit_block_b200 as sba
    lib = sba.lib()
    cap = lib.sba_noalloc_scratch_bytes()
    # 720p-sized routing of 40 heads needs far more than the fixed scratch
    assert sba.workspace_size(1, 40, 75648, 128) > cap
    A = ctypes.c_void_p(0x10000)   # never dereferenced: every check runs on the host first
    st = lib.sba_pool_select_noalloc(A, A, 1, 40, 75648, 128, None, 64, 0.8, 237, A, A, _stream())
    assert st == 7   # SBA_ERR_SCRATCH_TOO_SMALL
    assert b"scratch" in lib.sba_strerror(7)


def test_noalloc_reports_bad_arguments_before_the_size():
    """A bad argument is SBA_ERR_INVALID_ARG (or ALIGNMENT) on a small problem and on one
    too large for the scratch alike."""
    import video_dit_block_b200 as sba
    lib = sba.lib()
    A = ctypes.c_void_p(0x10000)
    MIS = ctypes.c_void_p(0x10008)
    for H, Npad, kmax in ((2, 1024, 8), (40, 75648, 237)):
        f = lambda q=A, s=0.8, km=kmax: lib.sba_pool_select_noalloc(q, A, 1, H, Npad, 128, None, 64, s, km, A, A,
                                                                    _stream())
        assert f(s=1.0) == 1 and f(s=-0.1) == 1
        assert f(q=None) == 1
        assert f(km=1) == 1
        assert f(q=MIS) == 3
