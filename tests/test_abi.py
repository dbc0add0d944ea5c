"""C-ABI checks that need no GPU: the library loads, exports every function declared
in include/sba.h, and rejects bad arguments on the host before touching device memory."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sba.h")


@pytest.fixture(scope="module")
def lib():
    from video_dit_block_b200 import build
    build.build()
    import video_dit_block_b200 as sba
    return sba.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sba_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("sba_pool_select", "sba_attention", "sba_dense_attention", "sba_keep_count",
              "sba_get_device_status", "sba_strerror"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


@pytest.mark.parametrize("n", [1, 2, 3, 7, 10, 16, 100, 512, 841, 1182, 4096])
@pytest.mark.parametrize("s", [0.0, 0.1, 0.3, 0.5, 0.7, 0.75, 0.8, 0.9, 0.95, 0.999])
def test_keep_count_matches_oracle(lib, oracle_mod, n, s):
    assert lib.sba_keep_count(n, s) == oracle_mod.keep_count(n, s)


def test_strerror(lib):
    for code in range(7):
        assert lib.sba_strerror(code)
    assert lib.sba_strerror(99) == b"unknown status"


def test_workspace_size(lib):
    assert lib.sba_pool_select_workspace_size(1, 24, 32768, 128, 64) > 0
    assert lib.sba_pool_select_workspace_size(1, 24, 32768, 96, 64) == 0
    assert lib.sba_pool_select_workspace_size(1, 24, 32760, 128, 64) == 0


# Fake device pointers: every call below must fail validation before any CUDA call.
A = ctypes.c_void_p(0x10000)       # 16-byte aligned
MIS = ctypes.c_void_p(0x10008)     # 8-byte aligned only
NULL = None
S = None                           # stream


def pool_select(lib, q=A, k=A, B=1, H=2, Npad=1024, D=64, vl=NULL, block=64, s=0.5, kmax=8,
                idx=A, cnt=A, ws=A, wsb=1 << 30):
    return lib.sba_pool_select(q, k, B, H, Npad, D, vl, block, s, kmax, idx, cnt, ws, wsb, S)


def attention(lib, q=A, k=A, v=A, o=A, lse=A, B=1, H=2, Npad=1024, D=64, vl=NULL, block=64,
              idx=A, cnt=A, kmax=8, scale=0.0):
    return lib.sba_attention(q, k, v, o, lse, B, H, Npad, D, vl, block, idx, cnt, kmax, scale, S)


@pytest.mark.parametrize("kwargs,code", [
    (dict(q=NULL), 1), (dict(k=NULL), 1), (dict(idx=NULL), 1), (dict(cnt=NULL), 1), (dict(ws=NULL), 1),
    (dict(B=0), 1), (dict(H=-1), 1), (dict(Npad=1000), 1), (dict(D=96), 2), (dict(block=32), 2),
    (dict(Npad=262144 + 64), 2), (dict(s=1.0), 1), (dict(s=-0.1), 1), (dict(s=float("nan")), 1),
    (dict(kmax=7), 1), (dict(wsb=16), 1), (dict(q=MIS), 3), (dict(vl=MIS), 3), (dict(ws=MIS), 3),
])
def test_pool_select_rejects(lib, kwargs, code):
    assert pool_select(lib, **kwargs) == code


@pytest.mark.parametrize("kwargs,code", [
    (dict(q=NULL), 1), (dict(v=NULL), 1), (dict(o=NULL), 1), (dict(idx=NULL), 1), (dict(cnt=NULL), 1),
    (dict(kmax=0), 1), (dict(D=32), 2), (dict(block=128), 2), (dict(Npad=100), 1),
    (dict(scale=float("inf")), 1), (dict(scale=float("nan")), 1), (dict(o=MIS), 3),
    (dict(lse=ctypes.c_void_p(0x10002)), 3), (dict(idx=ctypes.c_void_p(0x10002)), 3),
])
def test_attention_rejects(lib, kwargs, code):
    assert attention(lib, **kwargs) == code


def test_dense_attention_rejects(lib):
    assert lib.sba_dense_attention(A, A, NULL, A, A, 1, 2, 1024, 64, NULL, 0.0, S) == 1
    assert lib.sba_dense_attention(A, A, A, A, A, 1, 2, 1024, 80, NULL, 0.0, S) == 2
    assert lib.sba_dense_attention(MIS, A, A, A, A, 1, 2, 1024, 64, NULL, 0.0, S) == 3


def test_pairing_rejects(lib):
    assert lib.sba_pair_workspace_size(1, 2, 1024, 64) > 0
    assert lib.sba_pair_query_blocks(A, A, 1, 2, 1024, 8, NULL, 64, NULL, A, 1 << 30, S) == 1
    assert lib.sba_pair_query_blocks(A, A, 1, 2, 1024, 8, NULL, 64, A, A, 16, S) == 1
    assert lib.sba_pair_query_blocks(A, A, 1, 2, 1000, 8, NULL, 64, A, A, 1 << 30, S) == 1
    assert lib.sba_pair_query_blocks(A, A, 1, 2, 1024, 8, NULL, 64, A, MIS, 1 << 30, S) == 3
    # more (b, h) rows than one grid dimension holds: refused before any launch
    assert lib.sba_pair_query_blocks(A, A, 65535, 65535, 64, 8, NULL, 64, A, A, 1 << 62, S) == 2
    assert lib.sba_attention_paired(A, A, A, A, A, 1, 2, 1024, 64, NULL, 64, A, A, 8, NULL, 0.0, S) == 1
    assert lib.sba_attention_paired(A, A, A, A, A, 1, 2, 1024, 64, NULL, 64, A, A, 8,
                                    ctypes.c_void_p(0x10002), 0.0, S) == 3


def test_block_means_rejects(lib):
    assert lib.sba_block_means(NULL, 1, 2, 1024, 64, NULL, 64, A, S) == 1
    assert lib.sba_block_means(A, 1, 2, 1024, 64, NULL, 64, MIS, S) == 3
    assert lib.sba_block_means(A, 1, 2, 1024, 48, NULL, 64, A, S) == 2


def test_binding_refuses_cpu_tensors():
    import torch

    import video_dit_block_b200 as sba
    x = torch.zeros((1, 1, 64, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        sba.dense_attention(x, x, x)
    with pytest.raises(ValueError):
        sba.pool_select(x, x, None, 0.5)


def pool_select_lse(lib, q=A, k=A, B=1, H=2, Npad=1024, D=64, vl=NULL, block=64, nsub=4, s=0.5, budget=8,
                    kmax=8, idx=A, cnt=A, ws=A, wsb=1 << 30):
    return lib.sba_pool_select_lse(q, k, B, H, Npad, D, vl, block, nsub, s, budget, kmax, idx, cnt, ws, wsb, S)


@pytest.mark.parametrize("kwargs,code", [
    (dict(q=NULL), 1), (dict(ws=NULL), 1), (dict(nsub=2), 2), (dict(nsub=1), 2), (dict(nsub=16), 2),
    (dict(budget=0), 1), (dict(budget=-3), 1), (dict(s=1.0), 1), (dict(D=96), 2), (dict(Npad=1000), 1),
    # 16 blocks at s = 0.5 keep 8; a budget of 3 rounds that up to 9
    (dict(budget=3, kmax=8), 1), (dict(s=0.6, budget=1, kmax=6), 1),
    (dict(wsb=1024), 1), (dict(q=MIS), 3), (dict(vl=MIS), 3),
])
def test_pool_select_lse_rejects(lib, kwargs, code):
    assert pool_select_lse(lib, **kwargs) == code


def test_lse_workspace_size(lib):
    one = lib.sba_pool_select_workspace_size(1, 24, 32768, 128, 64)
    four = lib.sba_pool_select_lse_workspace_size(1, 24, 32768, 128, 64, 4)
    assert four > one
    assert lib.sba_pool_select_lse_workspace_size(1, 24, 32768, 128, 64, 2) == 0
    assert lib.sba_pool_select_lse_workspace_size(1, 24, 32760, 128, 64, 4) == 0


def producer(lib, x=A, w=A, pos=A, B=1, H=2, Npad=1024, D=128, vl=NULL, block=64, rd=96, base=10000.0,
             eps=1e-6, out=A, means=A):
    return lib.sba_qk_norm_rope_pool(x, w, pos, B, H, Npad, D, vl, block, rd, base, eps, out, means, S)


@pytest.mark.parametrize("kwargs,code", [
    (dict(x=NULL), 1), (dict(w=NULL), 1), (dict(pos=NULL), 1), (dict(out=NULL), 1),
    (dict(rd=100), 1), (dict(rd=-6), 1), (dict(rd=132), 1), (dict(base=0.0), 1), (dict(base=float("inf")), 1),
    (dict(eps=float("nan")), 1), (dict(eps=-1.0), 1), (dict(D=96), 2), (dict(Npad=1000), 1),
    (dict(x=MIS), 3), (dict(w=MIS), 3), (dict(means=MIS), 3), (dict(pos=ctypes.c_void_p(0x10002)), 3),
])
def test_producer_rejects(lib, kwargs, code):
    assert producer(lib, **kwargs) == code


def test_pool_select_means_rejects(lib):
    f = lambda qm=A, km=A, D=128, s=0.5, kmax=8, ws=A, wsb=1 << 30: lib.sba_pool_select_means(
        qm, km, 1, 2, 1024, D, NULL, 64, s, kmax, A, A, ws, wsb, S)
    assert f(qm=NULL) == 1 and f(km=NULL) == 1 and f(ws=NULL) == 1
    assert f(kmax=7) == 1 and f(s=1.0) == 1 and f(wsb=16) == 1
    assert f(D=80) == 2
    assert f(qm=MIS) == 3


def test_compensated_rejects(lib):
    f = lambda q=A, v=A, idx=A, cnt=A, kmax=8, D=128, po=NULL: lib.sba_attention_compensated(
        q, A, v, A, A, 1, 2, 1024, D, NULL, 64, idx, cnt, kmax, po, 0.0, S)
    assert f(q=NULL) == 1 and f(v=NULL) == 1 and f(idx=NULL) == 1 and f(cnt=NULL) == 1
    assert f(kmax=0) == 1
    assert f(D=96) == 2
    assert f(q=MIS) == 3 and f(po=ctypes.c_void_p(0x10002)) == 3


def test_mean_compensated_rejects(lib):
    f = lambda q=A, v=A, idx=A, cnt=A, kmax=8, D=128, ws=A, wsb=1 << 30, po=NULL: \
        lib.sba_attention_mean_compensated(q, A, v, A, A, 1, 2, 1024, D, NULL, 64, idx, cnt, kmax, po, 0.0, ws, wsb,
                                           S)
    assert lib.sba_mean_compensation_workspace_size(1, 2, 1024, 128, 64) > 0
    assert lib.sba_mean_compensation_workspace_size(1, 2, 1000, 128, 64) == 0
    assert f(q=NULL) == 1 and f(v=NULL) == 1 and f(idx=NULL) == 1 and f(cnt=NULL) == 1
    assert f(ws=NULL) == 1 and f(wsb=16) == 1 and f(kmax=0) == 1
    assert f(D=96) == 2
    assert f(ws=MIS) == 3 and f(po=ctypes.c_void_p(0x10002)) == 3


def test_keep_count_budget_export(lib):
    """The budget rule is the library's: the binding only forwards to it."""
    import video_dit_block_b200 as sba
    assert lib.sba_keep_count_budget(1182, 0.8, 1) == lib.sba_keep_count(1182, 0.8) == 237
    assert lib.sba_keep_count_budget(1182, 0.8, 8) == 240
    assert lib.sba_keep_count_budget(10, 0.05, 8) == 10        # capped at n
    assert lib.sba_keep_count_budget(10, 0.5, 0) == 0          # budget < 1
    assert lib.sba_keep_count_budget(0, 0.5, 8) == 0
    assert sba.keep_count_budget(1182, 0.8, 8) == 240


def test_attention_to_shards_rejects(lib):
    def f(n=2, ptrs=None, lptrs=None, h_total=4, h_first=2, H=2, Npad=1024, D=128, q=A, idx=A):
        arr = (ctypes.c_void_p * max(n, 1))(*(ptrs if ptrs is not None else [A.value] * max(n, 1)))
        larr = None if lptrs is None else (ctypes.c_void_p * max(n, 1))(*lptrs)
        return lib.sba_attention_to_shards(q, A, A, ctypes.cast(arr, ctypes.c_void_p),
                                           None if larr is None else ctypes.cast(larr, ctypes.c_void_p), n, h_total,
                                           h_first, 1, H, Npad, D, NULL, 64, idx, A, 8, NULL, 0.0, S)
    assert f(n=0) == 1 and f(n=9) == 1                    # 1 .. 8 shards
    assert f(Npad=1024, n=3) == 1                          # Npad must split evenly
    assert f(h_first=3) == 1 and f(h_first=-1) == 1        # heads outside h_total
    assert f(ptrs=[A.value, None]) == 1                    # a missing shard
    assert f(lptrs=[A.value, None]) == 1
    assert f(ptrs=[A.value, MIS.value]) == 3               # o shards 16-byte aligned
    assert f(lptrs=[A.value, 0x10002]) == 3                # lse shards 4-byte aligned
    assert f(q=NULL) == 1 and f(idx=NULL) == 1
    assert f(D=96) == 2


def test_set_attention_kernel_values(lib):
    for which in (0, 1, 2):
        assert lib.sba_set_attention_kernel(which) == 0
    assert lib.sba_set_attention_kernel(3) == 1 and lib.sba_set_attention_kernel(-1) == 1
    assert lib.sba_set_attention_kernel(0) == 0        # back to the default


def test_token_prune_rejects(lib):
    assert lib.sba_keep_token_count(63240, 0.5) == 31620
    assert lib.sba_keep_token_count(10, 1.5) == 0
    assert lib.sba_token_prune_workspace_size(2, 63240) >= 2 * 63240 * 8
    assert lib.sba_token_prune_workspace_size(0, 5) == 0
    f = lambda x=A, N=1000, C=64, r=0.5, npo=512, idx=A, vo=A, ws=A, wsb=1 << 20: lib.sba_token_prune_select(
        x, 2, N, C, NULL, r, npo, idx, vo, ws, wsb, S)
    assert f(x=NULL) == 1 and f(idx=NULL) == 1 and f(vo=NULL) == 1 and f(ws=NULL) == 1
    assert f(r=1.5) == 1 and f(r=-0.1) == 1
    assert f(npo=499) == 1                       # keep_tokens(1000, 0.5) = 500
    assert f(wsb=1000) == 1
    assert f(C=60) == 2                          # C % 8 != 0
    assert f(x=MIS) == 3 and f(ws=MIS) == 3 and f(idx=ctypes.c_void_p(0x10002)) == 3


def test_gather_tokens_rejects(lib):
    f = lambda src=A, rb=256, idx=A, vo=A, dst=A, npo=64: lib.sba_gather_tokens(src, 2, 4, 1000, rb, idx, vo, npo,
                                                                                 dst, S)
    assert f(src=NULL) == 1 and f(dst=NULL) == 1 and f(idx=NULL) == 1 and f(vo=NULL) == 1
    assert f(rb=0) == 1 and f(npo=0) == 1
    assert f(rb=6) == 2                          # not a multiple of 4
    assert f(src=MIS) == 3 and f(dst=MIS) == 3   # 16-byte units for 256-byte rows
    assert f(rb=12, src=ctypes.c_void_p(0x10002)) == 3
