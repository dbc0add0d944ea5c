"""The CTA-pair attention kernel (a 2-SM cluster per four query blocks, tcgen05 MMAs of
M = 256), chosen with set_attention_kernel("cta_pair"), against the fp64 oracle fed the
GPU routing, with the tolerances of the other attention tests: dense attention, routings
that keep every block and sparse ones, ragged lengths, clusters whose second CTA or
whole tile lies past the sequence, odd union lengths, query blocks whose last steps
keep nothing, and the timeout path."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, output_errors, to_device
from workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    yield m
    m.set_attention_kernel("auto")


def valid_rows(w):
    n = np.arange(w.Npad)
    return np.broadcast_to((n[None, :] < w.valid_len[:, None])[:, None, :], (w.B, w.H, w.Npad))


def check(sba, oracle_mod, w, o, lse, idx_h, cnt_h, qblocks=None):
    o_ref, lse_ref = oracle_mod.attention(w.q, w.k, w.v, idx_h, cnt_h, w.valid_len, qblocks=qblocks)
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    rows = valid_rows(w) & ~np.isnan(lse_ref)
    mx, mean = output_errors(og, o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    np.testing.assert_allclose(lg[rows], lse_ref[rows], rtol=0, atol=1e-4)
    if qblocks is None:
        pad = ~valid_rows(w)
        assert np.all(og[pad] == 0.0) and np.all(np.isneginf(lg[pad]))


# (B, H, grid, valid lengths or None): 5 and 6 query blocks leave the last cluster's
# second CTA empty; 7 leaves it half full; the short sample's tiles lie past its length
SHAPES = [
    (1, 2, (1, 8, 40), None),                 # 320 tokens, 5 blocks
    (2, 2, (2, 8, 24), [384, 200]),           # 6 blocks, ragged second sample
    (1, 3, (1, 16, 28), [441]),               # 7 blocks, ragged tail
    (2, 1, (4, 16, 32), [2048, 65]),          # 32 blocks; 2 blocks in the short sample
]


@pytest.mark.parametrize("shape", SHAPES)
def test_dense(sba, oracle_mod, shape):
    B, H, grid, vl = shape
    w = make_custom(B, H, 128, grid, 0.0, seed=51)
    if vl is not None:
        w.valid_len = np.array(vl, dtype=np.int32)
    q, k, v, vlt = to_device(w, DEV)
    sba.set_attention_kernel("cta_pair")
    try:
        o, lse = sba.dense_attention(q, k, v, vlt)
        assert sba.device_status() == 0
    finally:
        sba.set_attention_kernel("auto")
    nB = w.Npad // 64
    idx = np.broadcast_to(np.arange(nB, dtype=np.int32), (B, H, nB, nB)).copy()
    cnt = np.zeros((B, H, nB), dtype=np.int32)
    for b in range(B):
        nb = (int(w.valid_len[b]) + 63) // 64
        cnt[b, :, :nb] = nb
    check(sba, oracle_mod, w, o, lse, idx, cnt)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("s", [0.0, 0.5, 0.8])
def test_routed(sba, oracle_mod, shape, s):
    """Routings that keep every block (s = 0) and sparse ones."""
    B, H, grid, vl = shape
    w = make_custom(B, H, 128, grid, s, seed=52)
    if vl is not None:
        w.valid_len = np.array(vl, dtype=np.int32)
    q, k, v, vlt = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vlt, s)
    sba.set_attention_kernel("cta_pair")
    try:
        o, lse = sba.attention(q, k, v, idx, cnt, vlt)
        assert sba.device_status() == 0
    finally:
        sba.set_attention_kernel("auto")
    check(sba, oracle_mod, w, o, lse, idx.cpu().numpy(), cnt.cpu().numpy())


def test_kernels_agree_480p_sparse(sba, oracle_mod):
    """Both kernels on a full-length sparse head: equal up to accumulation order, and the
    CTA pair within tolerance of the oracle on sampled query blocks."""
    w = make_workload("480p_sparse", heads=2)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    sba.set_attention_kernel("query_pairs")
    o1, l1 = sba.attention(q, k, v, idx, cnt, vl)
    sba.set_attention_kernel("cta_pair")
    o2, l2 = sba.attention(q, k, v, idx, cnt, vl)
    sba.set_attention_kernel("auto")
    assert sba.device_status() == 0
    d = (o1.float() - o2.float()).abs()
    assert float(d.max()) <= 2e-2 and float(d.mean()) <= 1e-3
    fin = torch.isfinite(l1)
    assert torch.equal(fin, torch.isfinite(l2))
    assert float((l1[fin] - l2[fin]).abs().max()) <= 1e-4
    nB = w.Npad // 64
    qb = np.unique(np.concatenate([np.random.default_rng(5).choice(nB, 12, replace=False),
                                   [0, nB - 1]])).astype(np.int32)
    o_ref, lse_ref = oracle_mod.attention(w.q, w.k, w.v, idx.cpu().numpy(), cnt.cpu().numpy(), w.valid_len,
                                          qblocks=qb)
    rows = np.isfinite(lse_ref)
    mx, mean = output_errors(o2.float().cpu().numpy(), o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


def test_480p_dense_sampled(sba, oracle_mod):
    """A full-length dense head, sampled query blocks."""
    w = make_workload("480p_dense", heads=1)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.0)
    sba.set_attention_kernel("cta_pair")
    try:
        o, lse = sba.attention(q, k, v, idx, cnt, vl)
        assert sba.device_status() == 0
    finally:
        sba.set_attention_kernel("auto")
    nB = w.Npad // 64
    qb = np.unique(np.concatenate([np.random.default_rng(6).choice(nB, 10, replace=False),
                                   [0, nB - 1]])).astype(np.int32)
    check(sba, oracle_mod, w, o, lse, idx.cpu().numpy(), cnt.cpu().numpy(), qblocks=qb)


def test_timeout_then_correct(sba, oracle_mod):
    w = make_custom(1, 2, 128, (2, 8, 24), 0.0, seed=53)
    q, k, v, vl = to_device(w, DEV)
    sba.set_attention_kernel("cta_pair")
    try:
        sba.set_wait_limit(1)
        try:
            sba.dense_attention(q, k, v, vl)
            assert sba.device_status() == 5   # SBA_ERR_TIMEOUT
        finally:
            sba.set_wait_limit(0)
        o, lse = sba.dense_attention(q, k, v, vl)
        assert sba.device_status() == 0
    finally:
        sba.set_attention_kernel("auto")
    nB = w.Npad // 64
    idx = np.broadcast_to(np.arange(nB, dtype=np.int32), (1, 2, nB, nB)).copy()
    cnt = np.full((1, 2, nB), nB, dtype=np.int32)
    check(sba, oracle_mod, w, o, lse, idx, cnt)


def test_bad_routing_flagged(sba):
    w = make_custom(1, 1, 128, (2, 8, 24), 0.5, seed=54)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.5)
    bad = idx.clone()
    bad[0, 0, 1, 0] = 10_000
    sba.set_attention_kernel("cta_pair")
    try:
        sba.attention(q, k, v, bad, cnt, vl)
        assert sba.device_status() == 6
        sba.attention(q, k, v, idx, cnt, vl)
        assert sba.device_status() == 0
    finally:
        sba.set_attention_kernel("auto")


def test_max_length_sampled(sba, oracle_mod):
    """The CTA pair at the length limit (262144 tokens, 4096 blocks), a ragged second
    sample, s = 0.95; sampled query blocks against the oracle."""
    w = make_custom(2, 1, 128, (4, 256, 256), 0.95, drop_rate=0.0, seed=41)
    w.valid_len = np.array([262144, 200000], dtype=np.int32)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.95)
    sba.set_attention_kernel("cta_pair")
    try:
        o, lse = sba.attention(q, k, v, idx, cnt, vl)
        assert sba.device_status() == 0
    finally:
        sba.set_attention_kernel("auto")
    qb = np.array([0, 1, 2047, 3124], dtype=np.int32)   # 3124 = last block of the second sample
    for b in range(2):
        sl = lambda x: np.ascontiguousarray(x[b:b + 1])
        o_ref, lse_ref = oracle_mod.attention(sl(w.q), sl(w.k), sl(w.v), idx[b:b + 1].cpu().numpy(),
                                              cnt[b:b + 1].cpu().numpy(), w.valid_len[b:b + 1], qblocks=qb)
        rows = np.isfinite(lse_ref)
        mx, mean = output_errors(o[b:b + 1].float().cpu().numpy(), o_ref, rows)
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (b, mx, mean)


def test_d64_falls_back_to_query_pairs(sba, oracle_mod):
    """The CTA pair is D = 128 only: chosen with D = 64, the query-pair kernel runs."""
    w = make_custom(1, 2, 64, (2, 8, 24), 0.5, seed=55)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.5)
    o_ref_gpu, _ = sba.attention(q, k, v, idx, cnt, vl)
    sba.set_attention_kernel("cta_pair")
    try:
        o, lse = sba.attention(q, k, v, idx, cnt, vl)
        assert sba.device_status() == 0
    finally:
        sba.set_attention_kernel("auto")
    assert torch.equal(o.view(torch.int16), o_ref_gpu.view(torch.int16))
    check(sba, oracle_mod, w, o, lse, idx.cpu().numpy(), cnt.cpu().numpy())
