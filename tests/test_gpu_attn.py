"""GPU attention (sba_attention, sba_dense_attention) against the fp64 oracle.

The oracle is fed the GPU's own routing, so the output check is independent of the
routing check.  Tolerance (bf16 inputs): max-abs 2e-2 and mean-abs 2e-3 over the
valid rows; padding rows must be exactly 0 with lse = -inf."""
import math

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
    return m


def valid_rows(w):
    n = np.arange(w.Npad)
    return np.broadcast_to((n[None, :] < w.valid_len[:, None])[:, None, :], (w.B, w.H, w.Npad))


def check_attention(sba, oracle_mod, w, qblocks=None, scale=0.0):
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    o, lse = sba.attention(q, k, v, idx, cnt, vl, softmax_scale=scale)
    assert sba.device_status() == 0
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    o_ref, lse_ref = oracle_mod.attention(w.q, w.k, w.v, idx_h, cnt_h, w.valid_len, scale=scale,
                                          qblocks=qblocks)
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    rows = valid_rows(w) & ~np.isnan(lse_ref)
    mx, mean = output_errors(og, o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    np.testing.assert_allclose(lg[rows], lse_ref[rows], rtol=0, atol=1e-4)
    pad = ~valid_rows(w)
    assert np.all(og[pad] == 0.0) and np.all(np.isneginf(lg[pad]))
    return mx, mean


@pytest.mark.parametrize("name,heads,nq", [("tiny", None, None), ("480p_dense", 1, 24),
                                           ("480p_sparse", 2, 48), ("720p", 1, 40),
                                           ("long_clip", 1, 32)])
def test_named_configs(sba, oracle_mod, name, heads, nq):
    w = make_workload(name, heads=heads)
    qb = None
    if nq is not None:
        nB = w.Npad // 64
        qb = np.sort(np.random.default_rng(7).choice(nB, size=nq, replace=False)).astype(np.int32)
        qb = np.unique(np.concatenate([qb, [0, nB - 1]])).astype(np.int32)   # include the ragged tail
    check_attention(sba, oracle_mod, w, qblocks=qb)


CUSTOM = [
    (1, 2, 128, (2, 16, 40), 0.75, 0.0),
    (2, 3, 128, (3, 10, 50), 0.5, 0.15),
    (1, 1, 64, (5, 9, 37), 0.8, 0.1),
    (3, 2, 128, (1, 7, 9), 0.5, 0.0),
    (1, 2, 128, (4, 16, 64), 0.95, 0.0),
    (2, 2, 64, (7, 13, 29), 0.3, 0.2),
    (1, 2, 128, (3, 12, 40), 0.0, 0.05),
]


@pytest.mark.parametrize("case", CUSTOM)
def test_custom_shapes(sba, oracle_mod, case):
    B, H, D, grid, s, drop = case
    w = make_custom(B, H, D, grid, s, drop_rate=drop, seed=hash(case) % 1000 + 1)
    check_attention(sba, oracle_mod, w)


def test_custom_scale(sba, oracle_mod):
    w = make_custom(1, 2, 128, (2, 16, 40), 0.5, seed=77)
    check_attention(sba, oracle_mod, w, scale=0.05)


def test_sparse_s0_equals_dense(sba, oracle_mod):
    w = make_custom(2, 2, 128, (3, 10, 50), 0.0, seed=11, drop_rate=0.1)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.0)
    o_s, l_s = sba.attention(q, k, v, idx, cnt, vl)
    o_d, l_d = sba.dense_attention(q, k, v, vl)
    assert sba.device_status() == 0
    # same tiles, same order of key blocks: identical results
    assert torch.equal(o_s, o_d)
    assert torch.equal(l_s, l_d)
    o_ref, _ = oracle_mod.dense(w.q, w.k, w.v, w.valid_len)
    mx, mean = output_errors(o_d.float().cpu().numpy(), o_ref, valid_rows(w))
    assert mx <= MAX_ABS and mean <= MEAN_ABS


def test_dense_against_oracle(sba, oracle_mod):
    for case in [(1, 2, 64, (4, 16, 16)), (2, 1, 128, (3, 9, 33))]:
        B, H, D, grid = case
        w = make_custom(B, H, D, grid, 0.0, seed=13, drop_rate=0.1 if B > 1 else 0.0)
        q, k, v, vl = to_device(w, DEV)
        o, lse = sba.dense_attention(q, k, v, vl)
        o_ref, lse_ref = oracle_mod.dense(w.q, w.k, w.v, w.valid_len)
        rows = valid_rows(w)
        mx, mean = output_errors(o.float().cpu().numpy(), o_ref, rows)
        assert mx <= MAX_ABS and mean <= MEAN_ABS
        np.testing.assert_allclose(lse.cpu().numpy()[rows], lse_ref[rows], rtol=0, atol=1e-4)


def test_oracle_routing_fed_to_gpu(sba, oracle_mod):
    w = make_custom(1, 2, 128, (3, 10, 50), 0.75, seed=19)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.75)
    q, k, v, vl = to_device(w, DEV)
    o, _ = sba.attention(q, k, v, torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV), vl)
    o_ref, _ = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    mx, mean = output_errors(o.float().cpu().numpy(), o_ref, valid_rows(w))
    assert mx <= MAX_ABS and mean <= MEAN_ABS


def test_arbitrary_routing_and_empty_rows(sba, oracle_mod):
    """Routings the router would not produce: random kept sets of varying size, and
    empty rows (their valid query rows get o = 0, lse = -inf)."""
    w = make_custom(1, 2, 128, (2, 16, 40), 0.5, seed=23, drop_rate=0.0)
    nB = w.Npad // 64
    rng = np.random.default_rng(3)
    kmax = nB
    idx = np.full((1, 2, nB, kmax), -1, dtype=np.int32)
    cnt = np.zeros((1, 2, nB), dtype=np.int32)
    for h in range(2):
        for I in range(nB):
            c = 0 if (I % 7 == 3) else int(rng.integers(1, nB + 1))
            sel = np.sort(rng.choice(nB, size=c, replace=False))
            idx[0, h, I, :c] = sel
            cnt[0, h, I] = c
    q, k, v, vl = to_device(w, DEV)
    o, lse = sba.attention(q, k, v, torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV), vl)
    assert sba.device_status() == 0
    o_ref, lse_ref = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    mx, mean = output_errors(og, o_ref, valid_rows(w))
    assert mx <= MAX_ABS and mean <= MEAN_ABS
    empty = np.repeat(cnt == 0, 64, axis=2)
    assert np.all(og[empty] == 0.0) and np.all(np.isneginf(lg[empty]))


def test_poisoned_padding(sba, oracle_mod):
    w = make_custom(2, 2, 128, (3, 8, 30), 0.75, seed=29, drop_rate=0.15, pad_value=1e4)
    check_attention(sba, oracle_mod, w)


def test_valid_len_one_and_partial(sba, oracle_mod):
    w = make_custom(2, 2, 128, (2, 8, 40), 0.5, seed=43)
    w.valid_len = np.array([1, 577], dtype=np.int32)
    check_attention(sba, oracle_mod, w)


def test_constant_v(sba, oracle_mod):
    from workloads import f64_to_bf16_bits
    w = make_custom(1, 2, 128, (2, 16, 40), 0.75, seed=47)
    w.v = f64_to_bf16_bits(np.full(w.v.shape, 1.5))
    q, k, v, vl = to_device(w, DEV)
    o, _ = sba.sparse_attention(q, k, v, vl, 0.75)[:2]
    assert torch.all((o.float() - 1.5).abs() <= 2e-2)


def test_max_length(sba, oracle_mod):
    w = make_custom(1, 1, 128, (16, 128, 128), 0.95, seed=41)
    nB = w.Npad // 64
    qb = np.unique(np.concatenate([np.random.default_rng(2).choice(nB, 16, replace=False),
                                   [0, nB - 1]])).astype(np.int32)
    check_attention(sba, oracle_mod, w, qblocks=qb)
