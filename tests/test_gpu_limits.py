"""The largest sequence the library accepts (SBA_MAX_NPAD = 262144 tokens, 4096 blocks)
and the smallest sample (one token), through every routing and attention entry
point, against the oracle on samples it computes one by one."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, compare_routing, output_errors, to_device
from workloads import make_custom

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


@pytest.fixture(scope="module")
def maxw():
    # two samples of one head on a 4 x 256 x 256 latent grid: 262144 tokens; the tests
    # shorten the second sample through valid_len
    return make_custom(2, 1, 128, (4, 256, 256), 0.95, drop_rate=0.0, seed=41)


def test_max_length_routing_and_attention(sba, oracle_mod, maxw):
    w = maxw
    assert w.q.shape[2] == 262144
    w.valid_len = np.array([262144, 262144 - 4096 - 17], dtype=np.int32)
    q, k, v, vl = to_device(w, DEV)
    o, lse, idx, cnt = sba.sparse_attention(q, k, v, vl, 0.95)
    assert sba.device_status() == 0
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    io, co, _, _, S = oracle_mod.select(w.q, w.k, w.valid_len, 0.95, kmax=idx_h.shape[-1],
                                        return_intermediates=True)
    bad, _ = compare_routing(idx_h, cnt_h, io, co, S)
    assert not bad, bad[:3]
    rng = np.random.default_rng(3)
    for b in range(2):
        nB = (int(w.valid_len[b]) + 63) // 64
        qb = np.unique(np.concatenate([rng.choice(nB, 4, replace=False), [0, nB - 1]])).astype(np.int32)
        sl = lambda x: np.ascontiguousarray(x[b:b + 1])
        o_ref, lse_ref = oracle_mod.attention(sl(w.q), sl(w.k), sl(w.v), idx_h[b:b + 1], cnt_h[b:b + 1],
                                              w.valid_len[b:b + 1], qblocks=qb)
        rows = np.isfinite(lse_ref)
        mx, mean = output_errors(o[b:b + 1].float().cpu().numpy(), o_ref, rows)
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (b, mx, mean)


def test_max_length_compensated_and_lse_router(sba, oracle_mod, maxw):
    w = maxw
    w.valid_len = np.array([262144, 200000], dtype=np.int32)
    q, k, v, vl = to_device(w, DEV)
    # the sub-block router at 16384 sub-blocks per head (its parity is covered at 720p):
    # kept counts, ascending distinct indices in range
    idx, cnt = sba.pool_select_lse(q, k, vl, 0.95, budget=8)
    assert sba.device_status() == 0
    ih, ch = idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(2):
        nB = (int(w.valid_len[b]) + 63) // 64
        assert np.all(ch[b, :, :nB] == oracle_mod.keep_count_budget(nB, 0.95, 8))
        assert np.all(ch[b, :, nB:] == 0)
        for I in range(0, nB, 211):
            row = ih[b, 0, I, :ch[b, 0, I]]
            assert np.all(np.diff(row) > 0) and row[0] >= 0 and row[-1] < nB
    idx, cnt = sba.pool_select(q, k, vl, 0.95)
    po = sba.pair_query_blocks(idx, cnt, vl)
    o, lse = sba.attention_compensated(q, k, v, idx, cnt, vl, pair_order=po)
    assert sba.device_status() == 0
    qb = np.array([0, 1, 2047, 3124], dtype=np.int32)   # 3124 = last block of the second sample
    for b in range(2):
        sl = lambda x: np.ascontiguousarray(x[b:b + 1])
        o_ref, lse_ref = oracle_mod.attention_compensated(sl(w.q), sl(w.k), sl(w.v), idx[b:b + 1].cpu().numpy(),
                                                          cnt[b:b + 1].cpu().numpy(), w.valid_len[b:b + 1],
                                                          qblocks=qb)
        rows = np.isfinite(lse_ref)
        mx, mean = output_errors(o[b:b + 1].float().cpu().numpy(), o_ref, rows)
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (b, mx, mean)


def test_one_token_sample(sba, oracle_mod):
    """valid_len = 1 beside a full sample: one block of one token, every path."""
    w = make_custom(2, 2, 128, (2, 8, 16), 0.75, seed=43)
    w.valid_len = np.array([256, 1], dtype=np.int32)
    q, k, v, vl = to_device(w, DEV)
    o, lse, idx, cnt = sba.sparse_attention(q, k, v, vl, 0.75)
    o2, lse2 = sba.attention_compensated(q, k, v, idx, cnt, vl)
    i3, c3 = sba.pool_select_lse(q, k, vl, 0.75, budget=8)
    assert sba.device_status() == 0
    assert np.all(cnt[1, :, 0].cpu().numpy() == 1) and np.all(cnt[1, :, 1:].cpu().numpy() == 0)
    assert np.all(c3[1, :, 0].cpu().numpy() == 1)
    o_ref, lse_ref = oracle_mod.attention(w.q, w.k, w.v, idx.cpu().numpy(), cnt.cpu().numpy(), w.valid_len)
    # the one-token sample attends to itself: o = v of that token, lse = its logit
    np.testing.assert_allclose(o[1, :, 0].float().cpu().numpy(), o_ref[1, :, 0], rtol=0, atol=1e-2)
    np.testing.assert_allclose(lse[1, :, 0].cpu().numpy(), lse_ref[1, :, 0], rtol=0, atol=1e-4)
    assert np.all(np.isneginf(lse[1, :, 1:].cpu().numpy()))
    assert torch.equal(o2[1, :, 0], o[1, :, 0])
