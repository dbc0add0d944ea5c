"""GPU compensated block-sparse attention (sba_attention_compensated) against the fp64
oracle, under the GPU's own routing.  Same tolerances as the plain attention path:
the block means are the same bf16 values on both sides (fp64 sums, one rounding), so
what remains is the attention arithmetic."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, output_errors, to_device
from workloads import f64_to_bf16_bits, make_custom, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def check(sba, oracle_mod, w, s, paired=True, qblocks=None):
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, s)
    po = sba.pair_query_blocks(idx, cnt, vl) if paired else None
    o, lse = sba.attention_compensated(q, k, v, idx, cnt, vl, pair_order=po)
    assert sba.device_status() == 0
    o_ref, lse_ref = oracle_mod.attention_compensated(w.q, w.k, w.v, idx.cpu().numpy(), cnt.cpu().numpy(),
                                                      w.valid_len, qblocks=qblocks)
    rows = np.isfinite(lse_ref)
    mx, mean = output_errors(o.float().cpu().numpy(), o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    lg = lse.cpu().numpy()
    np.testing.assert_allclose(lg[rows], lse_ref[rows], rtol=0, atol=1e-4)
    if qblocks is None:
        # rows past each sample: o = 0, lse = -inf
        for b in range(w.q.shape[0]):
            L = int(w.valid_len[b])
            assert np.all(np.isneginf(lg[b, :, L:]))
    return o, lse, idx, cnt


CASES = [
    # B, H, D, grid, sparsity, drop
    (1, 2, 128, (2, 16, 40), 0.75, 0.0),
    (2, 3, 128, (3, 10, 50), 0.5, 0.15),     # ragged
    (1, 1, 64, (5, 9, 37), 0.8, 0.1),        # D = 64, odd block count
    (3, 2, 128, (1, 7, 9), 0.5, 0.0),        # one partial block
    (1, 2, 128, (9, 30, 52), 0.9, 0.0),      # 220 blocks: four mean steps
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("paired", [True, False])
def test_parity(sba, oracle_mod, case, paired):
    B, H, D, grid, s, drop = case
    w = make_custom(B, H, D, grid, s, drop_rate=drop, seed=hash(case) % 991)
    check(sba, oracle_mod, w, s, paired=paired)


def test_block_constant_inputs_give_dense(sba, oracle_mod):
    """Keys and values constant within blocks: the compensation is exact, so the output
    is dense attention's."""
    rng = np.random.default_rng(5)
    B, H, N, D = 1, 2, 1280, 128
    bfx = lambda x: f64_to_bf16_bits(np.asarray(x, dtype=np.float64))
    rep = lambda a: np.repeat(a, 64, axis=2)[:, :, :N]
    w = make_custom(B, H, D, (2, 16, 40), 0.8, seed=7)
    w.q = bfx(rng.normal(size=(B, H, N, D)))
    w.k = bfx(rep(rng.normal(size=(B, H, N // 64, D))))
    w.v = bfx(rep(rng.normal(size=(B, H, N // 64, D))))
    o, lse, _, _ = check(sba, oracle_mod, w, 0.8)
    o_d, lse_d = oracle_mod.dense(w.q, w.k, w.v, w.valid_len)
    mx, mean = output_errors(o.float().cpu().numpy(), o_d)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


def test_nothing_dropped_equals_plain_attention(sba, oracle_mod):
    w = make_custom(1, 2, 128, (2, 16, 40), 0.0, seed=9, drop_rate=0.1)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.0)
    po = sba.pair_query_blocks(idx, cnt, vl)
    o1, l1 = sba.attention_paired(q, k, v, idx, cnt, po, vl)
    o2, l2 = sba.attention_compensated(q, k, v, idx, cnt, vl, pair_order=po)
    assert sba.device_status() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)


def test_full_size_720p_sampled(sba, oracle_mod):
    w = make_workload("720p")
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    po = sba.pair_query_blocks(idx, cnt, vl)
    o, lse = sba.attention_compensated(q, k, v, idx, cnt, vl, pair_order=po)
    assert sba.device_status() == 0
    rng = np.random.default_rng(1)
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    nB = (int(w.valid_len[0]) + 63) // 64
    for h in (0, w.q.shape[1] - 1):
        sl = lambda x: np.ascontiguousarray(x[:, h:h + 1])
        qb = np.unique(np.concatenate([rng.choice(nB, 10, replace=False), [nB - 1]])).astype(np.int32)
        o_ref, lse_ref = oracle_mod.attention_compensated(sl(w.q), sl(w.k), sl(w.v), idx_h[:, h:h + 1],
                                                          cnt_h[:, h:h + 1], w.valid_len, qblocks=qb)
        rows = np.isfinite(lse_ref)
        mx, mean = output_errors(o[:, h:h + 1].float().cpu().numpy(), o_ref, rows)
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (h, mx, mean)
        np.testing.assert_allclose(lse[:, h:h + 1].cpu().numpy()[rows], lse_ref[rows], rtol=0, atol=1e-4)
