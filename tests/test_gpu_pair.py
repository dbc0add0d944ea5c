"""Query-block pairing (sba_pair_query_blocks) and attention over paired tiles
(sba_attention_paired): the pairing is a permutation of the query blocks, it cuts the
masked work of the union, and outputs still match the fp64 oracle."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, output_errors, to_device
from pair_rule import host_pairing
from workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def check_permutation(po, nQ):
    B, H, S = po.shape
    assert S == 2 * ((nQ + 1) // 2)
    for b in range(B):
        for h in range(H):
            row = po[b, h]
            vals = row[row >= 0]
            assert sorted(vals.tolist()) == list(range(nQ)), (b, h)
            assert (row < 0).sum() == S - nQ


def union_work(idx, cnt, tiles):
    tot = 0
    for a, c in tiles:
        sa = set(idx[a, :cnt[a]].tolist()) if a >= 0 else set()
        sc = set(idx[c, :cnt[c]].tolist()) if c >= 0 else set()
        tot += len(sa | sc)
    return tot


@pytest.mark.parametrize("name,heads", [("tiny", None), ("480p_sparse", 2), ("720p", 1), ("long_clip", 1)])
def test_pairing_is_permutation_and_cuts_union(sba, name, heads):
    w = make_workload(name, heads=heads)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    po = sba.pair_query_blocks(idx, cnt, vl)
    assert sba.device_status() == 0
    nQ = w.Npad // 64
    po_h, idx_h, cnt_h = po.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()
    check_permutation(po_h, nQ)
    paired = adjacent = 0
    for b in range(w.B):
        for h in range(w.H):
            tiles = list(zip(po_h[b, h, 0::2], po_h[b, h, 1::2]))
            adj = [(2 * t, 2 * t + 1 if 2 * t + 1 < nQ else -1) for t in range((nQ + 1) // 2)]
            paired += union_work(idx_h[b, h], cnt_h[b, h], tiles)
            adjacent += union_work(idx_h[b, h], cnt_h[b, h], adj)
    assert paired <= adjacent
    if w.sparsity > 0 and name != "tiny":
        assert paired < 0.98 * adjacent, (paired, adjacent)


@pytest.mark.parametrize("name,heads", [("tiny", None), ("480p_sparse", 1), ("long_clip", 1)])
def test_pairing_equals_host_statement(sba, name, heads):
    """The GPU tile list equals the plain statement of the rule on the GPU's own routing."""
    w = make_workload(name, heads=heads)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    po = sba.pair_query_blocks(idx, cnt, vl)
    assert sba.device_status() == 0
    nQ = w.Npad // 64
    po_h, idx_h, cnt_h = po.cpu().numpy(), idx.cpu().numpy(), cnt.cpu().numpy()
    for b in range(w.B):
        nB = (int(w.valid_len[b]) + 63) // 64
        for h in range(w.H):
            np.testing.assert_array_equal(po_h[b, h], host_pairing(idx_h[b, h], cnt_h[b, h], nB, nQ))


CASES = [
    (1, 2, 128, (2, 16, 40), 0.75, 0.0),
    (2, 3, 128, (3, 10, 50), 0.5, 0.15),
    (1, 1, 64, (5, 9, 37), 0.8, 0.1),      # odd number of query blocks, D = 64
    (3, 2, 128, (1, 7, 9), 0.5, 0.0),      # a single partial block
    (1, 2, 128, (3, 12, 40), 0.0, 0.05),   # dense routing
]


@pytest.mark.parametrize("case", CASES)
def test_paired_attention_matches_oracle(sba, oracle_mod, case):
    B, H, D, grid, s, drop = case
    w = make_custom(B, H, D, grid, s, drop_rate=drop, seed=hash(case) % 1000 + 7)
    q, k, v, vl = to_device(w, DEV)
    o, lse, idx, cnt = sba.sparse_attention(q, k, v, vl, s)
    assert sba.device_status() == 0
    o_ref, lse_ref = oracle_mod.attention(w.q, w.k, w.v, idx.cpu().numpy(), cnt.cpu().numpy(), w.valid_len)
    n = np.arange(w.Npad)
    valid = np.broadcast_to((n[None, :] < w.valid_len[:, None])[:, None, :], (w.B, w.H, w.Npad))
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    mx, mean = output_errors(og, o_ref, valid)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    np.testing.assert_allclose(lg[valid], lse_ref[valid], rtol=0, atol=1e-4)
    assert np.all(og[~valid] == 0.0) and np.all(np.isneginf(lg[~valid]))


def test_paired_equals_unpaired_closely(sba):
    w = make_workload("480p_sparse", heads=2)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    po = sba.pair_query_blocks(idx, cnt, vl)
    o1, l1 = sba.attention(q, k, v, idx, cnt, vl)
    o2, l2 = sba.attention_paired(q, k, v, idx, cnt, po, vl)
    assert sba.device_status() == 0
    assert (o1.float() - o2.float()).abs().max().item() <= 1e-2
    fin = torch.isfinite(l1)
    assert torch.equal(fin, torch.isfinite(l2))
    assert (l1[fin] - l2[fin]).abs().max().item() <= 1e-4
