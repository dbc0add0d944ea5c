"""GPU sub-block log-sum-exp routing (sba_pool_select_lse) against the fp64 oracle.

Kept sets must match the oracle's row for row.  Both sides evaluate the score in
fp64 in the same order, but their exp and log may round differently in the last
place, so a difference is excused only between blocks whose oracle scores lie
within the tie gap of the k-th score (counted, and expected to be rare)."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, compare_routing, output_errors, to_device
from workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def check_lse_routing(sba, oracle_mod, w, sparsity=None, budget=1):
    s = w.sparsity if sparsity is None else sparsity
    q, k, _, vl = to_device(w, DEV)
    idx_g, cnt_g = sba.pool_select_lse(q, k, vl, s, budget=budget)
    assert sba.device_status() == 0
    idx_o, cnt_o, S = oracle_mod.select_lse(w.q, w.k, w.valid_len, s, budget=budget, kmax=idx_g.shape[-1],
                                            return_scores=True)
    bad, excused = compare_routing(idx_g.cpu().numpy(), cnt_g.cpu().numpy(), idx_o, cnt_o, S)
    assert not bad, f"{len(bad)} routing rows differ, e.g. {bad[:3]}"
    assert len(excused) <= max(1, cnt_o.size // 100), f"{len(excused)} rows excused as ties"
    return idx_g, cnt_g


@pytest.mark.parametrize("name,heads", [("tiny", None), ("480p_sparse", 2), ("720p", 1), ("long_clip", 1)])
def test_named_configs(sba, oracle_mod, name, heads):
    w = make_workload(name, heads=heads)
    check_lse_routing(sba, oracle_mod, w)


@pytest.mark.parametrize("name", ["480p_sparse", "720p"])
def test_named_configs_budget8(sba, oracle_mod, name):
    w = make_workload(name, heads=1)
    check_lse_routing(sba, oracle_mod, w, budget=8)


CUSTOM = [
    # B, H, D, grid, sparsity, drop
    (1, 2, 128, (2, 16, 40), 0.75, 0.0),     # 20 blocks
    (2, 3, 128, (3, 10, 50), 0.5, 0.15),     # ragged batch: partial sub-blocks and empty ones
    (1, 1, 64, (5, 9, 37), 0.8, 0.1),        # odd block count, D = 64
    (3, 2, 128, (1, 7, 9), 0.5, 0.0),        # one partial block
    (1, 2, 128, (4, 16, 64), 0.95, 0.0),     # 64 blocks, keep 4
    (2, 2, 64, (7, 13, 29), 0.3, 0.2),
    (1, 2, 128, (9, 30, 52), 0.75, 0.0),     # 220 blocks: several score tiles in both directions
]


@pytest.mark.parametrize("case", CUSTOM)
def test_custom_shapes(sba, oracle_mod, case):
    B, H, D, grid, s, drop = case
    w = make_custom(B, H, D, grid, s, drop_rate=drop, seed=hash(case) % 1000)
    check_lse_routing(sba, oracle_mod, w)


@pytest.mark.parametrize("budget", [1, 3, 8])
@pytest.mark.parametrize("s", [0.0, 0.5, 0.8, 0.95])
def test_sparsity_budget_sweep(sba, oracle_mod, s, budget):
    w = make_custom(2, 2, 128, (3, 12, 40), s, seed=41, drop_rate=0.1)
    check_lse_routing(sba, oracle_mod, w, budget=budget)


def test_valid_lengths_at_sub_block_edges(sba, oracle_mod):
    """Lengths ending exactly on, and one token past, 16- and 64-token boundaries."""
    w = make_custom(6, 1, 128, (2, 16, 40), 0.6, seed=7)
    w.valid_len = np.array([1280, 1279, 1264, 1265, 1217, 1], dtype=np.int32)
    check_lse_routing(sba, oracle_mod, w)


def test_zero_queries_all_ties(sba, oracle_mod):
    """q = 0: every logit is 0 and full blocks tie exactly; the lowest indices win."""
    w = make_custom(1, 2, 128, (2, 16, 40), 0.7, seed=5)
    w.q = np.zeros_like(w.q)
    check_lse_routing(sba, oracle_mod, w)


def test_larger_kmax_and_reuse(sba, oracle_mod):
    """A wider kv_idx than needed, and a second call on the same workspace."""
    w = make_custom(1, 2, 128, (3, 12, 40), 0.75, seed=9)
    q, k, _, vl = to_device(w, DEV)
    kmax = sba.keep_count_budget(w.q.shape[2] // 64, 0.75, 8) + 5
    ws = torch.empty(sba.lse_workspace_size(1, 2, w.q.shape[2], 128), dtype=torch.uint8, device=DEV)
    for _ in range(2):
        idx, cnt = sba.pool_select_lse(q, k, vl, 0.75, budget=8, kmax=kmax, workspace=ws)
    io, co, S = oracle_mod.select_lse(w.q, w.k, w.valid_len, 0.75, budget=8, kmax=kmax, return_scores=True)
    bad, _ = compare_routing(idx.cpu().numpy(), cnt.cpu().numpy(), io, co, S)
    assert not bad


def test_sparse_attention_with_lse_router(sba, oracle_mod):
    """The whole path with the sub-block router: outputs against the oracle's
    attention under the oracle's own routing."""
    w = make_custom(2, 2, 128, (3, 12, 40), 0.75, seed=13, drop_rate=0.1)
    q, k, v, vl = to_device(w, DEV)
    o, lse, idx, cnt = sba.sparse_attention(q, k, v, vl, 0.75, router="lse", budget=8)
    assert sba.device_status() == 0
    io, co = oracle_mod.select_lse(w.q, w.k, w.valid_len, 0.75, budget=8, kmax=idx.shape[-1])
    o_ref, lse_ref = oracle_mod.attention(w.q, w.k, w.v, io, co, w.valid_len)
    rows = np.isfinite(lse_ref)
    mx, mean = output_errors(o.float().cpu().numpy(), o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    np.testing.assert_allclose(lse.cpu().numpy()[rows], lse_ref[rows], rtol=0, atol=1e-4)


@pytest.mark.parametrize("name", ["720p"])
def test_full_size_lse_routing_sampled_heads(sba, oracle_mod, name):
    """All heads routed on the GPU at full size; two heads checked against the oracle."""
    w = make_workload(name)
    q, k, _, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select_lse(q, k, vl, w.sparsity, budget=8)
    assert sba.device_status() == 0
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for h in (0, w.H - 1):
        sl = lambda x: np.ascontiguousarray(x[:, h:h + 1])
        io, co, S = oracle_mod.select_lse(sl(w.q), sl(w.k), w.valid_len, w.sparsity, budget=8,
                                          kmax=idx_h.shape[-1], return_scores=True)
        bad, _ = compare_routing(idx_h[:, h:h + 1], cnt_h[:, h:h + 1], io, co, S)
        assert not bad, (name, h, bad[:3])
