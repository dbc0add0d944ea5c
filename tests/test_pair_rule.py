"""The plain statement of the query-block pairing rule (tests/pair_rule.py), pinned on
hand-made kept sets whose pairing follows from the rule by inspection, and on the
oracle's routing of named workloads (a permutation of the query blocks that never
grows the union work).  The GPU pass is compared with this statement element for
element in test_gpu_pair.py."""
import numpy as np
import pytest

from pair_rule import host_pairing
from workloads import make_workload


def lists(sets, kmax=None):
    """kv_idx / kv_cnt rows from a list of kept sets (ascending, -1 padded)."""
    kmax = kmax or max(1, max(len(s) for s in sets))
    idx = np.full((len(sets), kmax), -1, dtype=np.int32)
    cnt = np.zeros(len(sets), dtype=np.int32)
    for a, s in enumerate(sets):
        v = sorted(s)
        idx[a, :len(v)] = v
        cnt[a] = len(v)
    return idx, cnt


def tiles_union(idx, cnt, order):
    tot = 0
    for a, c in zip(order[0::2], order[1::2]):
        sa = set(idx[a, :cnt[a]].tolist()) if a >= 0 else set()
        sc = set(idx[c, :cnt[c]].tolist()) if c >= 0 else set()
        tot += len(sa | sc)
    return tot


def test_equal_sets_pair_across_a_gap():
    # 0 and 2 keep the same blocks, as do 1 and 3: overlap outranks nearness
    idx, cnt = lists([{0, 1}, {2, 3}, {0, 1}, {2, 3}])
    assert host_pairing(idx, cnt, 4, 4).tolist() == [0, 2, 1, 3]


def test_overlap_outranks_distance():
    # block 0 shares one block with its neighbour 1 and three with block 5
    sets = [{0, 1, 2}, {0, 5}, {3}, {4}, {5}, {0, 1, 2, 3}]
    idx, cnt = lists(sets)
    order = host_pairing(idx, cnt, 6, 6)
    assert order[:2].tolist() == [0, 5]


def test_equal_overlaps_go_to_the_nearer_then_the_lower_block():
    # every block keeps the same single block: all overlaps equal.  Round 0 matches 0-1
    # (1 prefers 0, the lower of its two neighbours at distance 1); the next rounds
    # match 2-3, then 4-5, each taking its first still unmatched candidate.
    idx, cnt = lists([{0}] * 6)
    assert host_pairing(idx, cnt, 6, 6).tolist() == [0, 1, 2, 3, 4, 5]


def test_rows_keeping_every_block_propose_nothing():
    # dense routing (every row of a sample keeps the same count, here all blocks): the
    # tiles stay adjacent
    idx, cnt = lists([set(range(5))] * 5)
    assert host_pairing(idx, cnt, 5, 5).tolist() == [0, 1, 2, 3, 4, -1]


def test_blocks_past_the_valid_length_come_last():
    # nQ = 5 query blocks, 3 of them valid: the padding blocks 3 and 4 keep nothing
    idx, cnt = lists([{0}, {1, 2}, {0}, set(), set()], kmax=2)
    assert host_pairing(idx, cnt, 3, 5).tolist() == [0, 2, 1, 3, 4, -1]


def test_the_window_limits_candidates():
    # 0 and 70 keep the same blocks but lie 70 positions apart, beyond the +-64 window
    sets = [{0}] + [{i + 1} for i in range(69)] + [{0}]
    idx, cnt = lists(sets)
    order = host_pairing(idx, cnt, 71, 71)
    pos = {int(v): i for i, v in enumerate(order) if v >= 0}
    assert pos[0] // 2 != pos[70] // 2
    with_wider = host_pairing(idx, cnt, 71, 71, window=96)
    assert with_wider[:2].tolist() == [0, 70]


@pytest.mark.parametrize("name,heads", [("tiny", None), ("480p_sparse", 1)])
def test_oracle_routing_pairs_into_a_permutation_with_less_union(oracle_mod, name, heads):
    w = make_workload(name, heads=heads)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, w.sparsity)
    nQ = w.Npad // 64
    for b in range(w.B):
        nB = (int(w.valid_len[b]) + 63) // 64
        for h in range(w.H):
            order = host_pairing(idx[b, h], cnt[b, h], nB, nQ)
            assert len(order) == 2 * ((nQ + 1) // 2)
            assert sorted(order[order >= 0].tolist()) == list(range(nQ))
            adjacent = np.array([t if t < nQ else -1 for t in range(2 * ((nQ + 1) // 2))])
            paired, adj = tiles_union(idx[b, h], cnt[b, h], order), tiles_union(idx[b, h], cnt[b, h], adjacent)
            assert paired <= adj
            if name != "tiny":
                assert paired < 0.98 * adj, (paired, adj)
