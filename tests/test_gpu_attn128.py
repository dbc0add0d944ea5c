"""The query-pair attention kernel that walks its union two key blocks (128 keys) per
step, chosen with set_attention_kernel("key_pairs"), against the fp64 oracle fed the GPU
routing, with the tolerances of the other attention tests: dense attention, routings
that keep every block and sparse ones (odd and even union lengths, steps where one half
keeps neither block, one block or both), ragged lengths, paired tiles, the output to
sequence shards, full-length heads, and the timeout path."""
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


class kernel:
    """Select the two-key-block kernel for the duration of a with-block."""

    def __init__(self, sba, which="key_pairs"):
        self.sba, self.which = sba, which

    def __enter__(self):
        self.sba.set_attention_kernel(self.which)

    def __exit__(self, *exc):
        self.sba.set_attention_kernel("auto")


def valid_rows(w):
    n = np.arange(w.Npad)
    return np.broadcast_to((n[None, :] < w.valid_len[:, None])[:, None, :], (w.B, w.H, w.Npad))


def check(oracle_mod, w, o, lse, idx_h, cnt_h, qblocks=None):
    o_ref, lse_ref = oracle_mod.attention(w.q, w.k, w.v, idx_h, cnt_h, w.valid_len, qblocks=qblocks)
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    rows = valid_rows(w) & ~np.isnan(lse_ref)
    mx, mean = output_errors(og, o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    np.testing.assert_allclose(lg[rows], lse_ref[rows], rtol=0, atol=1e-4)
    if qblocks is None:
        pad = ~valid_rows(w)
        assert np.all(og[pad] == 0.0) and np.all(np.isneginf(lg[pad]))


SHAPES = [
    (1, 2, (1, 8, 40), None),                 # 320 tokens, 5 blocks: odd dense union
    (2, 2, (2, 8, 24), [384, 200]),           # ragged second sample
    (1, 3, (1, 16, 28), [441]),               # 7 blocks, ragged tail
    (2, 1, (4, 16, 32), [2048, 65]),          # 32 blocks; 2 blocks in the short sample
    (1, 2, (3, 10, 50), [1500]),              # 24 blocks, partial last block
]


@pytest.mark.parametrize("shape", SHAPES)
def test_dense(sba, oracle_mod, shape):
    B, H, grid, vl = shape
    w = make_custom(B, H, 128, grid, 0.0, seed=61)
    if vl is not None:
        w.valid_len = np.array(vl, dtype=np.int32)
    q, k, v, vlt = to_device(w, DEV)
    with kernel(sba):
        o, lse = sba.dense_attention(q, k, v, vlt)
        assert sba.device_status() == 0
    nB = w.Npad // 64
    idx = np.broadcast_to(np.arange(nB, dtype=np.int32), (B, H, nB, nB)).copy()
    cnt = np.zeros((B, H, nB), dtype=np.int32)
    for b in range(B):
        nb = (int(w.valid_len[b]) + 63) // 64
        cnt[b, :, :nb] = nb
    check(oracle_mod, w, o, lse, idx, cnt)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("s", [0.0, 0.5, 0.8, 0.95])
@pytest.mark.parametrize("paired", [False, True])
def test_routed(sba, oracle_mod, shape, s, paired):
    B, H, grid, vl = shape
    w = make_custom(B, H, 128, grid, s, seed=62)
    if vl is not None:
        w.valid_len = np.array(vl, dtype=np.int32)
    q, k, v, vlt = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vlt, s)
    with kernel(sba):
        if paired:
            o, lse = sba.attention_paired(q, k, v, idx, cnt, sba.pair_query_blocks(idx, cnt, vlt), vlt)
        else:
            o, lse = sba.attention(q, k, v, idx, cnt, vlt)
        assert sba.device_status() == 0
    check(oracle_mod, w, o, lse, idx.cpu().numpy(), cnt.cpu().numpy())


def test_random_routings(sba, oracle_mod):
    """External routings with random kept sets of every size (including empty rows):
    steps where a half keeps both blocks, one, or neither."""
    rng = np.random.default_rng(63)
    w = make_custom(1, 2, 128, (2, 16, 40), 0.5, seed=64)
    B, H, nB = 1, 2, w.Npad // 64
    idx = np.full((B, H, nB, nB), -1, dtype=np.int32)
    cnt = np.zeros((B, H, nB), dtype=np.int32)
    for h in range(H):
        for I in range(nB):
            c = 0 if I % 9 == 4 else int(rng.integers(1, nB + 1))
            idx[0, h, I, :c] = np.sort(rng.choice(nB, c, replace=False))
            cnt[0, h, I] = c
    q, k, v, vlt = to_device(w, DEV)
    with kernel(sba):
        o, lse = sba.attention(q, k, v, torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV), vlt)
        assert sba.device_status() == 0
    check(oracle_mod, w, o, lse, idx, cnt)


@pytest.mark.parametrize("name", ["480p_sparse", "long_clip"])
def test_kernels_agree_full_length(sba, oracle_mod, name):
    """Both query-pair kernels on full-length heads: equal up to accumulation order, and
    the two-key-block kernel within tolerance of the oracle on sampled query blocks."""
    w = make_workload(name, heads=2)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, w.sparsity)
    po = sba.pair_query_blocks(idx, cnt, vl)
    o1, l1 = sba.attention_paired(q, k, v, idx, cnt, po, vl)
    with kernel(sba):
        o2, l2 = sba.attention_paired(q, k, v, idx, cnt, po, vl)
        assert sba.device_status() == 0
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    fin = torch.isfinite(l1)
    assert torch.equal(fin, torch.isfinite(l2))
    assert (l1[fin] - l2[fin]).abs().max().item() <= 1e-4
    nB = (int(w.valid_len.min()) + 63) // 64
    qb = np.unique(np.concatenate([np.random.default_rng(5).choice(nB, 6, replace=False), [0, nB - 1]]))
    check(oracle_mod, w, o2, l2, idx.cpu().numpy(), cnt.cpu().numpy(), qblocks=qb.astype(np.int32))


def test_shard_output_equals_plain_output(sba, oracle_mod):
    """Output straight into sequence shards (the Ulysses exchange) stays on the other
    kernel; the two-key-block kernel's plain output matches it up to accumulation order."""
    w = make_custom(1, 2, 128, (2, 16, 32), 0.75, seed=65)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.75)
    shards = [torch.empty((1, 2, w.Npad // 2, 128), dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    with kernel(sba):
        o, _ = sba.attention(q, k, v, idx, cnt, vl)
        sba.attention_to_shards(q, k, v, idx, cnt, shards, None, valid_len=vl)
        assert sba.device_status() == 0
    assert (torch.cat(shards, dim=2).float() - o.float()).abs().max().item() <= 2e-2


def test_timeout_path(sba, oracle_mod):
    """A wait limit of one cycle makes every pending wait give up: the call reports
    SBA_ERR_TIMEOUT through the device status, and the next call is correct."""
    w = make_custom(1, 2, 128, (2, 16, 40), 0.5, seed=66)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.5)
    with kernel(sba):
        sba.set_wait_limit(1)
        try:
            sba.attention(q, k, v, idx, cnt, vl)
            st = sba.device_status()
        finally:
            sba.set_wait_limit(0)
        assert st == 5
        o, lse = sba.attention(q, k, v, idx, cnt, vl)
        assert sba.device_status() == 0
    check(oracle_mod, w, o, lse, idx.cpu().numpy(), cnt.cpu().numpy())


def test_bad_routing_entry_is_flagged_and_skipped(sba):
    w = make_custom(1, 2, 128, (2, 16, 40), 0.5, seed=67)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.5)
    bad = idx.clone()
    bad[0, 0, 3, 0] = 10_000           # outside [0, nB)
    bad[0, 1, 5, 1] = -2
    with kernel(sba):
        sba.attention(q, k, v, bad, cnt, vl)
        assert sba.device_status() == 6    # SBA_ERR_DEVICE_FLAG
        sba.attention(q, k, v, idx, cnt, vl)
        assert sba.device_status() == 0
