"""GPU routing (sba_pool_select, sba_block_means) against the fp64 oracle.

The kept sets must match the oracle row for row; the only tolerated difference is a
score tie (relative gap below 1e-6), which is counted.  Block means are compared
bit for bit (both sides sum the bf16 values of a block in token order in fp64)."""
import numpy as np
import pytest
import torch

from helpers import compare_routing, to_device
from workloads import f64_to_bf16_bits, make_custom, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def check_routing(sba, oracle_mod, w, sparsity=None):
    s = w.sparsity if sparsity is None else sparsity
    q, k, v, vl = to_device(w, DEV)
    idx_g, cnt_g = sba.pool_select(q, k, vl, s)
    assert sba.device_status() == 0
    idx_o, cnt_o, _, _, S = oracle_mod.select(w.q, w.k, w.valid_len, s, kmax=idx_g.shape[-1],
                                              return_intermediates=True)
    bad, excused = compare_routing(idx_g.cpu().numpy(), cnt_g.cpu().numpy(), idx_o, cnt_o, S)
    assert not bad, f"{len(bad)} routing rows differ, e.g. {bad[:3]}"
    return len(excused)


@pytest.mark.parametrize("name,heads", [("tiny", None), ("480p_dense", 1), ("480p_sparse", 2),
                                        ("720p", 1), ("long_clip", 1)])
def test_named_configs(sba, oracle_mod, name, heads):
    w = make_workload(name, heads=heads)
    check_routing(sba, oracle_mod, w)


CUSTOM = [
    # B, H, D, grid, sparsity, drop
    (1, 2, 128, (2, 16, 40), 0.75, 0.0),     # 20 blocks
    (2, 3, 128, (3, 10, 50), 0.5, 0.15),     # ragged batch
    (1, 1, 64, (5, 9, 37), 0.8, 0.1),        # odd block count, D = 64
    (3, 2, 128, (1, 7, 9), 0.5, 0.0),        # one partial block
    (1, 2, 128, (4, 16, 64), 0.95, 0.0),     # 64 blocks, keep 4
    (2, 2, 64, (7, 13, 29), 0.3, 0.2),
]


@pytest.mark.parametrize("case", CUSTOM)
def test_custom_shapes(sba, oracle_mod, case):
    B, H, D, grid, s, drop = case
    w = make_custom(B, H, D, grid, s, drop_rate=drop, seed=hash(case) % 1000)
    check_routing(sba, oracle_mod, w)


@pytest.mark.parametrize("s", [0.0, 0.5, 0.75, 0.8, 0.95])
def test_sparsity_sweep(sba, oracle_mod, s):
    w = make_custom(1, 2, 128, (3, 12, 40), s, seed=31, drop_rate=0.05)
    check_routing(sba, oracle_mod, w)


def test_block_means_bit_exact(sba, oracle_mod):
    for case in [(2, 2, 128, (3, 10, 50), 0.15), (1, 3, 64, (5, 9, 37), 0.0)]:
        B, H, D, grid, drop = case
        w = make_custom(B, H, D, grid, 0.5, drop_rate=drop, seed=3)
        q, _, _, vl = to_device(w, DEV)
        m = sba.block_means(q, vl).cpu().numpy()
        ref = oracle_mod.pool(w.q, w.valid_len)
        np.testing.assert_array_equal(m, ref)


def test_block_means_extreme_values(sba, oracle_mod):
    """Block means of random bf16 bit patterns -- every exponent, subnormals, the largest
    finite values, sums that cancel into the subnormal range -- equal the oracle's fp64
    token-order sums bit for bit; blocks holding inf or NaN too (they take the
    conversion-unit path)."""
    rng = np.random.default_rng(7)
    B, H, Np, D = 1, 2, 640, 64
    bits = rng.integers(0, 1 << 16, size=(B, H, Np, D), dtype=np.uint16)
    nonfinite = ((bits >> 7) & 0xFF) == 0xFF
    bits[nonfinite] &= 0x807F              # exponent 0: those become subnormals or zeros
    bits[0, 0, 64 * 3 + 5, 7] = 0x7F80     # +inf in block 3
    bits[0, 1, 64 * 7 + 60, 2] = 0x7FC1    # NaN in block 7
    bits[0, 1, 64 * 8:64 * 9, :] = bits[0, 1, 64 * 8, :]                       # block 8: one row repeated
    bits[0, 1, 64 * 8 + 32:64 * 9, :] = bits[0, 1, 64 * 8, :] ^ 0x8000         # ... then negated: cancels
    x = torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)
    m = sba.block_means(x, None).cpu().numpy()
    ref = oracle_mod.pool(bits, np.array([Np], dtype=np.int32))
    np.testing.assert_array_equal(m, ref)


def test_zero_queries_all_ties(sba, oracle_mod):
    """Every score is 0: the whole row is one tie band; the lowest indices win."""
    w = make_custom(1, 2, 128, (2, 16, 40), 0.7, seed=5)
    w.q = np.zeros_like(w.q)
    check_routing(sba, oracle_mod, w)


def test_integer_inputs_many_exact_ties(sba, oracle_mod):
    rng = np.random.default_rng(17)
    w = make_custom(1, 2, 64, (2, 16, 40), 0.6, seed=6)
    w.q = f64_to_bf16_bits(rng.integers(-1, 2, size=w.q.shape).astype(np.float64))
    w.k = f64_to_bf16_bits(rng.integers(-1, 2, size=w.k.shape).astype(np.float64))
    # make pairs of key blocks identical so whole score columns tie
    w.k[:, :, 64:128] = w.k[:, :, 0:64]
    w.k[:, :, 320:384] = w.k[:, :, 128:192]
    check_routing(sba, oracle_mod, w)


def test_poisoned_padding_changes_nothing(sba, oracle_mod):
    a = make_custom(2, 2, 128, (3, 8, 30), 0.75, seed=29, drop_rate=0.15)
    b = make_custom(2, 2, 128, (3, 8, 30), 0.75, seed=29, drop_rate=0.15, pad_value=1e4)
    qa, ka, _, vla = to_device(a, DEV)
    qb, kb, _, vlb = to_device(b, DEV)
    ia, ca = sba.pool_select(qa, ka, vla, 0.75)
    ib, cb = sba.pool_select(qb, kb, vlb, 0.75)
    assert torch.equal(ca, cb)
    for r in np.ndindex(tuple(ca.shape)):
        c = int(ca[r])
        assert torch.equal(ia[r][:c], ib[r][:c])


def test_max_length(sba, oracle_mod):
    """Npad at the library maximum (4096 blocks), one head."""
    w = make_custom(1, 1, 128, (16, 128, 128), 0.95, seed=41)
    assert w.Npad == sba.sba.MAX_NPAD
    check_routing(sba, oracle_mod, w)


def test_valid_len_one(sba, oracle_mod):
    w = make_custom(2, 2, 128, (2, 8, 40), 0.5, seed=43)
    w.valid_len = np.array([1, 577], dtype=np.int32)
    check_routing(sba, oracle_mod, w)


def test_tie_rows_beside_ordinary_rows(sba, oracle_mod):
    """Rows whose scores are all equal (a zero query block) and rows whose selection
    boundary falls inside a 24-way exact tie (24 identical key blocks: a tie band wider
    than the band cache, decided by the radix fallback) beside ordinary rows in one
    call: every row must match the oracle."""
    rng = np.random.default_rng(23)
    w = make_custom(1, 2, 128, (4, 16, 40), 0.75, seed=24)       # 40 blocks
    q = w.q.copy()
    q[:, :, 64 * 3:64 * 4] = f64_to_bf16_bits(np.zeros((1, 2, 64, 128)))   # block 3: all scores 0
    w.q = q
    k = w.k.copy()
    # 24 identical key blocks: every query block sees a 24-way exact tie, wider than the
    # band cache, wherever the k-th score falls among them
    for J in range(1, 25):
        k[:, 0, 64 * J:64 * (J + 1)] = k[:, 0, 0:64]
    w.k = k
    for s in (0.5, 0.75, 0.9):
        check_routing(sba, oracle_mod, w, s)


def test_wide_windows_fall_back_to_the_row_routine(sba, oracle_mod):
    """Rows with more than 64 blocks inside the fused screen's window: a zero query block
    (every score equal over 120 blocks) and, in head 0, an 81-way exact tie that the
    selection boundary falls into for the rows that rank it high.  Such rows leave the
    fused kernel with their screened scores and finish in the row routine; the ordinary
    rows of the same tiles stay in the fused kernel.  Every row must match the oracle."""
    w = make_custom(1, 2, 128, (4, 30, 64), 0.75, seed=26)       # 120 blocks
    q = w.q.copy()
    q[:, :, 64 * 5:64 * 6] = 0                                      # block 5: all scores 0
    w.q = q
    k = w.k.copy()
    for J in range(1, 81):
        k[:, 0, 64 * J:64 * (J + 1)] = k[:, 0, 0:64]
    w.k = k
    for s in (0.5, 0.75, 0.9):
        check_routing(sba, oracle_mod, w, s)


@pytest.mark.parametrize("n_blocks", [127, 128, 129, 255, 256, 257])
def test_chunk_boundaries(sba, oracle_mod, n_blocks):
    """Block counts just below, at and above one and two 128-block chunks of the fused
    screen (the last chunk partial or full, one or two query tiles per head)."""
    w = make_custom(1, 2, 128, (1, n_blocks, 64), 0.8, seed=50 + n_blocks)
    assert w.Npad // 64 == n_blocks
    check_routing(sba, oracle_mod, w)


def test_d64_several_chunks(sba, oracle_mod):
    """D = 64 (one 64-channel slice per operand tile) over three chunks, ragged."""
    w = make_custom(2, 2, 64, (5, 32, 120), 0.75, seed=61, drop_rate=0.1)
    assert w.Npad // 64 > 256
    check_routing(sba, oracle_mod, w)


def test_short_sample_beside_long_one(sba, oracle_mod):
    """A sample far shorter than the padded length: the range sample strides over the
    padded block count, so few of its 128 sampled blocks lie inside the short sample."""
    w = make_custom(2, 2, 128, (4, 32, 192), 0.75, seed=62)      # 384 blocks
    w.valid_len = np.array([w.Npad, 64 * 23 + 5], dtype=np.int32)  # 24 blocks in sample 1
    check_routing(sba, oracle_mod, w)
