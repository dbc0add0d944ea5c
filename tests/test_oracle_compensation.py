"""Pins of the oracle's compensated block-sparse attention (each dropped block enters
the softmax as one entry: logit s q.kbar_J + log c_J carrying vbar_J; the first-order
expansion of the dropped blocks' exponentials about their mean key, page "Sol Video
Inference Engine", section 4.2.2, PISA).  The pins rest on dense attention (pinned
on its own in test_oracle.py) and on closed forms:
  * keys and values constant within every block -> the expansion is exact, so the
    compensated output equals dense attention, whatever the routing;
  * nothing dropped -> plain sparse attention;
  * V constant -> the output is that constant;
  * compensation only adds mass: lse_compensated >= lse_sparse.
"""
import numpy as np
import pytest

from workloads import f64_to_bf16_bits, make_custom


def bf(x):
    return f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def blockwise_constant(rng, B, H, N, D, block=64, scale=1.0):
    vals = rng.normal(size=(B, H, N // block + 1, D)) * scale
    return bf(np.repeat(vals, block, axis=2)[:, :, :N])


@pytest.mark.parametrize("L", [640, 611, 577])
def test_block_constant_keys_and_values_give_dense(oracle_mod, L):
    rng = np.random.default_rng(L)
    B, H, N, D = 1, 2, 640, 32
    q = bf(rng.normal(size=(B, H, N, D)))
    k = blockwise_constant(rng, B, H, N, D)
    v = blockwise_constant(rng, B, H, N, D)
    vl = np.array([L], dtype=np.int32)
    for s in (0.5, 0.8):
        idx, cnt = oracle_mod.select(q, k, vl, s)
        o_c, lse_c = oracle_mod.attention_compensated(q, k, v, idx, cnt, vl)
        o_d, lse_d = oracle_mod.dense(q, k, v, vl)
        rows = np.arange(N) < L
        np.testing.assert_allclose(o_c[:, :, rows], o_d[:, :, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse_c[:, :, rows], lse_d[:, :, rows], rtol=0, atol=1e-12)


def test_random_routing_also_exact_for_block_constant_inputs(oracle_mod):
    """The equality does not depend on which blocks the router kept."""
    rng = np.random.default_rng(3)
    B, H, N, D = 1, 1, 512, 16
    q = bf(rng.normal(size=(B, H, N, D)))
    k = blockwise_constant(rng, B, H, N, D)
    v = blockwise_constant(rng, B, H, N, D)
    nB, kmax = 8, 3
    idx = np.full((B, H, nB, kmax), -1, dtype=np.int32)
    for I in range(nB):
        idx[0, 0, I] = np.sort(rng.choice(nB, kmax, replace=False))
    cnt = np.full((B, H, nB), kmax, dtype=np.int32)
    o_c, _ = oracle_mod.attention_compensated(q, k, v, idx, cnt)
    o_d, _ = oracle_mod.dense(q, k, v)
    np.testing.assert_allclose(o_c, o_d, rtol=0, atol=1e-12)


def test_nothing_dropped_is_plain_sparse(oracle_mod):
    w = make_custom(1, 2, 64, (2, 8, 16), 0.0, seed=5, drop_rate=0.1)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.0)
    o1, l1 = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    o2, l2 = oracle_mod.attention_compensated(w.q, w.k, w.v, idx, cnt, w.valid_len)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_constant_values_give_that_value(oracle_mod):
    w = make_custom(1, 1, 64, (2, 8, 16), 0.75, seed=7)
    v = np.full_like(w.v, bf(np.array([0.8125]))[0])
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.75)
    o, _ = oracle_mod.attention_compensated(w.q, w.k, v, idx, cnt, w.valid_len)
    np.testing.assert_allclose(o, 0.8125, rtol=0, atol=1e-12)


def test_compensation_only_adds_mass(oracle_mod):
    w = make_custom(2, 2, 64, (3, 8, 16), 0.8, seed=9, drop_rate=0.15)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.8)
    _, l1 = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    _, l2 = oracle_mod.attention_compensated(w.q, w.k, w.v, idx, cnt, w.valid_len)
    fin = np.isfinite(l1)
    assert np.array_equal(fin, np.isfinite(l2))
    assert np.all(l2[fin] >= l1[fin])
    assert np.any(l2[fin] > l1[fin] + 1e-9)


def test_values_varying_within_blocks_stay_within_rounding(oracle_mod):
    """Keys block-constant, values not: the only error left is the bf16 rounding of the
    dropped blocks' value means (at most 2^-9 relative, times their total weight)."""
    rng = np.random.default_rng(11)
    B, H, N, D = 1, 1, 640, 32
    q = bf(rng.normal(size=(B, H, N, D)))
    k = blockwise_constant(rng, B, H, N, D)
    v = bf(rng.normal(size=(B, H, N, D)))
    idx, cnt = oracle_mod.select(q, k, None, 0.8)
    o_c, _ = oracle_mod.attention_compensated(q, k, v, idx, cnt)
    o_d, _ = oracle_mod.dense(q, k, v)
    vmax = np.abs(oracle_mod.pool(v)).max()
    assert np.abs(o_c - o_d).max() <= 2.0 ** -9 * vmax + 1e-12
