"""Pins of the oracle's sub-block log-sum-exp router (CPU only).

The router (page "MiniMax-H3 on 8xH200 benchmark", section "How SubBlock sparse
attention works") estimates each key block's unnormalised softmax mass from pooled
16-token sub-blocks.  The pins use the mass itself, computed by brute force over
tokens, which the oracle never does:
  * tokens constant within each sub-block -> the estimate is exact;
  * any tokens -> the estimate never exceeds the true mass (Jensen: the mean of
    exp over a sub-block pair is at least exp of the mean logit, and the mean logit
    is qbar . kbar);
  * tokens constant within each 64-token block -> the 1x1 router's ranking, offset
    by log(64 * 64) for full blocks.
"""
import math

import numpy as np
import pytest

from workloads import bf16_bits_to_f32, f64_to_bf16_bits, make_custom


def bf(x):
    return f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def true_log_mass(q, k, L, D, blk=64):
    """log sum_{i in I, j in J} exp(q_i . k_j / sqrt(D)) over valid tokens, by brute force."""
    nB = (L + blk - 1) // blk
    s = q[:L] @ k[:L].T / math.sqrt(D)
    out = np.full((nB, nB), np.nan)
    for I in range(nB):
        for J in range(nB):
            blockv = s[I * blk:min((I + 1) * blk, L), J * blk:min((J + 1) * blk, L)]
            m = blockv.max()
            out[I, J] = m + math.log(np.exp(blockv - m).sum())
    return out


def constant_subblocks(rng, N, D, sub=16, scale=1.0):
    vals = rng.normal(size=(N // sub + 1, D)) * scale
    return np.repeat(vals, sub, axis=0)[:N]


@pytest.mark.parametrize("L", [512, 500, 449])
def test_exact_for_subblock_constant_tokens(oracle_mod, L):
    rng = np.random.default_rng(L)
    N, D = 512, 16
    q = bf(constant_subblocks(rng, N, D)[None, None])
    k = bf(constant_subblocks(rng, N, D)[None, None])
    vl = np.array([L], dtype=np.int32)
    _, _, S = oracle_mod.select_lse(q, k, vl, 0.5, return_scores=True)
    ref = true_log_mass(f64(q)[0, 0], f64(k)[0, 0], L, D)
    nB = (L + 63) // 64
    np.testing.assert_allclose(S[0, 0, :nB, :nB], ref, rtol=0, atol=1e-10)


def test_lower_bound_of_true_mass(oracle_mod):
    rng = np.random.default_rng(7)
    N, D, L = 640, 32, 611
    q = bf(rng.normal(size=(1, 1, N, D)))
    k = bf(rng.normal(size=(1, 1, N, D)))
    vl = np.array([L], dtype=np.int32)
    _, _, S = oracle_mod.select_lse(q, k, vl, 0.5, return_scores=True)
    ref = true_log_mass(f64(q)[0, 0], f64(k)[0, 0], L, D)
    nB = (L + 63) // 64
    assert np.all(S[0, 0, :nB, :nB] <= ref + 1e-12)


def test_block_constant_reduces_to_pooled_router(oracle_mod):
    rng = np.random.default_rng(11)
    N, D = 768, 16
    q = bf(constant_subblocks(rng, N, D, sub=64)[None, None])
    k = bf(constant_subblocks(rng, N, D, sub=64)[None, None])
    for s in (0.5, 0.75):
        i1, c1, _, _, S1 = oracle_mod.select(q, k, None, s, return_intermediates=True)
        i4, c4, S4 = oracle_mod.select_lse(q, k, None, s, return_scores=True)
        np.testing.assert_array_equal(c1, c4)
        np.testing.assert_array_equal(i1, i4)
        np.testing.assert_allclose(S4, S1 + math.log(64 * 64), rtol=0, atol=1e-10)


@pytest.mark.parametrize("n,s,budget,expect", [(16, 0.5, 8, 8), (20, 0.75, 8, 8), (20, 0.5, 8, 16),
                                               (5, 0.5, 8, 5), (1182, 0.8, 8, 240), (512, 0.75, 8, 128)])
def test_budget_rounding(oracle_mod, n, s, budget, expect):
    assert oracle_mod.keep_count_budget(n, s, budget) == expect


def test_zero_queries_tie_to_lower_index(oracle_mod):
    w = make_custom(1, 1, 32, (2, 8, 40), 0.7, seed=3)
    q = bf(np.zeros(w.q.shape))
    idx, cnt = oracle_mod.select_lse(q, w.k, None, 0.7)
    assert np.all(cnt == 3) and np.all(idx[..., :3] == np.array([0, 1, 2]))


def test_budget_nesting_and_kept_counts(oracle_mod):
    w = make_custom(2, 2, 32, (3, 8, 30), 0.75, seed=5, drop_rate=0.15)
    i1, c1 = oracle_mod.select_lse(w.q, w.k, w.valid_len, 0.75)
    i8, c8 = oracle_mod.select_lse(w.q, w.k, w.valid_len, 0.75, budget=8)
    for b in range(2):
        nB = (int(w.valid_len[b]) + 63) // 64
        assert np.all(c8[b, :, :nB] == oracle_mod.keep_count_budget(nB, 0.75, 8))
        for h in range(2):
            for I in range(nB):
                assert set(i1[b, h, I, :c1[b, h, I]]) <= set(i8[b, h, I, :c8[b, h, I]])
