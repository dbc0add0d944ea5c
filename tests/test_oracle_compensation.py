"""Pins of the oracle's compensated block-sparse attention (page "Sol Video Inference
Engine", section 4.2.2: PISA computes the critical blocks exactly and compensates the
others by a first-order Taylor approximation).  Each dropped block J is expanded about
its mean key: the normaliser gets c_J e^{s q.kbar_J}; the numerator gets
e^{s q.kbar_J} (c_J vbar_J + s q^T M_J) with M_J = sum_j (k_j - kbar_J) v_j^T
(order 1), or the first part alone (order 0, the mean-key form).

The pins rest on dense attention (pinned on its own in test_oracle.py) and on what the
expansion fixes:
  * the error against dense attention shrinks as the square of the keys' spread about
    their block means for order 1, and only linearly for order 0 -- a dropped,
    mis-signed, unscaled or transposed moment term leaves a linear error and fails;
  * keys constant within every block -> the expansion is exact (both orders), so the
    output equals dense attention whatever the routing and whatever the values;
  * values constant within every block -> the moment vanishes and both orders agree;
  * nothing dropped -> plain sparse attention;
  * V constant -> the output is that constant;
  * compensation only adds mass: lse_compensated >= lse_sparse.
"""
import numpy as np
import pytest

from workloads import f64_to_bf16_bits, make_custom


def bf(x):
    return f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def bf_to_f64(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def blockwise_constant(rng, B, H, N, D, block=64, scale=1.0):
    vals = rng.normal(size=(B, H, N // block + 1, D)) * scale
    return bf(np.repeat(vals, block, axis=2)[:, :, :N])


def random_routing(rng, nB, keep, B=1, H=1):
    idx = np.full((B, H, nB, keep), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for I in range(nB):
                idx[b, h, I] = np.sort(rng.choice(nB, keep, replace=False))
    return idx, np.full((B, H, nB), keep, dtype=np.int32)


ORDERS = [0, 1]


@pytest.mark.parametrize("order", ORDERS)
@pytest.mark.parametrize("L", [640, 611, 577])
def test_block_constant_keys_and_values_give_dense(oracle_mod, L, order):
    rng = np.random.default_rng(L)
    B, H, N, D = 1, 2, 640, 32
    q = bf(rng.normal(size=(B, H, N, D)))
    k = blockwise_constant(rng, B, H, N, D)
    v = blockwise_constant(rng, B, H, N, D)
    vl = np.array([L], dtype=np.int32)
    for s in (0.5, 0.8):
        idx, cnt = oracle_mod.select(q, k, vl, s)
        o_c, lse_c = oracle_mod.attention_compensated(q, k, v, idx, cnt, vl, order=order)
        o_d, lse_d = oracle_mod.dense(q, k, v, vl)
        rows = np.arange(N) < L
        np.testing.assert_allclose(o_c[:, :, rows], o_d[:, :, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse_c[:, :, rows], lse_d[:, :, rows], rtol=0, atol=1e-12)


@pytest.mark.parametrize("order", ORDERS)
def test_block_constant_keys_exact_for_any_values_and_routing(oracle_mod, order):
    """Keys constant within blocks, values arbitrary: the first-order moment is zero and
    the zeroth-order sum is exact, whichever blocks the routing kept."""
    rng = np.random.default_rng(3)
    B, H, N, D = 1, 1, 512, 16
    q = bf(rng.normal(size=(B, H, N, D)))
    k = blockwise_constant(rng, B, H, N, D)
    v = bf(rng.normal(size=(B, H, N, D)))
    idx, cnt = random_routing(rng, 8, 3)
    o_c, _ = oracle_mod.attention_compensated(q, k, v, idx, cnt, order=order)
    o_d, _ = oracle_mod.dense(q, k, v)
    np.testing.assert_allclose(o_c, o_d, rtol=0, atol=1e-12)


def test_block_constant_values_make_the_moment_vanish(oracle_mod):
    """sum_j (k_j - kbar) v^T = 0 when v is constant within the block: both orders agree."""
    rng = np.random.default_rng(4)
    B, H, N, D = 1, 2, 448, 16
    q = bf(rng.normal(size=(B, H, N, D)))
    k = bf(rng.normal(size=(B, H, N, D)))
    v = blockwise_constant(rng, B, H, N, D)
    vl = np.array([431], dtype=np.int32)
    idx, cnt = oracle_mod.select(q, k, vl, 0.7)
    o1, l1 = oracle_mod.attention_compensated(q, k, v, idx, cnt, vl, order=1)
    o0, l0 = oracle_mod.attention_compensated(q, k, v, idx, cnt, vl, order=0)
    rows = np.arange(N) < 431
    np.testing.assert_allclose(o1[:, :, rows], o0[:, :, rows], rtol=0, atol=1e-13)
    np.testing.assert_array_equal(l1, l0)


def spread_problem(L, eps, seed=21, N=512, D=16, block=64):
    """Keys k_j = kbar_J + eps * u_j with u_j = +-1 per channel, balanced within every
    block's valid tokens (sum_j u_j = 0 exactly); kbar on a 1/4 grid in [-1.5, 1.5] so
    that every key is exactly a bf16 value for eps >= 2^-6.  Q and V are fixed bf16
    draws, the routing a fixed random one."""
    rng = np.random.default_rng(seed)
    nB = N // block
    q = bf(0.5 * rng.normal(size=(1, 1, N, D)))
    v = bf(rng.normal(size=(1, 1, N, D)))
    kbar = rng.integers(-6, 7, size=(nB, D)) * 0.25
    u = np.zeros((N, D))
    for J in range(nB):
        c = min(block, L - J * block)
        if c <= 0:
            break
        for d in range(D):
            s = np.array([1.0] * (c // 2) + [-1.0] * (c // 2) + [0.0] * (c % 2))
            u[J * block:J * block + c, d] = rng.permutation(s)
    kf = np.repeat(kbar, block, axis=0)[:N] + eps * u
    k = bf(kf[None, None])
    assert np.array_equal(bf_to_f64(k), kf[None, None]), "keys must be exact bf16 values"
    idx, cnt = random_routing(np.random.default_rng(seed + 1), nB, 2)
    vl = np.array([L], dtype=np.int32)
    return q, k, v, idx, cnt, vl


@pytest.mark.parametrize("L", [512, 480])
def test_error_shrinks_quadratically_with_the_key_spread(oracle_mod, L):
    """Halving the spread of the keys about their block means divides the error against
    dense attention by about 4 for the first-order form and about 2 for the mean-key
    form: the moment term is what removes the linear error."""
    errs = {0: [], 1: []}
    eps_list = [2.0 ** -3, 2.0 ** -4, 2.0 ** -5, 2.0 ** -6]
    for eps in eps_list:
        q, k, v, idx, cnt, vl = spread_problem(L, eps)
        o_d, _ = oracle_mod.dense(q, k, v, vl)
        rows = np.arange(q.shape[2]) < L
        for order in (0, 1):
            o_c, _ = oracle_mod.attention_compensated(q, k, v, idx, cnt, vl, order=order)
            errs[order].append(np.abs(o_c - o_d)[:, :, rows].max())
    r1 = [errs[1][i] / errs[1][i + 1] for i in range(3)]
    r0 = [errs[0][i] / errs[0][i + 1] for i in range(3)]
    assert all(3.5 <= r <= 4.5 for r in r1), (r1, errs[1])
    assert all(1.7 <= r <= 2.3 for r in r0), (r0, errs[0])
    assert all(e1 < e0 for e1, e0 in zip(errs[1], errs[0]))


@pytest.mark.parametrize("order", ORDERS)
def test_nothing_dropped_is_plain_sparse(oracle_mod, order):
    w = make_custom(1, 2, 64, (2, 8, 16), 0.0, seed=5, drop_rate=0.1)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.0)
    o1, l1 = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    o2, l2 = oracle_mod.attention_compensated(w.q, w.k, w.v, idx, cnt, w.valid_len, order=order)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    np.testing.assert_array_equal(l1, l2)


@pytest.mark.parametrize("order", ORDERS)
def test_constant_values_give_that_value(oracle_mod, order):
    w = make_custom(1, 1, 64, (2, 8, 16), 0.75, seed=7)
    v = np.full_like(w.v, bf(np.array([0.8125]))[0])
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.75)
    o, _ = oracle_mod.attention_compensated(w.q, w.k, v, idx, cnt, w.valid_len, order=order)
    np.testing.assert_allclose(o, 0.8125, rtol=0, atol=1e-12)


@pytest.mark.parametrize("order", ORDERS)
def test_compensation_only_adds_mass(oracle_mod, order):
    w = make_custom(2, 2, 64, (3, 8, 16), 0.8, seed=9, drop_rate=0.15)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.8)
    _, l1 = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    _, l2 = oracle_mod.attention_compensated(w.q, w.k, w.v, idx, cnt, w.valid_len, order=order)
    fin = np.isfinite(l1)
    assert np.array_equal(fin, np.isfinite(l2))
    assert np.all(l2[fin] >= l1[fin])
    assert np.any(l2[fin] > l1[fin] + 1e-9)


def test_both_orders_share_the_normaliser(oracle_mod):
    """The moment term enters the numerator only: lse is the same for both orders."""
    w = make_custom(1, 2, 64, (3, 8, 16), 0.8, seed=13, drop_rate=0.1)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.8)
    _, l0 = oracle_mod.attention_compensated(w.q, w.k, w.v, idx, cnt, w.valid_len, order=0)
    _, l1 = oracle_mod.attention_compensated(w.q, w.k, w.v, idx, cnt, w.valid_len, order=1)
    np.testing.assert_array_equal(l0, l1)


def test_bad_order_is_rejected(oracle_mod):
    w = make_custom(1, 1, 64, (1, 8, 8), 0.5, seed=1)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.5)
    with pytest.raises(ValueError):
        oracle_mod.attention_compensated(w.q, w.k, w.v, idx, cnt, w.valid_len, order=2)
