"""Pins of the fp64 oracle against what the definition and mathematics fix (CPU only).

The router and the sparse attention follow the page "MiniMax-H3 on 8xH200 benchmark"
(news.paixiangai.cn), section "How SubBlock sparse attention works": block pooling and
scoring, top-scoring key blocks kept per query block and head (`sparsity` = fraction
dropped), exact attention over the kept blocks only.  Each pin below is independent of
the oracle's own code: hand-worked values, closed forms, brute-force enumeration,
a second (numpy, full-matrix) attention, and invariants of softmax attention.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

from workloads import f64_to_bf16_bits, bf16_bits_to_f32, make_custom

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf(x):
    """float array -> bf16 bits [B,H,N,D] (values must be bf16-representable for exact pins)."""
    return f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def f64(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def numpy_attention(q, k, v, allowed, scale):
    """Independent full-matrix attention: logits outside `allowed` are -inf."""
    s = scale * (q @ k.T)
    s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.where(allowed, np.exp(s - m), 0.0)
    return (e @ v) / e.sum(axis=1, keepdims=True)


def rand_int_inputs(rng, B, H, N, D, lo=-3, hi=3):
    return bf(rng.integers(lo, hi + 1, size=(B, H, N, D)))


# ----------------------------------------------------------------------------- keep count

@pytest.mark.parametrize("n,s,expect", [
    (16, 0.5, 8), (512, 0.0, 512), (512, 0.75, 128), (1182, 0.80, 237),
    (10, 0.7, 3), (3, 0.5, 2), (3, 0.7, 1), (1, 0.99, 1), (7, 0.0, 7), (100, 0.999, 1),
])
def test_keep_count_values(oracle_mod, n, s, expect):
    # ceil((1-s)*n) worked by hand; (1-0.7)*10 is 3.0000000000000004 in fp64
    assert oracle_mod.keep_count(n, s) == expect


# ----------------------------------------------------------------------------- hand example

def test_hand_example(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "hand_example.json")))
    blk, D = g["block"], g["D"]
    q = bf(np.array(g["q"], dtype=np.float64)[None, None])
    k = bf(np.array(g["k"], dtype=np.float64)[None, None])
    for case in g["cases"]:
        vl = np.array([case["valid_len"]], dtype=np.int32)
        pq = oracle_mod.pool(q, vl, blk)[0, 0]
        pk = oracle_mod.pool(k, vl, blk)[0, 0]
        np.testing.assert_array_equal(pq, np.array(case["pooled_q"], dtype=np.float64))
        np.testing.assert_array_equal(pk, np.array(case["pooled_k"], dtype=np.float64))
        S = oracle_mod.scores(pq[None, None], pk[None, None], vl, blk)[0, 0]
        np.testing.assert_allclose(S * math.sqrt(D), np.array(case["dots"], dtype=np.float64),
                                   rtol=1e-15, atol=0)
        for s, mask in case["masks"].items():
            idx, cnt = oracle_mod.select(q, k, vl, float(s), block=blk)
            for I, want in enumerate(mask):
                assert list(idx[0, 0, I, :cnt[0, 0, I]]) == want
    t = g["ties"]
    vl = np.array([t["valid_len"]], dtype=np.int32)
    for s, mask in t["masks"].items():
        idx, cnt = oracle_mod.select(np.zeros_like(q), k, vl, float(s), block=blk)
        for I, want in enumerate(mask):
            assert list(idx[0, 0, I, :cnt[0, 0, I]]) == want


# ----------------------------------------------------------------------------- pooling

def test_pool_closed_forms(oracle_mod):
    B, H, N, D, blk = 1, 2, 256, 4, 64
    x = np.zeros((B, H, N, D))
    x[0, 0, :, 0] = 3.0                         # constant block -> that constant
    n = np.arange(N, dtype=np.float64)
    x[0, 0, :, 1] = -2.0 + 0.5 * n              # affine a + b*n -> a + b*mean(n)
    x[0, 1, :, 2] = n % 7                       # small integers -> exact mean
    bits = bf(x)
    for L in (256, 200, 193):
        vl = np.array([L], dtype=np.int32)
        p = oracle_mod.pool(bits, vl, blk)
        for I in range(4):
            n0, n1 = I * blk, min((I + 1) * blk, L)
            if n1 <= n0:
                assert np.all(p[0, :, I] == 0.0)
                continue
            assert p[0, 0, I, 0] == 3.0
            assert p[0, 0, I, 1] == -2.0 + 0.5 * (n0 + n1 - 1) / 2.0
            assert p[0, 1, I, 2] == np.sum(np.arange(n0, n1) % 7) / (n1 - n0)


# ----------------------------------------------------------------------------- scores

def test_scores_exact_small_integers(oracle_mod):
    rng = np.random.default_rng(5)
    B, H, N, D, blk = 1, 2, 8 * 4, 4, 4
    q = rand_int_inputs(rng, B, H, N, D)
    k = rand_int_inputs(rng, B, H, N, D)
    vl = np.array([N], dtype=np.int32)
    _, _, pq, pk, S = oracle_mod.select(q, k, vl, 0.5, block=blk, return_intermediates=True)
    qq, kk = f64(q), f64(k)
    for h in range(H):
        for I in range(8):
            for J in range(8):
                # integer sums, divided by the power-of-two block size: exact in fp64
                sq = qq[0, h, I * blk:(I + 1) * blk].sum(axis=0)
                sk = kk[0, h, J * blk:(J + 1) * blk].sum(axis=0)
                dot = float(np.dot(sq, sk)) / (blk * blk)
                assert S[0, h, I, J] * math.sqrt(D) == pytest.approx(dot, rel=1e-15, abs=1e-15)


# ----------------------------------------------------------------------------- top-k routing

def test_topk_brute_force_with_ties(oracle_mod):
    """Over every size-k subset: the kept set maximises the summed score and, among the
    maximisers, is the lexicographically smallest sorted index tuple (lower index wins)."""
    rng = np.random.default_rng(11)
    for trial in range(40):
        nB = int(rng.integers(2, 9))
        blk = int(rng.choice([1, 2, 4]))   # power-of-two means: exact fp64 scores
        D = int(rng.integers(1, 5))
        N = nB * blk
        q = rand_int_inputs(rng, 1, 1, N, D, -1, 1)     # tiny integer range: many exact ties
        k = rand_int_inputs(rng, 1, 1, N, D, -1, 1)
        vl = np.array([N], dtype=np.int32)
        s = float(rng.choice([0.0, 0.3, 0.5, 0.75, 0.9]))
        idx, cnt, _, _, S = oracle_mod.select(q, k, vl, s, block=blk, return_intermediates=True)
        kk = max(1, min(nB, math.ceil((1 - s) * nB - 1e-9)))
        for I in range(nB):
            row = S[0, 0, I]
            best = None
            for sub in itertools.combinations(range(nB), kk):
                tot = sum(row[j] for j in sub)
                if best is None or tot > best[0] + 1e-12 or (abs(tot - best[0]) <= 1e-12 and sub < best[1]):
                    best = (tot, sub)
            assert cnt[0, 0, I] == kk
            assert tuple(idx[0, 0, I, :kk]) == best[1], (trial, I, row)


def test_topk_zero_queries_keep_first_blocks(oracle_mod):
    rng = np.random.default_rng(3)
    q = bf(np.zeros((1, 2, 640, 8)))
    k = rand_int_inputs(rng, 1, 2, 640, 8)
    idx, cnt = oracle_mod.select(q, k, None, 0.7)
    assert np.all(cnt == 3)
    assert np.all(idx[..., :3] == np.array([0, 1, 2]))


def test_topk_nesting_and_dense(oracle_mod):
    w = make_custom(1, 2, 16, (2, 8, 40), 0.5, seed=7)     # 640 tokens, 10 blocks
    prev = None
    for s in (0.9, 0.75, 0.5, 0.3, 0.0):
        idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, s)
        sets = [[set(idx[0, h, I, :cnt[0, h, I]]) for I in range(10)] for h in range(2)]
        if prev is not None:
            for h in range(2):
                for I in range(10):
                    assert prev[h][I] <= sets[h][I]
        prev = sets
    assert all(s == set(range(10)) for hs in prev for s in hs)


def test_topk_key_shift_invariance(oracle_mod):
    """Adding one vector c to every key shifts each score row by a constant."""
    rng = np.random.default_rng(9)
    q = rand_int_inputs(rng, 1, 2, 512, 8)
    k = rng.integers(-3, 4, size=(1, 2, 512, 8)).astype(np.float64)
    c = rng.integers(-2, 3, size=(8,)).astype(np.float64)
    for s in (0.5, 0.75):
        a = oracle_mod.select(q, bf(k), None, s)
        b = oracle_mod.select(q, bf(k + c), None, s)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


# ----------------------------------------------------------------------------- attention

def _allowed_matrix(idx, cnt, b, h, L, Npad, blk):
    """[Npad, Npad] boolean: query row i may see key j (kept block of i's block, j < L)."""
    A = np.zeros((Npad, Npad), dtype=bool)
    for I in range(Npad // blk):
        for J in idx[b, h, I, :cnt[b, h, I]]:
            A[I * blk:(I + 1) * blk, J * blk:min((J + 1) * blk, L)] = True
    A[L:, :] = False
    return A


def test_dense_equals_numpy_full_matrix(oracle_mod):
    w = make_custom(2, 2, 32, (2, 6, 30), 0.0, seed=3, drop_rate=0.1)
    o, lse = oracle_mod.dense(w.q, w.k, w.v, w.valid_len)
    q, k, v = f64(w.q), f64(w.k), f64(w.v)
    for b in range(2):
        L = int(w.valid_len[b])
        for h in range(2):
            allowed = np.ones((L, L), dtype=bool)
            ref = numpy_attention(q[b, h, :L], k[b, h, :L], v[b, h, :L], allowed, 1 / math.sqrt(32))
            np.testing.assert_allclose(o[b, h, :L], ref, rtol=0, atol=1e-12)
            s = q[b, h, :L] @ k[b, h, :L].T / math.sqrt(32)
            ref_lse = s.max(1) + np.log(np.exp(s - s.max(1, keepdims=True)).sum(1))
            np.testing.assert_allclose(lse[b, h, :L], ref_lse, rtol=0, atol=1e-12)
            assert np.all(o[b, h, L:] == 0.0) and np.all(np.isneginf(lse[b, h, L:]))


def test_sparse_s0_equals_dense(oracle_mod):
    w = make_custom(1, 2, 64, (2, 8, 36), 0.0, seed=4)          # 576 tokens
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.0)
    o, lse = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    od, lsed = oracle_mod.dense(w.q, w.k, w.v, w.valid_len)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lsed, rtol=0, atol=1e-12)


def test_sparse_equals_masked_dense_random_routings(oracle_mod):
    """Gather form == full-matrix attention with -inf logits outside the kept blocks, for
    every size-k subset of a tiny problem (and its ragged version)."""
    rng = np.random.default_rng(21)
    blk, nB, D = 4, 5, 3
    N = blk * nB
    q = bf(rng.normal(size=(1, 1, N, D)))
    k = bf(rng.normal(size=(1, 1, N, D)))
    v = bf(rng.normal(size=(1, 1, N, D)))
    qq, kk, vv = f64(q)[0, 0], f64(k)[0, 0], f64(v)[0, 0]
    for L in (N, N - 3):
        vl = np.array([L], dtype=np.int32)
        nBL = (L + blk - 1) // blk
        for kk_ in (1, 2, nBL):
            for sub in itertools.combinations(range(nBL), kk_):
                idx = np.full((1, 1, nB, kk_), -1, dtype=np.int32)
                cnt = np.zeros((1, 1, nB), dtype=np.int32)
                for I in range(nBL):
                    idx[0, 0, I] = sub
                    cnt[0, 0, I] = kk_
                o, lse = oracle_mod.attention(q, k, v, idx, cnt, vl, block=blk)
                A = _allowed_matrix(idx, cnt, 0, 0, L, N, blk)[:L]
                ref = numpy_attention(qq[:L], kk, vv, A, 1 / math.sqrt(D))
                np.testing.assert_allclose(o[0, 0, :L], ref, rtol=0, atol=1e-13)


def test_probability_rows_sum_to_one(oracle_mod):
    w = make_custom(1, 1, 32, (2, 8, 24), 0.6, seed=8, drop_rate=0.05)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.6)
    L = int(w.valid_len[0])
    for i in (0, 1, 63, 64, 200, L - 1):
        p = oracle_mod.probs(w.q, w.k, w.v, idx, cnt, 0, 0, i, w.valid_len)
        assert abs(p.sum() - 1.0) < 1e-12
        assert np.all(p >= 0) and np.all(p[L:] == 0)
        kept = set(idx[0, 0, i // 64, :cnt[0, 0, i // 64]])
        outside = [j for j in range(L) if j // 64 not in kept]
        assert np.all(p[outside] == 0)


def test_constant_v_gives_constant(oracle_mod):
    w = make_custom(1, 2, 64, (2, 8, 32), 0.75, seed=12)
    v = bf(np.full(w.v.shape, 1.5))
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.75)
    o, _ = oracle_mod.attention(w.q, w.k, v, idx, cnt, w.valid_len)
    np.testing.assert_allclose(o, 1.5, rtol=0, atol=1e-13)


def test_permutation_inside_blocks(oracle_mod):
    w = make_custom(1, 1, 32, (2, 8, 32), 0.5, seed=13)      # 512 tokens, 8 blocks
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.5)
    o, lse = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    rng = np.random.default_rng(0)
    # permute K and V together inside kept key block J0 of row 0: outputs unchanged
    J0 = int(idx[0, 0, 0, 0])
    perm = np.arange(512)
    perm[J0 * 64:(J0 + 1) * 64] = J0 * 64 + rng.permutation(64)
    o2, lse2 = oracle_mod.attention(w.q, w.k[:, :, perm], w.v[:, :, perm], idx, cnt, w.valid_len)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)
    # permute queries inside query block 3 (routing recomputed: pooled means are
    # order-independent, so it is unchanged): outputs permute the same way
    pq = np.arange(512)
    pq[192:256] = 192 + rng.permutation(64)
    idx3, cnt3 = oracle_mod.select(w.q[:, :, pq], w.k, w.valid_len, 0.5)
    np.testing.assert_array_equal(idx3, idx)
    o3, _ = oracle_mod.attention(w.q[:, :, pq], w.k, w.v, idx3, cnt3, w.valid_len)
    np.testing.assert_allclose(o3, o[:, :, pq], rtol=0, atol=1e-13)


def test_key_shift_leaves_outputs(oracle_mod):
    rng = np.random.default_rng(17)
    q = rand_int_inputs(rng, 1, 1, 384, 8, -2, 2)
    kf = rng.integers(-2, 3, size=(1, 1, 384, 8)).astype(np.float64)
    v = bf(rng.normal(size=(1, 1, 384, 8)))
    c = rng.integers(-1, 2, size=(8,)).astype(np.float64)
    a = oracle_mod.select(q, bf(kf), None, 0.5)
    b = oracle_mod.select(q, bf(kf + c), None, 0.5)
    np.testing.assert_array_equal(a[0], b[0])
    o1, _ = oracle_mod.attention(q, bf(kf), v, *a)
    o2, _ = oracle_mod.attention(q, bf(kf + c), v, *b)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-12)


def test_zero_queries_average_first_blocks(oracle_mod):
    w = make_custom(1, 1, 16, (2, 8, 40), 0.7, seed=19, drop_rate=0.1)
    q = bf(np.zeros(w.q.shape))
    idx, cnt = oracle_mod.select(q, w.k, w.valid_len, 0.7)
    o, _ = oracle_mod.attention(q, w.k, w.v, idx, cnt, w.valid_len)
    L = int(w.valid_len[0])
    nB = (L + 63) // 64
    kk = max(1, math.ceil(0.3 * nB - 1e-9))
    ref = f64(w.v)[0, 0, :min(kk * 64, L)].mean(axis=0)
    np.testing.assert_allclose(o[0, 0, :L], np.broadcast_to(ref, (L, 16)), rtol=0, atol=1e-13)


def test_block_size_one_dense(oracle_mod):
    w = make_custom(1, 1, 8, (1, 4, 16), 0.0, seed=23)
    idx, cnt = oracle_mod.select(w.q, w.k, None, 0.0, block=1)
    o, _ = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, None, block=1)
    od, _ = oracle_mod.dense(w.q, w.k, w.v, None)
    np.testing.assert_allclose(o, od, rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- ragged

def test_ragged_padding_and_batch_independence(oracle_mod):
    w = make_custom(2, 2, 32, (3, 8, 30), 0.75, seed=29, drop_rate=0.15)
    wp = make_custom(2, 2, 32, (3, 8, 30), 0.75, seed=29, drop_rate=0.15, pad_value=1e4)
    idx, cnt = oracle_mod.select(w.q, w.k, w.valid_len, 0.75)
    idxp, cntp = oracle_mod.select(wp.q, wp.k, wp.valid_len, 0.75)
    np.testing.assert_array_equal(cnt, cntp)
    np.testing.assert_array_equal(idx, idxp)
    o, lse = oracle_mod.attention(w.q, w.k, w.v, idx, cnt, w.valid_len)
    op, lsep = oracle_mod.attention(wp.q, wp.k, wp.v, idx, cnt, wp.valid_len)
    np.testing.assert_array_equal(o, op)
    np.testing.assert_array_equal(lse, lsep)
    for b in range(2):
        L = int(w.valid_len[b])
        Np = 64 * ((L + 63) // 64)
        sl = lambda x: np.ascontiguousarray(x[b:b + 1, :, :Np])
        vl = np.array([L], dtype=np.int32)
        i1, c1 = oracle_mod.select(sl(w.q), sl(w.k), vl, 0.75)
        nB = Np // 64
        np.testing.assert_array_equal(c1[0], cnt[b, :, :nB])
        for h in range(2):
            for I in range(nB):
                assert list(i1[0, h, I, :c1[0, h, I]]) == list(idx[b, h, I, :cnt[b, h, I]])
        o1, _ = oracle_mod.attention(sl(w.q), sl(w.k), sl(w.v), i1, c1, vl)
        np.testing.assert_array_equal(o1[0], o[b, :, :Np])
    # valid_len == Npad is the unpadded problem
    full = np.full(2, w.Npad, dtype=np.int32)
    a = oracle_mod.select(w.q, w.k, full, 0.5)
    b2 = oracle_mod.select(w.q, w.k, None, 0.5)
    np.testing.assert_array_equal(a[0], b2[0])
