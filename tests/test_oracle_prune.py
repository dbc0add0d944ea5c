"""Pins of the oracle's token pruning by feature-norm saliency (page "Sol Video
Inference Engine", LTX-2.3 appendix, stage 2: keep 50% of the video tokens by
feat_norm).  The oracle ranks tokens by the squared Euclidean norm of their feature
vector (fp64, channel order), keeps the keep_tokens(L, r) = clamp(ceil(r L - 1e-9), 1, L)
largest, equal norms to the lower index, and lists them in their original order.

Pins: a hand-worked example; exact integer norms; brute force over every subset of
tiny problems with many exact ties (the kept set maximises the norm sum and is the
lexicographically smallest maximiser); the kept-count rule's values; ragged samples
equal the sample pruned alone; invariance under exact scaling and sign flips; a
permutation of distinct-norm tokens maps the kept set."""
import itertools

import numpy as np
import pytest

from workloads import f64_to_bf16_bits


def bf(x):
    return f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def test_hand_example(oracle_mod):
    # token features (3,4), (1,1), (0,5), (2,2): squared norms 25, 2, 25, 8
    x = bf([[[3, 4], [1, 1], [0, 5], [2, 2]]])
    for ratio, kept in ((0.25, [0]), (0.5, [0, 2]), (0.75, [0, 2, 3]), (1.0, [0, 1, 2, 3])):
        idx, vout, n2 = oracle_mod.token_prune(x, ratio=ratio, npad_out=4)
        assert vout[0] == len(kept)
        assert idx[0, :len(kept)].tolist() == kept
        assert np.all(idx[0, len(kept):] == -1)
        assert n2[0].tolist() == [25.0, 2.0, 25.0, 8.0]


@pytest.mark.parametrize("n,r,k", [(63240, 0.5, 31620), (53754, 0.5, 26877), (53755, 0.5, 26878),
                                   (10, 0.3, 3), (10, 0.0, 1), (7, 1.0, 7), (1, 0.5, 1), (0, 0.5, 0),
                                   (100, 0.07, 7), (3, 0.999, 3)])
def test_keep_count(oracle_mod, n, r, k):
    assert oracle_mod.keep_tokens(n, r) == k


def test_integer_norms_are_exact(oracle_mod):
    rng = np.random.default_rng(1)
    xi = rng.integers(-40, 41, size=(2, 50, 96))
    _, _, n2 = oracle_mod.token_prune(bf(xi), ratio=0.5)
    np.testing.assert_array_equal(n2, (xi.astype(np.int64) ** 2).sum(axis=2).astype(np.float64))


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_subsets(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    N = 9
    xi = rng.integers(-2, 3, size=(1, N, 3))       # many exact ties among squared norms
    L = int(rng.integers(3, N + 1))
    norms = (xi[0, :L] ** 2).sum(axis=1)
    for ratio in (0.2, 0.45, 0.6, 0.9):
        k = oracle_mod.keep_tokens(L, ratio)
        idx, vout, _ = oracle_mod.token_prune(bf(xi), np.array([L]), ratio=ratio, npad_out=N)
        got = tuple(idx[0, :k].tolist())
        best = max(sum(norms[list(c)]) for c in itertools.combinations(range(L), k))
        maximisers = [c for c in itertools.combinations(range(L), k) if sum(norms[list(c)]) == best]
        assert vout[0] == k
        assert got == min(maximisers), (got, min(maximisers))


def test_ragged_sample_equals_itself_alone(oracle_mod):
    rng = np.random.default_rng(4)
    x = bf(rng.normal(size=(2, 300, 64)))
    vl = np.array([300, 211], dtype=np.int32)
    idx, vout, n2 = oracle_mod.token_prune(x, vl, ratio=0.5)
    assert np.all(n2[1, 211:] == 0.0)
    for b in range(2):
        L = int(vl[b])
        i1, v1, _ = oracle_mod.token_prune(np.ascontiguousarray(x[b:b + 1, :L]), ratio=0.5)
        assert vout[b] == v1[0]
        np.testing.assert_array_equal(idx[b, :vout[b]], i1[0, :v1[0]])
        assert idx[b, :vout[b]].max() < L and np.all(np.diff(idx[b, :vout[b]]) > 0)
        assert np.all(idx[b, vout[b]:] == -1)


def test_scaling_and_sign_do_not_change_the_selection(oracle_mod):
    rng = np.random.default_rng(5)
    xf = rng.normal(size=(1, 200, 32))
    i0, _, _ = oracle_mod.token_prune(bf(xf), ratio=0.4)
    i1, _, _ = oracle_mod.token_prune(bf(2.0 * xf), ratio=0.4)     # exact in bf16
    i2, _, _ = oracle_mod.token_prune(bf(-xf), ratio=0.4)
    np.testing.assert_array_equal(i0, i1)
    np.testing.assert_array_equal(i0, i2)


def test_permutation_maps_the_kept_set(oracle_mod):
    rng = np.random.default_rng(6)
    xf = rng.normal(size=(1, 128, 16))
    perm = rng.permutation(128)
    i0, v0, n0 = oracle_mod.token_prune(bf(xf), ratio=0.3)
    assert len(np.unique(n0)) == 128            # distinct norms: no ties involved
    i1, v1, _ = oracle_mod.token_prune(bf(xf[:, perm]), ratio=0.3)
    # token j of the permuted sequence is token perm[j] of the original
    assert set(perm[i1[0, :v1[0]]].tolist()) == set(i0[0, :v0[0]].tolist())
