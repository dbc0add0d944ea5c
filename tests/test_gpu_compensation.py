"""GPU compensated block-sparse attention against the fp64 oracle, under the GPU's own
routing (page "Sol Video Inference Engine", section 4.2.2: PISA computes the critical
blocks exactly and compensates the others by a first-order Taylor approximation).

  sba_attention_compensated        the first-order expansion of each dropped block about
                                   its mean key (oracle order 1); the kernel evaluates it
                                   token by token, the oracle through the D x D moment
  sba_attention_mean_compensated   the zeroth-order, mean-key form (oracle order 0)

Outputs: the plain path's tolerances (max-abs 2e-2, mean-abs 2e-3).  LSE: 1e-4 for the
first-order call.  The mean-key call stores the block means in bf16 (2^-9 relative),
which moves a dropped block's logit by at most s * sum_d |q_d| max_J |kbar_Jd| * 2^-9, so
its LSE tolerance per row is that bound plus 1e-4 (the log-sum-exp moves by no more
than the largest logit change)."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, output_errors, to_device
from workloads import bf16_bits_to_f32, f64_to_bf16_bits, make_custom, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def mean_lse_bound(oracle_mod, q, k, valid_len):
    """Per-row LSE tolerance of the mean-key call (see the module docstring)."""
    D = q.shape[3]
    km = np.abs(oracle_mod.pool(k, valid_len)).max(axis=2)                 # [B, H, D]
    qa = np.abs(bf16_bits_to_f32(q).astype(np.float64))                    # [B, H, Npad, D]
    return np.einsum("bhnd,bhd->bhn", qa, km) / np.sqrt(D) * 2.0 ** -9 + 1e-4


def run(sba, oracle_mod, w, s, order, paired=True, qblocks=None, heads=None):
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, s)
    po = sba.pair_query_blocks(idx, cnt, vl) if paired else None
    if order == 1:
        o, lse = sba.attention_compensated(q, k, v, idx, cnt, vl, pair_order=po)
    else:
        o, lse = sba.attention_mean_compensated(q, k, v, idx, cnt, vl, pair_order=po)
    assert sba.device_status() == 0
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for h in (heads if heads is not None else [None]):
        sl = (lambda x: x) if h is None else (lambda x: np.ascontiguousarray(x[:, h:h + 1]))
        wq, wk, wv = sl(w.q), sl(w.k), sl(w.v)
        o_ref, lse_ref = oracle_mod.attention_compensated(wq, wk, wv, sl(idx_h), sl(cnt_h), w.valid_len,
                                                          qblocks=qblocks, order=order)
        rows = np.isfinite(lse_ref)
        mx, mean = output_errors(sl(og), o_ref, rows)
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (h, mx, mean)
        if order == 1:
            tol = 1e-4
        else:
            tol = mean_lse_bound(oracle_mod, wq, wk, w.valid_len)[rows]
        assert np.all(np.abs(sl(lg)[rows] - lse_ref[rows]) <= tol), np.abs(sl(lg)[rows] - lse_ref[rows]).max()
    if qblocks is None:
        # rows past each sample: o = 0, lse = -inf
        for b in range(w.q.shape[0]):
            L = int(w.valid_len[b])
            assert np.all(np.isneginf(lg[b, :, L:]))
            assert np.all(og[b, :, L:] == 0)
    return o, lse, idx, cnt


CASES = [
    # B, H, D, grid, sparsity, drop
    (1, 2, 128, (2, 16, 40), 0.75, 0.0),
    (2, 3, 128, (3, 10, 50), 0.5, 0.15),     # ragged
    (1, 1, 64, (5, 9, 37), 0.8, 0.1),        # D = 64, odd block count
    (3, 2, 128, (1, 7, 9), 0.5, 0.0),        # one partial block
    (1, 2, 128, (9, 30, 52), 0.9, 0.0),      # 220 blocks: four mean steps
]


@pytest.mark.parametrize("order", [1, 0])
@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("paired", [True, False])
def test_parity(sba, oracle_mod, case, paired, order):
    B, H, D, grid, s, drop = case
    w = make_custom(B, H, D, grid, s, drop_rate=drop, seed=hash(case) % 991)
    run(sba, oracle_mod, w, s, order, paired=paired)


def spread_workload(eps, seed=3, D=128, grid=(2, 16, 40)):
    """Keys = block mean + eps * (+-1 per channel, balanced within each block), exact
    in bf16 (block means on a 1/4 grid); random Q and V."""
    rng = np.random.default_rng(seed)
    w = make_custom(1, 2, D, grid, 0.8, seed=seed)
    B, H, N, _ = w.q.shape
    nB = N // 64
    kbar = rng.integers(-6, 7, size=(B, H, nB, D)) * 0.25
    u = np.empty((B, H, N, D))
    base = np.array([1.0] * 32 + [-1.0] * 32)
    for b in range(B):
        for h in range(H):
            for J in range(nB):
                for d in range(D):
                    u[b, h, J * 64:(J + 1) * 64, d] = rng.permutation(base)
    kf = np.repeat(kbar, 64, axis=2) + eps * u
    w.k = f64_to_bf16_bits(kf)
    w.q = f64_to_bf16_bits(rng.normal(size=w.q.shape))
    return w


def test_first_order_tracks_the_expansion(sba, oracle_mod):
    """Keys spread about their block means.  Each call sits much closer to its own
    oracle than the two orders are to each other, and the first-order call's distance
    to dense attention shrinks about fourfold when the spread halves (the mean-key
    call's about twofold); bf16 output rounding (about 2e-3 here) blurs the ratios a
    little, hence the margins."""
    d1, d0 = [], []
    for eps in (2.0 ** -1, 2.0 ** -2, 2.0 ** -3):
        w = spread_workload(eps)
        o1, _, idx, cnt = run(sba, oracle_mod, w, 0.8, 1)
        o0, _, _, _ = run(sba, oracle_mod, w, 0.8, 0)
        idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
        r1, _ = oracle_mod.attention_compensated(w.q, w.k, w.v, idx_h, cnt_h, w.valid_len, order=1)
        r0, _ = oracle_mod.attention_compensated(w.q, w.k, w.v, idx_h, cnt_h, w.valid_len, order=0)
        sep = np.abs(r1 - r0).max()
        g1, g0 = o1.float().cpu().numpy(), o0.float().cpu().numpy()
        assert np.abs(g1 - r1).max() < 0.2 * sep, (eps, np.abs(g1 - r1).max(), sep)
        assert np.abs(g0 - r0).max() < 0.2 * sep, (eps, np.abs(g0 - r0).max(), sep)
        o_d, _ = oracle_mod.dense(w.q, w.k, w.v, w.valid_len)
        d1.append(np.abs(g1 - o_d).max())
        d0.append(np.abs(g0 - o_d).max())
    assert d1[0] / d1[1] > 3.3 and d1[1] / d1[2] > 2.7, d1
    assert d0[0] / d0[1] < 2.6 and d0[1] / d0[2] < 2.6, d0


@pytest.mark.parametrize("order", [1, 0])
def test_block_constant_inputs_give_dense(sba, oracle_mod, order):
    """Keys and values constant within blocks: the compensation is exact, so the output
    is dense attention's."""
    rng = np.random.default_rng(5)
    B, H, N, D = 1, 2, 1280, 128
    bfx = lambda x: f64_to_bf16_bits(np.asarray(x, dtype=np.float64))
    rep = lambda a: np.repeat(a, 64, axis=2)[:, :, :N]
    w = make_custom(B, H, D, (2, 16, 40), 0.8, seed=7)
    w.q = bfx(rng.normal(size=(B, H, N, D)))
    w.k = bfx(rep(rng.normal(size=(B, H, N // 64, D))))
    w.v = bfx(rep(rng.normal(size=(B, H, N // 64, D))))
    o, lse, _, _ = run(sba, oracle_mod, w, 0.8, order)
    o_d, lse_d = oracle_mod.dense(w.q, w.k, w.v, w.valid_len)
    mx, mean = output_errors(o.float().cpu().numpy(), o_d)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


@pytest.mark.parametrize("order", [1, 0])
def test_nothing_dropped_equals_plain_attention(sba, oracle_mod, order):
    w = make_custom(1, 2, 128, (2, 16, 40), 0.0, seed=9, drop_rate=0.1)
    q, k, v, vl = to_device(w, DEV)
    idx, cnt = sba.pool_select(q, k, vl, 0.0)
    po = sba.pair_query_blocks(idx, cnt, vl)
    o1, l1 = sba.attention_paired(q, k, v, idx, cnt, po, vl)
    if order == 1:
        o2, l2 = sba.attention_compensated(q, k, v, idx, cnt, vl, pair_order=po)
    else:
        o2, l2 = sba.attention_mean_compensated(q, k, v, idx, cnt, vl, pair_order=po)
    assert sba.device_status() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)


@pytest.mark.parametrize("order", [1, 0])
def test_full_size_720p_sampled(sba, oracle_mod, order):
    w = make_workload("720p")
    nB = (int(w.valid_len[0]) + 63) // 64
    rng = np.random.default_rng(1)
    qb = np.unique(np.concatenate([rng.choice(nB, 6, replace=False), [nB - 1]])).astype(np.int32)
    run(sba, oracle_mod, w, w.sparsity, order, qblocks=qb, heads=(0, w.q.shape[1] - 1))
