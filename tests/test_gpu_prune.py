"""GPU token pruning by feature-norm saliency (page "Sol Video Inference Engine",
LTX-2.3 appendix, stage 2: keep 50% of the video tokens by feat_norm) against the
fp64 oracle, and the pruned sequence through the rest of the path.

The saliencies are the sequential fp64 sums of exact squares on both sides, so the
squared norms and the kept index lists must be equal bit for bit (ties included:
equal norms go to the lower index on both sides).  The gather is a copy: bit-exact.
The end-to-end case prunes synthetic token features, gathers Q, K, V and the
positions, and runs routing and attention on the ragged result against the oracle on
the same compacted inputs."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, compare_routing, output_errors, to_device
from workloads import f64_to_bf16_bits, make_custom, make_hidden

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def bf_dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(torch.bfloat16)


def prune_both(sba, oracle_mod, x, vl, ratio, npad_out=None):
    B, N, C = x.shape
    xd = bf_dev(x)
    vld = None if vl is None else torch.from_numpy(vl).to(DEV)
    ws = torch.empty(int(sba.lib().sba_token_prune_workspace_size(B, N)), dtype=torch.uint8, device=DEV)
    idx, vout = sba.token_prune(xd, vld, ratio, npad_out=npad_out, workspace=ws)
    assert sba.device_status() == 0
    npo = idx.shape[1]
    io, vo, n2 = oracle_mod.token_prune(x, vl, ratio, npad_out=npo)
    np.testing.assert_array_equal(vout.cpu().numpy(), vo)
    np.testing.assert_array_equal(idx.cpu().numpy(), io)
    norms = ws[:B * N * 8].view(torch.float64).cpu().numpy().reshape(B, N)
    np.testing.assert_array_equal(norms, n2)
    return idx, vout


@pytest.mark.parametrize("C", [8, 64, 136, 512])
@pytest.mark.parametrize("ratio", [0.5, 0.3, 1.0])
def test_parity_random_features(sba, oracle_mod, C, ratio):
    rng = np.random.default_rng(C)
    x = f64_to_bf16_bits(rng.normal(size=(2, 1000, C)))
    prune_both(sba, oracle_mod, x, np.array([1000, 777], dtype=np.int32), ratio)


def test_parity_many_exact_ties(sba, oracle_mod):
    """Small integer features: many tokens share a squared norm, so the lower-index rule
    decides across the selection boundary."""
    rng = np.random.default_rng(2)
    x = f64_to_bf16_bits(rng.integers(-2, 3, size=(3, 2049, 16)).astype(np.float64))
    for ratio in (0.1, 0.5, 0.9):
        prune_both(sba, oracle_mod, x, np.array([2049, 1500, 65], dtype=np.int32), ratio)
    # every token equal: the first k are kept
    xs = f64_to_bf16_bits(np.ones((1, 300, 24)))
    idx, vout = prune_both(sba, oracle_mod, xs, None, 0.5)
    assert idx[0, :150].cpu().tolist() == list(range(150))


def test_parity_one_token_and_ratio_zero(sba, oracle_mod):
    rng = np.random.default_rng(3)
    x = f64_to_bf16_bits(rng.normal(size=(2, 70, 32)))
    prune_both(sba, oracle_mod, x, np.array([1, 70], dtype=np.int32), 0.5)
    prune_both(sba, oracle_mod, x, None, 0.0)         # keeps one token per sample


def test_parity_full_length(sba, oracle_mod):
    """The long-clip grid (31 x 34 x 60 = 63240 tokens, two samples) with 512 channels."""
    x = make_hidden(2, (31, 34, 60), 512, seed=9)
    prune_both(sba, oracle_mod, x, np.array([63240, 53754], dtype=np.int32), 0.5)


def test_gather_is_exact(sba, oracle_mod):
    rng = np.random.default_rng(4)
    B, H, N, D = 2, 3, 500, 128
    x = f64_to_bf16_bits(rng.normal(size=(B, N, 64)))
    vl = np.array([500, 321], dtype=np.int32)
    idx, vout = prune_both(sba, oracle_mod, x, vl, 0.5)
    ih, vo = idx.cpu().numpy(), vout.cpu().numpy()
    src = f64_to_bf16_bits(rng.normal(size=(B, H, N, D)))
    pos = rng.integers(0, 1000, size=(B, N, 3)).astype(np.int32)
    got = sba.gather_tokens(bf_dev(src), idx, vout).view(torch.int16).cpu().numpy().view(np.uint16)
    gpos = sba.gather_tokens(torch.from_numpy(pos).to(DEV), idx, vout).cpu().numpy()
    assert sba.device_status() == 0
    npo = ih.shape[1]
    for b in range(B):
        k = int(vo[b])
        np.testing.assert_array_equal(got[b, :, :k], src[b][:, ih[b, :k]])
        assert np.all(got[b, :, k:] == 0)
        np.testing.assert_array_equal(gpos[b, :k], pos[b, ih[b, :k]])
        assert np.all(gpos[b, k:] == 0)
    assert got.shape == (B, H, npo, D) and gpos.shape == (B, npo, 3)


def test_pruned_sequence_through_the_path(sba, oracle_mod):
    """Token features -> saliency pruning (50%) -> gathered Q, K, V -> routing and
    attention on the ragged, pruned sequence, against the oracle on the same inputs."""
    grid = (4, 12, 40)                                    # 1920 tokens
    w = make_custom(2, 2, 128, grid, 0.75, seed=21)
    x = make_hidden(2, grid, 256, seed=22)
    vl = np.array([1920, 1500], dtype=np.int32)           # the second sample already shorter
    idx, vout = prune_both(sba, oracle_mod, x, vl, 0.5)
    q, k, v, _ = to_device(w, DEV)
    qp, kp, vp = (sba.gather_tokens(t, idx, vout) for t in (q, k, v))
    o, lse, kv_idx, kv_cnt = sba.sparse_attention(qp, kp, vp, vout, 0.75)
    assert sba.device_status() == 0
    ih, vo = idx.cpu().numpy(), vout.cpu().numpy()
    npo = ih.shape[1]
    # the same compaction on the host, from the oracle's (equal) index lists
    qh, kh, vh = (np.zeros((2, 2, npo, 128), dtype=np.uint16) for _ in range(3))
    for b in range(2):
        kb = int(vo[b])
        for dst, src in ((qh, w.q), (kh, w.k), (vh, w.v)):
            dst[b, :, :kb] = src[b][:, ih[b, :kb]]
    io, co, _, _, S = oracle_mod.select(qh, kh, vo, 0.75, kmax=kv_idx.shape[-1], return_intermediates=True)
    bad, excused = compare_routing(kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), io, co, S)
    assert not bad, bad[:3]
    o_ref, lse_ref = oracle_mod.attention(qh, kh, vh, kv_idx.cpu().numpy(), kv_cnt.cpu().numpy(), vo)
    rows = np.isfinite(lse_ref)
    mx, mean = output_errors(o.float().cpu().numpy(), o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    assert np.all(vo == [960, 750])
