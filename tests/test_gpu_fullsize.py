"""The four large problems at full size, in the bench's launch configuration, checked
on samples the oracle can compute one by one: the routing of two sampled heads (every
row), and the outputs of sampled query blocks of those heads."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, compare_routing, output_errors, to_device
from workloads import make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


@pytest.mark.parametrize("name", ["480p_dense", "480p_sparse", "720p", "long_clip"])
def test_full_size_sampled(sba, oracle_mod, name):
    w = make_workload(name)
    q, k, v, vl = to_device(w, DEV)
    # the bench's path: routing, tile pairing, paired attention
    o, lse, idx, cnt = sba.sparse_attention(q, k, v, vl, w.sparsity)
    assert sba.device_status() == 0
    rng = np.random.default_rng(len(name))
    idx_h, cnt_h = idx.cpu().numpy(), cnt.cpu().numpy()
    for (b, h) in [(0, 0), (w.B - 1, int(rng.integers(1, w.H)))]:
        sl = lambda x: np.ascontiguousarray(x[b:b + 1, h:h + 1])
        vlb = w.valid_len[b:b + 1]
        io, co, _, _, S = oracle_mod.select(sl(w.q), sl(w.k), vlb, w.sparsity, kmax=idx_h.shape[-1],
                                            return_intermediates=True)
        bad, _ = compare_routing(idx_h[b:b + 1, h:h + 1], cnt_h[b:b + 1, h:h + 1], io, co, S)
        assert not bad, (name, b, h, bad[:3])
        nB = (int(vlb[0]) + 63) // 64
        qb = np.unique(np.concatenate([rng.choice(nB, 12, replace=False), [nB - 1]])).astype(np.int32)
        o_ref, lse_ref = oracle_mod.attention(sl(w.q), sl(w.k), sl(w.v), idx_h[b:b + 1, h:h + 1],
                                              cnt_h[b:b + 1, h:h + 1], vlb, qblocks=qb)
        og = o[b:b + 1, h:h + 1].float().cpu().numpy()
        rows = ~np.isnan(lse_ref) & np.isfinite(lse_ref)
        mx, mean = output_errors(og, o_ref, rows)
        assert mx <= MAX_ABS and mean <= MEAN_ABS, (name, b, h, mx, mean)
        lg = lse[b:b + 1, h:h + 1].cpu().numpy()
        np.testing.assert_allclose(lg[rows], lse_ref[rows], rtol=0, atol=1e-4)
