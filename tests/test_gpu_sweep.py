"""A seeded sweep over small random problems: both head dims, one or two samples,
ragged lengths from token dropping, grids from a single block up to about fifty, sparsities
from 0 to 0.9, both routers, and each attention path (adjacent tiles, paired tiles,
compensated, the CTA pair).  Routing must match the oracle exactly (ties excused as in
the other routing tests); outputs must be within the attention tolerances of the oracle
fed the GPU routing; rows past a sample's length must be 0 with lse -inf."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, compare_routing, output_errors, to_device
from workloads import make_custom

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")

_rng = np.random.default_rng(2026)
CASES = []
for i in range(40):
    D = (64, 128)[i % 2]
    path = ("adjacent", "paired", "compensated", "cta_pair")[i % 4]
    if path == "cta_pair" and D == 64:
        path = "paired"
    big = i >= 24   # the last sixteen: grids of up to 3 x 16 x 64 tokens
    CASES.append(dict(i=i, D=D, B=1 + (i % 3 == 0), H=1 + i % 3,
                      grid=(int(_rng.integers(1, 4)), int(_rng.integers(2, 17 if big else 9)),
                            int(_rng.integers(4, 65 if big else 40))),
                      s=(0.0, 0.3, 0.5, 0.75, 0.9)[i % 5], drop=(0.0, 0.15)[(i // 2) % 2],
                      router=("mean", "lse")[(i // 3) % 2], path=path))


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    yield m
    m.set_attention_kernel("auto")


@pytest.mark.parametrize("c", CASES, ids=lambda c: f"{c['i']}-D{c['D']}-{c['router']}-{c['path']}")
def test_sweep(sba, oracle_mod, c):
    w = make_custom(c["B"], c["H"], c["D"], c["grid"], c["s"], drop_rate=c["drop"], seed=100 + c["i"])
    q, k, v, vl = to_device(w, DEV)
    if c["router"] == "lse":
        idx, cnt = sba.pool_select_lse(q, k, vl, c["s"], budget=8)
        io, co, S = oracle_mod.select_lse(w.q, w.k, w.valid_len, c["s"], budget=8, kmax=idx.shape[-1],
                                          return_scores=True)
    else:
        idx, cnt = sba.pool_select(q, k, vl, c["s"])
        io, co, _, _, S = oracle_mod.select(w.q, w.k, w.valid_len, c["s"], kmax=idx.shape[-1],
                                            return_intermediates=True)
    assert sba.device_status() == 0
    ih, ch = idx.cpu().numpy(), cnt.cpu().numpy()
    bad, _ = compare_routing(ih, ch, io, co, S)
    assert not bad, bad[:3]
    path = c["path"]
    if path == "adjacent":
        o, lse = sba.attention(q, k, v, idx, cnt, vl)
    elif path == "paired":
        o, lse = sba.attention_paired(q, k, v, idx, cnt, sba.pair_query_blocks(idx, cnt, vl), vl)
    elif path == "compensated":
        o, lse = sba.attention_compensated(q, k, v, idx, cnt, vl)
    else:
        sba.set_attention_kernel("cta_pair")
        try:
            o, lse = sba.attention(q, k, v, idx, cnt, vl)
        finally:
            sba.set_attention_kernel("auto")
    assert sba.device_status() == 0
    ref = oracle_mod.attention_compensated if path == "compensated" else oracle_mod.attention
    o_ref, lse_ref = ref(w.q, w.k, w.v, ih, ch, w.valid_len)
    n = np.arange(w.Npad)
    rows = np.broadcast_to((n[None, :] < w.valid_len[:, None])[:, None, :], lse_ref.shape)
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    mx, mean = output_errors(og, o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)
    np.testing.assert_allclose(lg[rows], lse_ref[rows], rtol=0, atol=1e-4)
    assert np.all(og[~rows] == 0.0) and np.all(np.isneginf(lg[~rows]))
