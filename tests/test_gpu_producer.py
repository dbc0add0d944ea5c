"""GPU producer step (sba_qk_norm_rope_pool) and routing from its means
(sba_pool_select_means) against the fp64 oracle.

The GPU rounds to bf16 at the same two points as the oracle but computes in fp32, so the
rounded norm y may land one bf16 step from the oracle's, and the rotation
o = y0 cos - y1 sin carries that step into the output (amplified relative to o where the
two terms cancel).  The bound per output is therefore one step of o plus one step of
each of its pair's two inputs, 2^-7 (|o| + |y_2i| + |y_2i+1|); outputs off by anything
must also stay under 1%.  The block means are compared bit for bit with the pooling of
the GPU's own output, and the routing from them with the routing computed from that
output."""
import numpy as np
import pytest
import torch

from helpers import MAX_ABS, MEAN_ABS, compare_routing, output_errors, to_device
from workloads import make_custom, make_norm_weights, make_workload

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def dev_bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(DEV).view(torch.bfloat16)


def run_producer(sba, x, wbits, pos, vl, rope_dim=96, inplace=False):
    xd = dev_bf16(x)
    wd = dev_bf16(wbits)
    pd = torch.from_numpy(np.ascontiguousarray(pos)).to(DEV)
    vld = torch.from_numpy(np.ascontiguousarray(vl)).to(DEV)
    out, means = sba.qk_norm_rope_pool(xd, wd, pd, vld, rope_dim=rope_dim, out=xd if inplace else None)
    assert sba.device_status() == 0
    return out, means


def check_against_oracle(oracle_mod, x, wbits, pos, out_gpu, rope_dim=96):
    ref = oracle_mod.qk_norm_rope(x, wbits, pos, rope_dim=rope_dim)
    y = f64b(oracle_mod.qk_norm_rope(x, wbits, pos, rope_dim=0))  # the rounded norm
    g = out_gpu.view(torch.int16).cpu().numpy().view(np.uint16)
    err = np.abs(f64b(g) - f64b(ref))
    pair = np.abs(y[..., 0::2]) + np.abs(y[..., 1::2])
    pair = np.repeat(pair, 2, axis=-1)
    bound = 2.0 ** -7 * (np.abs(f64b(ref)) + pair)
    assert np.all(err <= bound), f"max excess {float((err - bound).max()):.3e}"
    frac = float((err > 0).mean())
    assert frac < 0.01, f"{frac:.4f} of outputs off"
    return g, frac


def f64b(bits):
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


CASES = [
    # B, H, D, grid, drop, rope_dim
    (1, 2, 128, (2, 8, 16), 0.0, 96),
    (2, 2, 128, (3, 7, 9), 0.2, 96),     # ragged, pruned positions
    (1, 3, 64, (4, 5, 12), 0.0, 48),     # D = 64
    (1, 1, 128, (2, 8, 8), 0.0, 0),      # no rotation
    (1, 1, 128, (2, 8, 8), 0.0, 126),    # rotation on all but two channels
]


@pytest.mark.parametrize("case", CASES)
def test_producer_parity(sba, oracle_mod, case):
    B, H, D, grid, drop, rd = case
    w = make_custom(B, H, D, grid, 0.5, drop_rate=drop, seed=hash(case) % 997)
    wq, _ = make_norm_weights(D)
    out, means = run_producer(sba, w.q, wq, w.positions, w.valid_len, rope_dim=rd)
    g, _ = check_against_oracle(oracle_mod, w.q, wq, w.positions, out, rope_dim=rd)
    # the means are exactly the pooling of the GPU's own output
    np.testing.assert_array_equal(means.cpu().numpy(), oracle_mod.pool(g, w.valid_len))
    vld = torch.from_numpy(w.valid_len).to(DEV)
    np.testing.assert_array_equal(means.cpu().numpy(), sba.block_means(out, vld).cpu().numpy())


def test_in_place(sba, oracle_mod):
    w = make_custom(1, 2, 128, (2, 8, 16), 0.5, seed=3)
    wq, _ = make_norm_weights(128)
    out, _ = run_producer(sba, w.q, wq, w.positions, w.valid_len, inplace=True)
    check_against_oracle(oracle_mod, w.q, wq, w.positions, out)


@pytest.mark.parametrize("name,heads", [("480p_sparse", 2), ("720p", 1), ("long_clip", 1)])
def test_named_workloads(sba, oracle_mod, name, heads):
    w = make_workload(name, heads=heads)
    wq, wk = make_norm_weights(w.D if hasattr(w, "D") else w.q.shape[3])
    for x, wt in ((w.q, wq), (w.k, wk)):
        out, _ = run_producer(sba, x, wt, w.positions, w.valid_len)
        check_against_oracle(oracle_mod, x, wt, w.positions, out)


def test_routing_from_means_equals_routing_from_outputs(sba, oracle_mod):
    w = make_custom(2, 2, 128, (3, 12, 40), 0.75, drop_rate=0.1, seed=21)
    wq, wk = make_norm_weights(128)
    qo, qm = run_producer(sba, w.q, wq, w.positions, w.valid_len)
    ko, km = run_producer(sba, w.k, wk, w.positions, w.valid_len)
    vld = torch.from_numpy(w.valid_len).to(DEV)
    i1, c1 = sba.pool_select_means(qm, km, vld, 0.75)
    i2, c2 = sba.pool_select(qo, ko, vld, 0.75)
    assert sba.device_status() == 0
    c1, c2 = c1.cpu().numpy(), c2.cpu().numpy()
    np.testing.assert_array_equal(c1, c2)
    a1, a2 = i1.cpu().numpy(), i2.cpu().numpy()
    for r in np.ndindex(c1.shape):
        assert np.array_equal(a1[r][:c1[r]], a2[r][:c2[r]])
    # and the oracle's routing of the GPU's own outputs
    qg = qo.view(torch.int16).cpu().numpy().view(np.uint16)
    kg = ko.view(torch.int16).cpu().numpy().view(np.uint16)
    io, co, _, _, S = oracle_mod.select(qg, kg, w.valid_len, 0.75, kmax=a1.shape[-1], return_intermediates=True)
    bad, _ = compare_routing(a1, c1, io, co, S)
    assert not bad


def test_whole_path_from_unnormalised_inputs(sba, oracle_mod):
    """producer (Q, K) -> routing from means -> pairing -> attention, against the oracle's
    attention of the GPU's normalised Q, K under the same routing."""
    w = make_custom(1, 2, 128, (3, 12, 40), 0.75, seed=23)
    wq, wk = make_norm_weights(128)
    qo, qm = run_producer(sba, w.q, wq, w.positions, w.valid_len)
    ko, km = run_producer(sba, w.k, wk, w.positions, w.valid_len)
    vld = torch.from_numpy(w.valid_len).to(DEV)
    v = dev_bf16(w.v)
    idx, cnt = sba.pool_select_means(qm, km, vld, 0.75)
    po = sba.pair_query_blocks(idx, cnt, vld)
    o, lse = sba.attention_paired(qo, ko, v, idx, cnt, po, vld)
    assert sba.device_status() == 0
    qg = qo.view(torch.int16).cpu().numpy().view(np.uint16)
    kg = ko.view(torch.int16).cpu().numpy().view(np.uint16)
    o_ref, lse_ref = oracle_mod.attention(qg, kg, w.v, idx.cpu().numpy(), cnt.cpu().numpy(), w.valid_len)
    rows = np.isfinite(lse_ref)
    mx, mean = output_errors(o.float().cpu().numpy(), o_ref, rows)
    assert mx <= MAX_ABS and mean <= MEAN_ABS, (mx, mean)


def test_full_size_720p_sampled_heads(sba, oracle_mod):
    w = make_workload("720p")
    wq, _ = make_norm_weights(128)
    out, means = run_producer(sba, w.q, wq, w.positions, w.valid_len)
    g = out.view(torch.int16).cpu().numpy().view(np.uint16)
    for h in (0, w.q.shape[1] - 1):
        sl = np.ascontiguousarray(w.q[:, h:h + 1])
        gh = np.ascontiguousarray(g[:, h:h + 1])
        check_against_oracle(oracle_mod, sl, wq, w.positions,
                             torch.from_numpy(gh.view(np.int16)).view(torch.bfloat16))
        np.testing.assert_array_equal(means[:, h:h + 1].cpu().numpy(),
                                      oracle_mod.pool(np.ascontiguousarray(g[:, h:h + 1]), w.valid_len))
