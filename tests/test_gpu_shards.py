"""Attention with the output stored straight into sequence shards (sba_attention_to_shards,
the output exchange of Ulysses head sharding fused into the epilogue), on one GPU: P
"ranks" are emulated by calling it once per head group with P local shard buffers.  The
shards, put back together, must equal the unsharded path bit for bit (same kernel, same
tiles: only where each row is stored differs), lse included, with 0 / -inf past each
sample's valid length."""
import numpy as np
import pytest
import torch

from helpers import to_device
from workloads import make_custom

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


@pytest.fixture(scope="module")
def sba():
    import video_dit_block_b200 as m
    return m


def unsharded(sba, q, k, v, vl, s):
    idx, cnt = sba.pool_select(q, k, vl, s)
    po = sba.pair_query_blocks(idx, cnt, vl)
    return sba.attention_paired(q, k, v, idx, cnt, po, vl)


@pytest.mark.parametrize("P", [1, 2, 4, 8])
@pytest.mark.parametrize("D,s,vl", [(128, 0.5, [512, 300]), (64, 0.75, [512, 512]), (128, 0.0, [512, 65])])
def test_shards_equal_unsharded(sba, P, D, s, vl):
    w = make_custom(2, 8, D, (2, 8, 32), s, seed=61)     # 512 tokens, 8 blocks
    w.valid_len = np.array(vl, dtype=np.int32)
    q, k, v, vlt = to_device(w, DEV)
    B, H, N, _ = q.shape
    o_ref, lse_ref = unsharded(sba, q, k, v, vlt, s)
    Nl, Hl = N // P, H // P
    o_sh = [torch.full((B, H, Nl, D), float("nan"), dtype=torch.bfloat16, device=DEV) for _ in range(P)]
    l_sh = [torch.full((B, H, Nl), float("nan"), dtype=torch.float32, device=DEV) for _ in range(P)]
    for r in range(P):           # rank r: heads r*Hl .. (r+1)*Hl, the whole sequence
        hs = slice(r * Hl, (r + 1) * Hl)
        qr, kr, vr = (t[:, hs].contiguous() for t in (q, k, v))
        idx, cnt = sba.pool_select(qr, kr, vlt, s)
        po = sba.pair_query_blocks(idx, cnt, vlt)
        sba.attention_to_shards(qr, kr, vr, idx, cnt, o_sh, l_sh, h_first=r * Hl, valid_len=vlt, pair_order=po)
    assert sba.device_status() == 0
    o_cat = torch.cat(o_sh, dim=2)
    l_cat = torch.cat(l_sh, dim=2)
    assert torch.equal(o_cat.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(l_cat.view(torch.int32), lse_ref.view(torch.int32))
    for b in range(B):
        assert torch.all(o_cat[b, :, vl[b]:] == 0) and torch.all(torch.isneginf(l_cat[b, :, vl[b]:]))


def test_raw_pointers_no_lse_and_untouched_heads(sba):
    """Shards given as raw device pointers (the form peer memory takes), no lse; only the
    caller's heads are written."""
    w = make_custom(1, 4, 128, (2, 8, 32), 0.5, seed=62)
    q, k, v, vlt = to_device(w, DEV)
    o_ref, _ = unsharded(sba, q, k, v, vlt, 0.5)
    P, N = 2, q.shape[2]
    o_sh = [torch.full((1, 4, N // P, 128), 7.0, dtype=torch.bfloat16, device=DEV) for _ in range(P)]
    hs = slice(2, 4)
    qr, kr, vr = (t[:, hs].contiguous() for t in (q, k, v))
    idx, cnt = sba.pool_select(qr, kr, vlt, 0.5)
    sba.attention_to_shards(qr, kr, vr, idx, cnt, [t.data_ptr() for t in o_sh], None, h_first=2, h_total=4,
                            valid_len=vlt)
    assert sba.device_status() == 0
    o_cat = torch.cat(o_sh, dim=2)
    assert torch.all(o_cat[:, :2] == 7.0)
    # adjacent tiles here against paired tiles in the reference: equal up to accumulation order
    d = (o_cat[:, 2:].float() - o_ref[:, 2:].float()).abs()
    assert float(d.max()) <= 2e-2


def test_fused_ulysses_single_rank(sba):
    """ulysses_attention_fused on a one-rank NCCL group: the sharded output is the whole
    output of the unsharded path."""
    import datetime
    import socket

    import torch.distributed as dist
    from video_dit_block_b200 import ulysses
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    torch.cuda.set_device(DEV)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=120), device_id=DEV)
    try:
        w = make_custom(1, 4, 128, (2, 8, 32), 0.5, seed=63)
        q, k, v, vlt = to_device(w, DEV)
        o_ref, lse_ref = unsharded(sba, q, k, v, vlt, 0.5)
        o = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
        ulysses.ulysses_attention_fused(q, k, v, vlt, 0.5, [o], [lse])
        assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), lse_ref.view(torch.int32))
    finally:
        dist.destroy_process_group()
