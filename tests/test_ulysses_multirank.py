"""The Ulysses head-sharding plumbing (video_dit_block_b200/ulysses.py) on gloo ranks
on the CPU: the two all-to-alls move exactly the right tokens and heads, and
sequence-sharded attention equals the single-process result.  The attention itself
is the fp64 oracle here (the CUDA path needs a GPU; the exchange is what is tested)."""
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def oracle_attention(q, k, v, valid_len, sparsity):
    """CPU stand-in for the sparse path on gathered [B, H/P, N, D] bf16 tensors."""
    import oracle
    from workloads import f64_to_bf16_bits
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    qn, kn, vn = bits(q), bits(k), bits(v)
    vl = None if valid_len is None else valid_len.numpy()
    idx, cnt = oracle.select(qn, kn, vl, sparsity)
    o, lse = oracle.attention(qn, kn, vn, idx, cnt, vl)
    ob = torch.from_numpy(f64_to_bf16_bits(np.nan_to_num(o)).view(np.int16)).view(torch.bfloat16)
    return ob, torch.from_numpy(lse.astype(np.float32)), idx, cnt


def _rank(rank, world, port, q_out, case):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from video_dit_block_b200 import ulysses
    from workloads import make_custom
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, D, grid, s, drop = case
        w = make_custom(B, H, D, grid, s, drop_rate=drop, seed=17)
        N = w.q.shape[2]
        Nl = N // world
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        mine = [t(a[:, :, rank * Nl:(rank + 1) * Nl]) for a in (w.q, w.k, w.v)]
        # the exchange alone: heads of this rank, every token
        qh = ulysses.seq_to_heads(mine[0])
        Hl = H // world
        want = t(w.q[:, rank * Hl:(rank + 1) * Hl])
        ok_a2a = bool(torch.equal(qh.view(torch.int16), want.view(torch.int16)))
        back = ulysses.heads_to_seq(qh)
        ok_back = bool(torch.equal(back.view(torch.int16), mine[0].view(torch.int16)))
        vl = torch.from_numpy(w.valid_len)
        o, lse = ulysses.ulysses_attention(*mine, vl, s, attention=oracle_attention)
        q_out.put((rank, ok_a2a, ok_back, o.view(torch.int16).numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


CASES = [
    # B, H, D, grid, sparsity, drop
    (1, 4, 64, (2, 8, 16), 0.5, 0.0),    # 256 tokens, 2 ranks x 128
    (2, 4, 64, (2, 8, 16), 0.75, 0.2),   # ragged lengths
]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("case", CASES)
def test_sharded_attention_equals_single_process(case, world):
    sys.path.insert(0, ROOT)
    from workloads import make_custom
    B, H, D, grid, s, drop = case
    w = make_custom(B, H, D, grid, s, drop_rate=drop, seed=17)
    N = w.q.shape[2]
    if N % (64 * world) != 0:
        pytest.skip("the padded length must split into whole blocks per rank")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29000 + (os.getpid() * 7 + world * 131 + hash(case)) % 900
    procs = [ctx.Process(target=_rank, args=(r, world, port, q, case)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, ok_a2a, ok_back, o, lse = q.get(timeout=300)
        res[r] = (ok_a2a, ok_back, o, lse)
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert all(res[r][0] for r in res), "seq_to_heads moved the wrong tokens"
    assert all(res[r][1] for r in res), "heads_to_seq did not invert seq_to_heads"
    # reassemble and compare with the whole problem on one process
    o_full = np.concatenate([res[r][2] for r in range(world)], axis=2)
    lse_full = np.concatenate([res[r][3] for r in range(world)], axis=2)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    o_ref, lse_ref, _, _ = oracle_attention(t(w.q), t(w.k), t(w.v), torch.from_numpy(w.valid_len), s)
    np.testing.assert_array_equal(o_full, o_ref.view(torch.int16).numpy())
    np.testing.assert_array_equal(lse_full, lse_ref.numpy())


def test_fused_wrapper_rejects_wrong_shard_count():
    """ulysses_attention_fused checks its shard list against the group before any exchange
    or device work (one gloo rank on the CPU)."""
    import socket

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from video_dit_block_b200 import ulysses
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        x = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
        with pytest.raises(ValueError):
            ulysses.ulysses_attention_fused(x, x, x, None, 0.5, [x, x])
        with pytest.raises(ValueError):
            ulysses.ulysses_attention_fused(x, x, x, None, 0.5, [x], lse_shards=[x, x])
        with pytest.raises(ValueError):
            ulysses.ulysses_attention_fused(x, x, x, None, 0.5, [x], router="topk")
    finally:
        dist.destroy_process_group()
