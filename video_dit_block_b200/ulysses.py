"""Head sharding with a Ulysses all-to-all around the block-sparse path.

A video DiT run with sequence parallelism holds, on each of P ranks, a contiguous
1/P of the token sequence for all heads.  Attention needs the whole sequence, so
the page "MiniMax-H3 on 8xH200 benchmark" runs it under SP/Ulysses-8: one
all-to-all turns [B, H, N/P, D] per rank into [B, H/P, N, D] (every token, a
1/P share of the heads), attention runs per head unchanged -- routing and the
kernels see whole sequences -- and a second all-to-all turns the output back.

The exchange is torch.distributed's all_to_all_single (NCCL between GPUs, gloo on
CPU); the tensors travel as int32 pairs of bf16 bit patterns, so the exchange is
exact and works on either backend.  Token range r * N/P .. (r+1) * N/P lives on
rank r; heads p * H/P .. (p+1) * H/P are attended on rank p.

ulysses_attention_fused replaces the second exchange: the attention kernel's epilogue
stores every output row straight into the sequence shard of the rank that owns its
token (sba_attention_to_shards), so the output crosses the interconnect once, with no
all-to-all and no copy after it.  The shard buffers are one per rank; across GPUs they
are peer pointers (symmetric memory), which the caller provides.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def _as_words(x):
    """A [.., D] bf16 (or int16) tensor viewed as int32 pairs, D even."""
    return x.contiguous().view(torch.int32)


def seq_to_heads(x, group=None):
    """[B, H, N_local, D] on every rank -> [B, H/P, P * N_local, D] (this rank's heads,
    the whole sequence).  H must be a multiple of P."""
    P = dist.get_world_size(group)
    B, H, Nl, D = x.shape
    if H % P != 0:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    w = _as_words(x)                                   # [B, H, Nl, D/2]
    send = w.reshape(B, P, H // P, Nl, D // 2).transpose(0, 1).contiguous()  # [P dst, B, H/P, Nl, D/2]
    recv = torch.empty_like(send)                      # [P src, B, H/P, Nl, D/2]
    dist.all_to_all_single(recv, send, group=group)
    out = recv.permute(1, 2, 0, 3, 4).reshape(B, H // P, P * Nl, D // 2)
    return out.contiguous().view(x.dtype)


def heads_to_seq(y, group=None):
    """The inverse: [B, H/P, N, D] on every rank -> [B, H, N/P, D]."""
    P = dist.get_world_size(group)
    B, Hl, N, D = y.shape
    if N % P != 0:
        raise ValueError(f"{N} tokens do not split over {P} ranks")
    Nl = N // P
    w = _as_words(y)
    send = w.reshape(B, Hl, P, Nl, D // 2).permute(2, 0, 1, 3, 4).contiguous()  # [P dst, B, Hl, Nl, D/2]
    recv = torch.empty_like(send)                      # [P src (head group), B, Hl, Nl, D/2]
    dist.all_to_all_single(recv, send, group=group)
    out = recv.transpose(0, 1).reshape(B, P * Hl, Nl, D // 2)
    return out.contiguous().view(y.dtype)


def lse_heads_to_seq(lse, group=None):
    """[B, H/P, N] fp32 -> [B, H, N/P]."""
    P = dist.get_world_size(group)
    B, Hl, N = lse.shape
    Nl = N // P
    send = lse.contiguous().view(torch.int32).reshape(B, Hl, P, Nl).permute(2, 0, 1, 3).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.transpose(0, 1).reshape(B, P * Hl, Nl).contiguous().view(lse.dtype)


def ulysses_attention(q, k, v, valid_len=None, sparsity: float = 0.75, group=None, attention=None, **kwargs):
    """Sequence-sharded block-sparse attention.  q, k, v: this rank's [B, H, N/P, D]
    token range (N the padded length, a multiple of 64 P); valid_len: the samples'
    full lengths.  `attention(q, k, v, valid_len, sparsity, **kwargs) -> (o, lse, ...)`
    runs on the gathered [B, H/P, N, D] tensors; by default the library's
    sparse_attention.  Returns this rank's (o [B, H, N/P, D], lse [B, H, N/P])."""
    if attention is None:
        from .sba import sparse_attention as attention
    qh, kh, vh = (seq_to_heads(t, group) for t in (q, k, v))
    res = attention(qh, kh, vh, valid_len, sparsity, **kwargs)
    o_h, lse_h = res[0], res[1]
    return heads_to_seq(o_h, group), lse_heads_to_seq(lse_h, group)


def ulysses_attention_fused(q, k, v, valid_len, sparsity: float, o_shards, lse_shards=None, group=None,
                            h_total=None, softmax_scale: float = 0.0, router: str = "mean", budget: int = 1):
    """Sequence-sharded block-sparse attention with the output exchange fused into the
    attention kernel.  q, k, v: this rank's [B, H, N/P, D] token range (N a multiple of
    64 P); valid_len: the samples' full lengths.  o_shards[p] / lse_shards[p]: rank p's
    output buffers, bf16 [B, H, N/P, D] / fp32 [B, H, N/P] (tensors on this GPU, or raw
    device pointers to other ranks' memory, then h_total = H is required).  Every rank
    writes its heads' rows into every rank's shard; the call ends with a barrier of the
    group, after which each rank's own shard holds its token range for all heads.  router /
    budget as in sparse_attention."""
    from .sba import attention_to_shards, pair_query_blocks, pool_select, pool_select_lse
    P = dist.get_world_size(group)
    r = dist.get_rank(group)
    if len(o_shards) != P or (lse_shards is not None and len(lse_shards) != P):
        raise ValueError(f"one output shard per rank ({P})")
    if router not in ("mean", "lse"):
        raise ValueError(f"unknown router {router!r}")
    qh, kh, vh = (seq_to_heads(t, group) for t in (q, k, v))
    Hl = qh.shape[1]
    if router == "mean":
        idx, cnt = pool_select(qh, kh, valid_len, sparsity)
    else:
        idx, cnt = pool_select_lse(qh, kh, valid_len, sparsity, budget=budget)
    po = pair_query_blocks(idx, cnt, valid_len)
    attention_to_shards(qh, kh, vh, idx, cnt, o_shards, lse_shards, h_first=r * Hl, h_total=h_total,
                        valid_len=valid_len, pair_order=po, softmax_scale=softmax_scale)
    # every rank's stores into the shards land before any rank reads its own
    torch.cuda.current_stream().synchronize()
    dist.barrier(group)
