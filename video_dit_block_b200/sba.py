"""Python binding of the C ABI in include/sba.h (argument marshalling only).

Every function takes torch CUDA tensors, allocates outputs with torch (device
memory and streams are PyTorch's job here), and calls the CUDA library through
ctypes.  There is no fallback: if libsba.so is missing or a tensor is not on a
CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

from .build import LIB

SBA_OK = 0
_STATUS = {0: "SBA_OK", 1: "SBA_ERR_INVALID_ARG", 2: "SBA_ERR_UNSUPPORTED", 3: "SBA_ERR_ALIGNMENT",
           4: "SBA_ERR_CUDA", 5: "SBA_ERR_TIMEOUT", 6: "SBA_ERR_DEVICE_FLAG",
           7: "SBA_ERR_SCRATCH_TOO_SMALL"}
MAX_NPAD = 262144
BLOCK = 64


class SbaError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_STATUS.get(code, code)} ({_lib.sba_strerror(code).decode()})")


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libsba.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"CUDA library not built: {LIB} is missing "
                               "(run `python -m video_dit_block_b200.build`)")
        L = ctypes.CDLL(LIB)
        vp, i32, f64, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_float, ctypes.c_size_t
        L.sba_keep_count.restype = ctypes.c_int32
        L.sba_keep_count.argtypes = [ctypes.c_int32, f64]
        L.sba_pool_select_workspace_size.restype = sz
        L.sba_pool_select_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.sba_pool_select.restype = i32
        L.sba_pool_select.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, f64, i32, vp, vp, vp, sz, vp]
        L.sba_pool_select_lse_workspace_size.restype = sz
        L.sba_pool_select_lse_workspace_size.argtypes = [i32, i32, i32, i32, i32, i32]
        L.sba_pool_select_lse.restype = i32
        L.sba_pool_select_lse.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, i32, f64, i32, i32, vp, vp, vp,
                                          sz, vp]
        L.sba_qk_norm_rope_pool.restype = i32
        L.sba_qk_norm_rope_pool.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, i32, i32, f64, f32, vp, vp, vp]
        L.sba_pool_select_means.restype = i32
        L.sba_pool_select_means.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, f64, i32, vp, vp, vp, sz, vp]
        L.sba_keep_count_budget.restype = ctypes.c_int32
        L.sba_keep_count_budget.argtypes = [ctypes.c_int32, f64, ctypes.c_int32]
        L.sba_mean_compensation_workspace_size.restype = sz
        L.sba_mean_compensation_workspace_size.argtypes = [i32, i32, i32, i32, i32]
        L.sba_attention_mean_compensated.restype = i32
        L.sba_attention_mean_compensated.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, i32,
                                                     vp, f32, vp, sz, vp]
        L.sba_attention_compensated.restype = i32
        L.sba_attention_compensated.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, i32, vp,
                                                f32, vp]
        L.sba_block_means.restype = i32
        L.sba_block_means.argtypes = [vp, i32, i32, i32, i32, vp, i32, vp, vp]
        L.sba_attention.restype = i32
        L.sba_attention.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, i32, f32, vp]
        L.sba_pair_workspace_size.restype = sz
        L.sba_pair_workspace_size.argtypes = [i32, i32, i32, i32]
        L.sba_pair_query_blocks.restype = i32
        L.sba_pair_query_blocks.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, sz, vp]
        L.sba_attention_paired.restype = i32
        L.sba_attention_paired.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, i32, vp,
                                           f32, vp]
        L.sba_dense_attention.restype = i32
        L.sba_dense_attention.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, f32, vp]
        L.sba_attention_to_shards.restype = i32
        L.sba_attention_to_shards.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, vp, i32,
                                              vp, vp, i32, vp, f32, vp]
        L.sba_get_device_status.restype = i32
        L.sba_get_device_status.argtypes = [vp]
        L.sba_set_wait_limit.restype = None
        L.sba_set_wait_limit.argtypes = [ctypes.c_uint64]
        L.sba_set_attention_kernel.restype = i32
        L.sba_set_attention_kernel.argtypes = [i32]
        L.sba_pool_select_noalloc.restype = i32
        L.sba_pool_select_noalloc.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, f64, i32, vp, vp, vp]
        L.sba_noalloc_scratch_bytes.restype = sz
        L.sba_noalloc_scratch_bytes.argtypes = []
        L.sba_keep_token_count.restype = ctypes.c_int32
        L.sba_keep_token_count.argtypes = [ctypes.c_int32, f64]
        L.sba_token_prune_workspace_size.restype = sz
        L.sba_token_prune_workspace_size.argtypes = [i32, i32]
        L.sba_token_prune_select.restype = i32
        L.sba_token_prune_select.argtypes = [vp, i32, i32, i32, vp, f64, i32, vp, vp, vp, sz, vp]
        L.sba_gather_tokens.restype = i32
        L.sba_gather_tokens.argtypes = [vp, i32, i32, i32, i32, vp, vp, i32, vp, vp]
        L.sba_strerror.restype = ctypes.c_char_p
        L.sba_strerror.argtypes = [i32]
        _lib = L
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(code, what):
    if code != SBA_OK:
        raise SbaError(code, what)


def _qkv(*ts):
    for t in ts:
        if not (t.is_cuda and t.dtype == torch.bfloat16 and t.dim() == 4 and t.is_contiguous()):
            raise ValueError("expected contiguous bf16 CUDA tensors [B, H, Npad, D]")
    return ts[0].shape


def _valid_len(valid_len, device):
    if valid_len is None:
        return None
    if not (valid_len.is_cuda and valid_len.dtype == torch.int32 and valid_len.is_contiguous()):
        raise ValueError("valid_len must be a contiguous int32 CUDA tensor [B]")
    return valid_len


def keep_count(n_blocks: int, sparsity: float) -> int:
    return int(lib().sba_keep_count(int(n_blocks), float(sparsity)))


def kmax_for(Npad: int, sparsity: float, block: int = BLOCK) -> int:
    """Row capacity of kv_idx that every sample of padded length Npad fits in."""
    return keep_count(Npad // block, sparsity)


def workspace_size(B: int, H: int, Npad: int, D: int, block: int = BLOCK) -> int:
    return int(lib().sba_pool_select_workspace_size(B, H, Npad, D, block))


def pool_select(q, k, valid_len=None, sparsity: float = 0.0, kmax: int | None = None,
                block: int = BLOCK, kv_idx=None, kv_cnt=None, workspace=None, stream=None):
    """Routing: returns (kv_idx int32 [B,H,Npad/64,kmax], kv_cnt int32 [B,H,Npad/64])."""
    B, H, Npad, D = _qkv(q, k)
    vl = _valid_len(valid_len, q.device)
    nB = Npad // block
    if kmax is None:
        kmax = kmax_for(Npad, sparsity, block)
    if kv_idx is None:
        kv_idx = torch.empty((B, H, nB, kmax), dtype=torch.int32, device=q.device)
    if kv_cnt is None:
        kv_cnt = torch.empty((B, H, nB), dtype=torch.int32, device=q.device)
    wsz = workspace_size(B, H, Npad, D, block)
    if workspace is None:
        workspace = torch.empty(wsz, dtype=torch.uint8, device=q.device)
    _check(lib().sba_pool_select(_ptr(q), _ptr(k), B, H, Npad, D, _ptr(vl), block, float(sparsity),
                                 int(kmax), _ptr(kv_idx), _ptr(kv_cnt), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)),
           "sba_pool_select")
    return kv_idx, kv_cnt


def keep_count_budget(n_blocks: int, sparsity: float, budget: int = 1) -> int:
    """keep(n, s) rounded up to a multiple of `budget`, at most n (sba_keep_count_budget)."""
    if budget < 1:
        raise ValueError("budget must be >= 1")
    return int(lib().sba_keep_count_budget(int(n_blocks), float(sparsity), int(budget)))


def lse_workspace_size(B: int, H: int, Npad: int, D: int, nsub: int = 4, block: int = BLOCK) -> int:
    return int(lib().sba_pool_select_lse_workspace_size(B, H, Npad, D, block, nsub))


def pool_select_lse(q, k, valid_len=None, sparsity: float = 0.0, nsub: int = 4, budget: int = 1,
                    kmax: int | None = None, block: int = BLOCK, kv_idx=None, kv_cnt=None, workspace=None,
                    stream=None):
    """Sub-block log-sum-exp routing: (kv_idx int32 [B,H,Npad/64,kmax], kv_cnt int32 [B,H,Npad/64])."""
    B, H, Npad, D = _qkv(q, k)
    vl = _valid_len(valid_len, q.device)
    nB = Npad // block
    if kmax is None:
        kmax = keep_count_budget(nB, sparsity, budget)
    if kv_idx is None:
        kv_idx = torch.empty((B, H, nB, kmax), dtype=torch.int32, device=q.device)
    if kv_cnt is None:
        kv_cnt = torch.empty((B, H, nB), dtype=torch.int32, device=q.device)
    if workspace is None:
        workspace = torch.empty(lse_workspace_size(B, H, Npad, D, nsub, block), dtype=torch.uint8,
                                device=q.device)
    _check(lib().sba_pool_select_lse(_ptr(q), _ptr(k), B, H, Npad, D, _ptr(vl), block, int(nsub),
                                     float(sparsity), int(budget), int(kmax), _ptr(kv_idx), _ptr(kv_cnt),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)), "sba_pool_select_lse")
    return kv_idx, kv_cnt


def qk_norm_rope_pool(x, weight, pos, valid_len=None, rope_dim: int = 96, rope_base: float = 10000.0,
                      eps: float = 1e-6, out=None, means=None, want_means: bool = True, block: int = BLOCK,
                      stream=None):
    """QK RMSNorm + 3D RoPE (see include/sba.h), with the block means of the output.
    weight: bf16 [D]; pos: int32 [B, Npad, 3].  Returns (out bf16, means fp64 or None)."""
    B, H, Npad, D = _qkv(x)
    if not (weight.is_cuda and weight.dtype == torch.bfloat16 and weight.shape == (D,) and weight.is_contiguous()):
        raise ValueError("weight must be a contiguous bf16 CUDA tensor [D]")
    if not (pos.is_cuda and pos.dtype == torch.int32 and pos.shape == (B, Npad, 3) and pos.is_contiguous()):
        raise ValueError("pos must be a contiguous int32 CUDA tensor [B, Npad, 3]")
    if out is None:
        out = torch.empty_like(x)
    if means is None and want_means:
        means = torch.empty((B, H, Npad // block, D), dtype=torch.float64, device=x.device)
    _check(lib().sba_qk_norm_rope_pool(_ptr(x), _ptr(weight), _ptr(pos), B, H, Npad, D,
                                       _ptr(_valid_len(valid_len, x.device)), block, int(rope_dim),
                                       float(rope_base), float(eps), _ptr(out), _ptr(means), _stream(stream)),
           "sba_qk_norm_rope_pool")
    return out, means


def pool_select_means(qmean, kmean, valid_len=None, sparsity: float = 0.0, kmax: int | None = None,
                      block: int = BLOCK, kv_idx=None, kv_cnt=None, workspace=None, stream=None):
    """Routing from given fp64 block means [B, H, Npad/64, D] (no pass over Q and K)."""
    B, H, nB, D = qmean.shape
    for t in (qmean, kmean):
        if not (t.is_cuda and t.dtype == torch.float64 and t.is_contiguous() and t.shape == (B, H, nB, D)):
            raise ValueError("qmean / kmean must be contiguous fp64 CUDA tensors [B, H, Npad/64, D]")
    Npad = nB * block
    vl = _valid_len(valid_len, qmean.device)
    if kmax is None:
        kmax = kmax_for(Npad, sparsity, block)
    if kv_idx is None:
        kv_idx = torch.empty((B, H, nB, kmax), dtype=torch.int32, device=qmean.device)
    if kv_cnt is None:
        kv_cnt = torch.empty((B, H, nB), dtype=torch.int32, device=qmean.device)
    if workspace is None:
        workspace = torch.empty(workspace_size(B, H, Npad, D, block), dtype=torch.uint8, device=qmean.device)
    _check(lib().sba_pool_select_means(_ptr(qmean), _ptr(kmean), B, H, Npad, D, _ptr(vl), block, float(sparsity),
                                       int(kmax), _ptr(kv_idx), _ptr(kv_cnt), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(stream)),
           "sba_pool_select_means")
    return kv_idx, kv_cnt


def block_means(x, valid_len=None, block: int = BLOCK, stream=None):
    """fp64 block means [B, H, Npad/64, D]."""
    B, H, Npad, D = _qkv(x)
    out = torch.empty((B, H, Npad // block, D), dtype=torch.float64, device=x.device)
    _check(lib().sba_block_means(_ptr(x), B, H, Npad, D, _ptr(_valid_len(valid_len, x.device)), block,
                                 _ptr(out), _stream(stream)), "sba_block_means")
    return out


def attention(q, k, v, kv_idx, kv_cnt, valid_len=None, softmax_scale: float = 0.0, out=None,
              lse=None, want_lse: bool = True, block: int = BLOCK, stream=None):
    """Block-sparse attention under a routing.  Returns (o bf16, lse fp32 or None)."""
    B, H, Npad, D = _qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Npad), dtype=torch.float32, device=q.device)
    if not (kv_idx.dtype == torch.int32 and kv_cnt.dtype == torch.int32 and kv_idx.is_contiguous()
            and kv_cnt.is_contiguous() and kv_idx.is_cuda and kv_cnt.is_cuda):
        raise ValueError("kv_idx / kv_cnt must be contiguous int32 CUDA tensors")
    _check(lib().sba_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Npad, D,
                               _ptr(_valid_len(valid_len, q.device)), block, _ptr(kv_idx),
                               _ptr(kv_cnt), kv_idx.shape[-1], float(softmax_scale), _stream(stream)),
           "sba_attention")
    return out, lse


def pair_query_blocks(kv_idx, kv_cnt, valid_len=None, block: int = BLOCK, pair_order=None,
                      workspace=None, stream=None):
    """Tiles of two query blocks with overlapping kept lists: int32 [B, H, 2*ceil(nQ/2)]."""
    B, H, nQ, kmax = kv_idx.shape
    Npad = nQ * block
    if pair_order is None:
        pair_order = torch.empty((B, H, 2 * ((nQ + 1) // 2)), dtype=torch.int32, device=kv_idx.device)
    if workspace is None:
        workspace = torch.empty(int(lib().sba_pair_workspace_size(B, H, Npad, block)), dtype=torch.uint8,
                                device=kv_idx.device)
    _check(lib().sba_pair_query_blocks(_ptr(kv_idx), _ptr(kv_cnt), B, H, Npad, kmax,
                                       _ptr(_valid_len(valid_len, kv_idx.device)), block, _ptr(pair_order),
                                       _ptr(workspace), workspace.numel(), _stream(stream)),
           "sba_pair_query_blocks")
    return pair_order


def attention_paired(q, k, v, kv_idx, kv_cnt, pair_order, valid_len=None, softmax_scale: float = 0.0,
                     out=None, lse=None, want_lse: bool = True, block: int = BLOCK, stream=None):
    """sba_attention over the tiles of `pair_order`.  Returns (o bf16, lse fp32 or None)."""
    B, H, Npad, D = _qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Npad), dtype=torch.float32, device=q.device)
    _check(lib().sba_attention_paired(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Npad, D,
                                      _ptr(_valid_len(valid_len, q.device)), block, _ptr(kv_idx),
                                      _ptr(kv_cnt), kv_idx.shape[-1], _ptr(pair_order), float(softmax_scale),
                                      _stream(stream)), "sba_attention_paired")
    return out, lse


def attention_to_shards(q, k, v, kv_idx, kv_cnt, o_shards, lse_shards=None, h_first: int = 0, h_total=None,
                        valid_len=None, pair_order=None, softmax_scale: float = 0.0, block: int = BLOCK,
                        stream=None):
    """Attention for this caller's heads h_first .. h_first + H - 1 (q, k, v: [B, H, Npad, D],
    the whole sequence), each output row stored straight into the sequence shard that owns
    its token: o_shards[s] is bf16 [B, h_total, Npad / len(o_shards), D] (a tensor, or a raw
    device pointer such as a peer's symmetric-memory buffer, then h_total is required);
    lse_shards likewise fp32 [B, h_total, Npad / len(o_shards)] or None."""
    B, H, Npad, D = _qkv(q, k, v)
    n = len(o_shards)
    if n < 1 or n > 8:
        raise ValueError("between 1 and 8 output shards")
    ptr = lambda t: int(t) if isinstance(t, int) else t.data_ptr()
    if h_total is None:
        if isinstance(o_shards[0], int):
            raise ValueError("h_total is required with raw shard pointers")
        h_total = o_shards[0].shape[1]
    for t in list(o_shards) + list(lse_shards or []):
        if not isinstance(t, int):
            exp = torch.bfloat16 if t.dim() == 4 else torch.float32
            shape = (B, h_total, Npad // n) + ((D,) if t.dim() == 4 else ())
            if t.dtype != exp or tuple(t.shape) != shape or not t.is_contiguous() or t.device != q.device:
                raise ValueError(f"shard of shape {tuple(t.shape)} / {t.dtype}; expected {shape} / {exp}, contiguous")
    o_arr = (ctypes.c_void_p * n)(*[ptr(t) for t in o_shards])
    l_arr = None if lse_shards is None else (ctypes.c_void_p * n)(*[ptr(t) for t in lse_shards])
    _check(lib().sba_attention_to_shards(_ptr(q), _ptr(k), _ptr(v), ctypes.cast(o_arr, ctypes.c_void_p),
                                         None if l_arr is None else ctypes.cast(l_arr, ctypes.c_void_p), n,
                                         int(h_total), int(h_first), B, H, Npad, D,
                                         _ptr(_valid_len(valid_len, q.device)), block, _ptr(kv_idx), _ptr(kv_cnt),
                                         kv_idx.shape[-1], _ptr(pair_order), float(softmax_scale), _stream(stream)),
           "sba_attention_to_shards")


def attention_compensated(q, k, v, kv_idx, kv_cnt, valid_len=None, pair_order=None, softmax_scale: float = 0.0,
                          out=None, lse=None, want_lse: bool = True, block: int = BLOCK, stream=None):
    """Block-sparse attention with the dropped blocks compensated to first order about
    their mean keys (see include/sba.h).  Returns (o bf16, lse fp32 or None)."""
    B, H, Npad, D = _qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Npad), dtype=torch.float32, device=q.device)
    _check(lib().sba_attention_compensated(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Npad, D,
                                           _ptr(_valid_len(valid_len, q.device)), block, _ptr(kv_idx), _ptr(kv_cnt),
                                           kv_idx.shape[-1], _ptr(pair_order), float(softmax_scale),
                                           _stream(stream)), "sba_attention_compensated")
    return out, lse


def mean_compensation_workspace_size(B: int, H: int, Npad: int, D: int, block: int = BLOCK) -> int:
    return int(lib().sba_mean_compensation_workspace_size(B, H, Npad, D, block))


def attention_mean_compensated(q, k, v, kv_idx, kv_cnt, valid_len=None, pair_order=None, softmax_scale: float = 0.0,
                               out=None, lse=None, want_lse: bool = True, workspace=None, block: int = BLOCK,
                               stream=None):
    """Block-sparse attention with each dropped block as one softmax entry carrying its
    mean key and value (the zeroth-order form; see include/sba.h).  Returns (o, lse)."""
    B, H, Npad, D = _qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Npad), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(mean_compensation_workspace_size(B, H, Npad, D, block), dtype=torch.uint8,
                                device=q.device)
    _check(lib().sba_attention_mean_compensated(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Npad, D,
                                                _ptr(_valid_len(valid_len, q.device)), block, _ptr(kv_idx),
                                                _ptr(kv_cnt), kv_idx.shape[-1], _ptr(pair_order),
                                                float(softmax_scale), _ptr(workspace), workspace.numel(),
                                                _stream(stream)), "sba_attention_mean_compensated")
    return out, lse


def dense_attention(q, k, v, valid_len=None, softmax_scale: float = 0.0, out=None, lse=None,
                    want_lse: bool = True, stream=None):
    """Dense attention over each sample's valid tokens.  Returns (o bf16, lse fp32 or None)."""
    B, H, Npad, D = _qkv(q, k, v)
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Npad), dtype=torch.float32, device=q.device)
    _check(lib().sba_dense_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Npad, D,
                                     _ptr(_valid_len(valid_len, q.device)), float(softmax_scale),
                                     _stream(stream)), "sba_dense_attention")
    return out, lse


def sparse_attention(q, k, v, valid_len=None, sparsity: float = 0.75, softmax_scale: float = 0.0,
                     router: str = "mean", budget: int = 1, stream=None):
    """The whole path: routing, tile pairing, block-sparse attention.
    router "mean": block-mean scores (sba_pool_select); "lse": sub-block
    log-sum-exp scores with an optional kept-count budget (sba_pool_select_lse).
    Returns (o, lse, kv_idx, kv_cnt)."""
    if router == "mean":
        kv_idx, kv_cnt = pool_select(q, k, valid_len, sparsity, stream=stream)
    elif router == "lse":
        kv_idx, kv_cnt = pool_select_lse(q, k, valid_len, sparsity, budget=budget, stream=stream)
    else:
        raise ValueError(f"unknown router {router!r}")
    pair_order = pair_query_blocks(kv_idx, kv_cnt, valid_len, stream=stream)
    o, lse = attention_paired(q, k, v, kv_idx, kv_cnt, pair_order, valid_len, softmax_scale, stream=stream)
    return o, lse, kv_idx, kv_cnt


def keep_token_count(n_tokens: int, ratio: float) -> int:
    """Tokens saliency pruning keeps of n: clamp(ceil(ratio * n - 1e-9), 1, n)."""
    return int(lib().sba_keep_token_count(int(n_tokens), float(ratio)))


def token_prune(x, valid_len=None, ratio: float = 0.5, npad_out: int | None = None, idx=None, valid_out=None,
                workspace=None, stream=None):
    """Token pruning by feature-norm saliency (see include/sba.h).  x: bf16 [B, N, C]
    token features.  Returns (idx int32 [B, npad_out]: the kept tokens' indices in
    their original order, then -1; valid_out int32 [B]: the kept counts).  npad_out
    defaults to the kept count of a full sample rounded up to a multiple of 64."""
    if not (x.is_cuda and x.dtype == torch.bfloat16 and x.dim() == 3 and x.is_contiguous()):
        raise ValueError("expected a contiguous bf16 CUDA tensor [B, N, C]")
    B, N, C = x.shape
    if npad_out is None:
        npad_out = -(-keep_token_count(N, ratio) // BLOCK) * BLOCK
    if idx is None:
        idx = torch.empty((B, npad_out), dtype=torch.int32, device=x.device)
    if valid_out is None:
        valid_out = torch.empty((B,), dtype=torch.int32, device=x.device)
    if workspace is None:
        workspace = torch.empty(int(lib().sba_token_prune_workspace_size(B, N)), dtype=torch.uint8,
                                device=x.device)
    _check(lib().sba_token_prune_select(_ptr(x), B, N, C, _ptr(_valid_len(valid_len, x.device)), float(ratio),
                                        int(npad_out), _ptr(idx), _ptr(valid_out), _ptr(workspace),
                                        workspace.numel(), _stream(stream)), "sba_token_prune_select")
    return idx, valid_out


def gather_tokens(src, idx, valid_out, out=None, stream=None):
    """The kept rows of a per-token tensor, compacted: src [B, H, N, ...] or [B, N, ...]
    (any dtype, a row of 4k bytes), idx / valid_out as token_prune returns them.  Rows
    past a sample's kept count are zero.  Returns [B, H, npad_out, ...] / [B, npad_out, ...]."""
    if not (src.is_cuda and src.is_contiguous() and src.dim() >= 3):
        raise ValueError("expected a contiguous CUDA tensor [B, H, N, ...] or [B, N, ...]")
    B, npad_out = idx.shape
    heads = src.dim() == 4
    H, N = (src.shape[1], src.shape[2]) if heads else (1, src.shape[1])
    rest = src.shape[3:] if heads else src.shape[2:]
    row_bytes = src.element_size() * math.prod(rest)
    shape = (B, H, npad_out, *rest) if heads else (B, npad_out, *rest)
    if out is None:
        out = torch.empty(shape, dtype=src.dtype, device=src.device)
    _check(lib().sba_gather_tokens(_ptr(src), B, H, N, row_bytes, _ptr(idx), _ptr(valid_out), int(npad_out),
                                   _ptr(out), _stream(stream)), "sba_gather_tokens")
    return out


def device_status(stream=None) -> int:
    """Synchronise the stream; return and clear the device-side error word (an SBA_* code)."""
    return int(lib().sba_get_device_status(_stream(stream)))


def set_wait_limit(cycles: int) -> None:
    lib().sba_set_wait_limit(int(cycles))


_ATTN_KERNELS = {"auto": 0, "query_pairs": 1, "cta_pair": 2}


def set_attention_kernel(which: str) -> None:
    """Which D = 128 attention kernel the attention calls run (process-wide):
    "query_pairs" (one SM per two query blocks), "cta_pair" (a 2-SM cluster per four
    query blocks) or "auto" (the query pairs, the faster one on B200)."""
    if which not in _ATTN_KERNELS:
        raise ValueError(f"unknown attention kernel {which!r}; one of {sorted(_ATTN_KERNELS)}")
    _check(lib().sba_set_attention_kernel(_ATTN_KERNELS[which]), "sba_set_attention_kernel")
