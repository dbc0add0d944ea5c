"""fp64 CPU oracle of training-free block-sparse self-attention (test infrastructure).

Only the tests, `__graft_entry__.smoke()` and the bench's CPU-baseline leg may import
this package.  It wraps `oracle.c` (plain C, fp64, OpenMP over independent rows) with
ctypes and numpy arrays; it shares nothing with the CUDA library.

The method follows the SubBlock router of the page "MiniMax-H3 on 8xH200 benchmark"
(news.paixiangai.cn), section "How SubBlock sparse attention works", in its
one-sub-block form: block means of Q and K, score = mean(q).mean(k)/sqrt(D), keep the
ceil((1-s)*nKV) best key blocks per query block (ties to the lower index), then exact
softmax attention over the kept tokens.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (no fast-math: IEEE fp64)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        i32, f64, vp = ctypes.c_int32, ctypes.c_double, ctypes.c_void_p
        _lib.oracle_keep_count.restype = i32
        _lib.oracle_keep_count.argtypes = [i32, f64]
        _lib.oracle_pool.restype = None
        _lib.oracle_pool.argtypes = [vp, i32, i32, i32, i32, vp, i32, vp]
        _lib.oracle_scores.restype = None
        _lib.oracle_scores.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, vp]
        _lib.oracle_topk.restype = i32
        _lib.oracle_topk.argtypes = [vp, i32, i32, i32, vp, i32, f64, i32, vp, vp]
        _lib.oracle_select.restype = i32
        _lib.oracle_select.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, f64, i32, vp, vp,
                                       vp, vp, vp]
        _lib.oracle_select_lse.restype = i32
        _lib.oracle_select_lse.argtypes = [vp, vp, i32, i32, i32, i32, vp, i32, i32, f64, i32, i32, vp,
                                           vp, vp]
        _lib.oracle_qk_norm_rope.restype = i32
        _lib.oracle_qk_norm_rope.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, f64, f64, vp, vp]
        _lib.oracle_attention_compensated.restype = i32
        _lib.oracle_attention_compensated.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, i32,
                                                      f64, i32, vp, i32, vp, vp]
        _lib.oracle_attention.restype = i32
        _lib.oracle_attention.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, i32,
                                          f64, vp, i32, vp, vp]
        _lib.oracle_dense.restype = None
        _lib.oracle_dense.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, f64, vp, vp]
        _lib.oracle_keep_tokens.restype = i32
        _lib.oracle_keep_tokens.argtypes = [i32, f64]
        _lib.oracle_token_prune.restype = i32
        _lib.oracle_token_prune.argtypes = [vp, i32, i32, i32, vp, f64, i32, vp, vp, vp]
        _lib.oracle_probs.restype = i32
        _lib.oracle_probs.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp, i32, f64,
                                      i32, i32, i32, vp]
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _bf16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16 and a.ndim == 4, "bf16 bit patterns [B,H,Npad,D] expected"
    return a


def _vl(valid_len, B, Npad):
    if valid_len is None:
        return np.full(B, Npad, dtype=np.int32)
    return np.ascontiguousarray(valid_len, dtype=np.int32)


def keep_count(n_blocks: int, sparsity: float) -> int:
    """Kept key blocks per query block: clamp(ceil((1-s)*n - 1e-9), 1, n)."""
    return int(_load().oracle_keep_count(int(n_blocks), float(sparsity)))


def n_blocks(valid_len: int, block: int = 64) -> int:
    return (int(valid_len) + block - 1) // block


def kmax_for(valid_len, sparsity: float, block: int = 64) -> int:
    return max(keep_count(n_blocks(L, block), sparsity) for L in np.atleast_1d(valid_len))


def pool(x, valid_len=None, block: int = 64) -> np.ndarray:
    """fp64 block means [B, H, Npad/block, D] over valid tokens."""
    x = _bf16(x)
    B, H, Npad, D = x.shape
    vl = _vl(valid_len, B, Npad)
    out = np.zeros((B, H, Npad // block, D), dtype=np.float64)
    _load().oracle_pool(_p(x), B, H, Npad, D, _p(vl), block, _p(out))
    return out


def scores(qbar, kbar, valid_len, block: int = 64) -> np.ndarray:
    """fp64 block scores [B, H, nB, nB]; NaN outside each sample's block square."""
    qbar = np.ascontiguousarray(qbar, dtype=np.float64)
    kbar = np.ascontiguousarray(kbar, dtype=np.float64)
    B, H, nB, D = qbar.shape
    vl = np.ascontiguousarray(valid_len, dtype=np.int32)
    S = np.empty((B, H, nB, nB), dtype=np.float64)
    _load().oracle_scores(_p(qbar), _p(kbar), B, H, nB, D, _p(vl), block, _p(S))
    return S


def topk(S, valid_len, sparsity: float, kmax: int | None = None, block: int = 64):
    """Routing from scores: (kv_idx [B,H,nB,kmax] ascending, -1 tail; kv_cnt [B,H,nB])."""
    S = np.ascontiguousarray(S, dtype=np.float64)
    B, H, nB, _ = S.shape
    vl = np.ascontiguousarray(valid_len, dtype=np.int32)
    if kmax is None:
        kmax = kmax_for(vl, sparsity, block)
    idx = np.empty((B, H, nB, kmax), dtype=np.int32)
    cnt = np.empty((B, H, nB), dtype=np.int32)
    st = _load().oracle_topk(_p(S), B, H, nB, _p(vl), block, float(sparsity), kmax, _p(idx), _p(cnt))
    if st != 0:
        raise ValueError("kmax smaller than the kept count")
    return idx, cnt


def select(q, k, valid_len=None, sparsity: float = 0.0, kmax: int | None = None,
           block: int = 64, return_intermediates: bool = False):
    """Pool -> score -> top-k.  Returns (kv_idx, kv_cnt[, pooled_q, pooled_k, scores])."""
    q, k = _bf16(q), _bf16(k)
    B, H, Npad, D = q.shape
    vl = _vl(valid_len, B, Npad)
    if kmax is None:
        kmax = kmax_for(vl, sparsity, block)
    nB = Npad // block
    idx = np.empty((B, H, nB, kmax), dtype=np.int32)
    cnt = np.empty((B, H, nB), dtype=np.int32)
    pq = pk = S = None
    if return_intermediates:
        pq = np.empty((B, H, nB, D))
        pk = np.empty((B, H, nB, D))
        S = np.empty((B, H, nB, nB))
    st = _load().oracle_select(_p(q), _p(k), B, H, Npad, D, _p(vl), block, float(sparsity), kmax,
                               _p(idx), _p(cnt), _p(pq), _p(pk), _p(S))
    if st != 0:
        raise ValueError("kmax smaller than the kept count")
    if return_intermediates:
        return idx, cnt, pq, pk, S
    return idx, cnt


def keep_count_budget(n_blocks: int, sparsity: float, budget: int = 1) -> int:
    """keep(n, s) rounded up to a multiple of `budget`, at most n."""
    k = keep_count(n_blocks, sparsity)
    if budget > 1:
        k = min(int(n_blocks), -(-k // budget) * budget)
    return k


def select_lse(q, k, valid_len=None, sparsity: float = 0.0, nsub: int = 4, budget: int = 1,
               kmax: int | None = None, block: int = 64, return_scores: bool = False):
    """Sub-block log-sum-exp router: (kv_idx, kv_cnt[, scores [B,H,nB,nB]])."""
    q, k = _bf16(q), _bf16(k)
    B, H, Npad, D = q.shape
    vl = _vl(valid_len, B, Npad)
    if kmax is None:
        kmax = max(keep_count_budget(n_blocks(L, block), sparsity, budget) for L in vl)
    nB = Npad // block
    idx = np.empty((B, H, nB, kmax), dtype=np.int32)
    cnt = np.empty((B, H, nB), dtype=np.int32)
    S = np.empty((B, H, nB, nB)) if return_scores else None
    st = _load().oracle_select_lse(_p(q), _p(k), B, H, Npad, D, _p(vl), block, nsub, float(sparsity),
                                   int(budget), kmax, _p(idx), _p(cnt), _p(S))
    if st == -2:
        raise ValueError("nsub must divide the block size and be at most 16")
    if st != 0:
        raise ValueError("kmax smaller than the kept count")
    return (idx, cnt, S) if return_scores else (idx, cnt)


def qk_norm_rope(x, weight, pos, rope_dim: int = 96, base: float = 10000.0, eps: float = 1e-6,
                 return_unrounded: bool = False):
    """QK RMSNorm (over D, weight [D]) then 3D RoPE on channels [0, rope_dim), rounding
    to bf16 after the norm and after the rotation.  Returns bf16 bits [B,H,Npad,D]
    (and the fp64 values before the last rounding)."""
    x = _bf16(x)
    B, H, Npad, D = x.shape
    w = np.ascontiguousarray(weight, dtype=np.uint16)
    assert w.shape == (D,)
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    assert pos.shape == (B, Npad, 3)
    out = np.empty_like(x)
    out64 = np.empty(x.shape) if return_unrounded else None
    st = _load().oracle_qk_norm_rope(_p(x), _p(w), _p(pos), B, H, Npad, D, int(rope_dim), float(base),
                                     float(eps), _p(out), _p(out64))
    if st == -2:
        raise ValueError("rope_dim must be a multiple of 6 in [0, D]")
    return (out, out64) if return_unrounded else out


def attention(q, k, v, kv_idx, kv_cnt, valid_len=None, scale: float = 0.0, block: int = 64,
              qblocks=None):
    """fp64 block-sparse attention under a routing.  Returns (o [B,H,Npad,D], lse [B,H,Npad]).
    With `qblocks`, only those query blocks are computed; other rows are NaN."""
    q, k, v = _bf16(q), _bf16(k), _bf16(v)
    B, H, Npad, D = q.shape
    vl = _vl(valid_len, B, Npad)
    kv_idx = np.ascontiguousarray(kv_idx, dtype=np.int32)
    kv_cnt = np.ascontiguousarray(kv_cnt, dtype=np.int32)
    assert kv_idx.shape[:3] == (B, H, Npad // block) and kv_cnt.shape == (B, H, Npad // block)
    kmax = kv_idx.shape[3]
    o = np.full((B, H, Npad, D), np.nan)
    lse = np.full((B, H, Npad), np.nan)
    qb = None if qblocks is None else np.ascontiguousarray(qblocks, dtype=np.int32)
    st = _load().oracle_attention(_p(q), _p(k), _p(v), B, H, Npad, D, _p(vl), block, _p(kv_idx),
                                  _p(kv_cnt), kmax, float(scale), _p(qb),
                                  0 if qb is None else len(qb), _p(o), _p(lse))
    if st != 0:
        raise ValueError("routing entry outside the sample's blocks")
    return o, lse


def attention_compensated(q, k, v, kv_idx, kv_cnt, valid_len=None, scale: float = 0.0, block: int = 64,
                          qblocks=None, order: int = 1):
    """Block-sparse attention with the dropped blocks compensated by the first-order
    expansion of their exponentials about each block's mean key (order=1: the count-
    weighted mean value plus the moment term s q^T sum_j (k_j - kbar)v_j^T), or by the
    mean key and value alone (order=0).  Means in fp64.  Returns (o, lse) like
    `attention`."""
    q, k, v = _bf16(q), _bf16(k), _bf16(v)
    B, H, Npad, D = q.shape
    vl = _vl(valid_len, B, Npad)
    kv_idx = np.ascontiguousarray(kv_idx, dtype=np.int32)
    kv_cnt = np.ascontiguousarray(kv_cnt, dtype=np.int32)
    o = np.full((B, H, Npad, D), np.nan)
    lse = np.full((B, H, Npad), np.nan)
    qb = None if qblocks is None else np.ascontiguousarray(qblocks, dtype=np.int32)
    st = _load().oracle_attention_compensated(_p(q), _p(k), _p(v), B, H, Npad, D, _p(vl), block, _p(kv_idx),
                                              _p(kv_cnt), kv_idx.shape[3], float(scale), int(order), _p(qb),
                                              0 if qb is None else len(qb), _p(o), _p(lse))
    if st == -2:
        raise ValueError("order must be 0 or 1")
    if st != 0:
        raise ValueError("routing entry outside the sample's blocks")
    return o, lse


def attention_mean_compensated(q, k, v, kv_idx, kv_cnt, valid_len=None, scale: float = 0.0, block: int = 64,
                               qblocks=None):
    """The zeroth-order form: each dropped block is one softmax entry of logit
    s q.kbar_J + log c_J carrying vbar_J (fp64 means)."""
    return attention_compensated(q, k, v, kv_idx, kv_cnt, valid_len, scale, block, qblocks, order=0)


def dense(q, k, v, valid_len=None, scale: float = 0.0):
    """fp64 dense softmax attention over each sample's valid tokens."""
    q, k, v = _bf16(q), _bf16(k), _bf16(v)
    B, H, Npad, D = q.shape
    vl = _vl(valid_len, B, Npad)
    o = np.empty((B, H, Npad, D))
    lse = np.empty((B, H, Npad))
    _load().oracle_dense(_p(q), _p(k), _p(v), B, H, Npad, D, _p(vl), float(scale), _p(o), _p(lse))
    return o, lse


def probs(q, k, v, kv_idx, kv_cnt, b, h, i, valid_len=None, scale: float = 0.0, block: int = 64):
    """Softmax probability row [Npad] of query row i of (b, h) under a routing."""
    q, k, v = _bf16(q), _bf16(k), _bf16(v)
    B, H, Npad, D = q.shape
    vl = _vl(valid_len, B, Npad)
    kv_idx = np.ascontiguousarray(kv_idx, dtype=np.int32)
    kv_cnt = np.ascontiguousarray(kv_cnt, dtype=np.int32)
    p = np.zeros(Npad)
    st = _load().oracle_probs(_p(q), _p(k), _p(v), B, H, Npad, D, _p(vl), block, _p(kv_idx),
                              _p(kv_cnt), kv_idx.shape[3], float(scale), b, h, i, _p(p))
    if st != 0:
        raise ValueError("routing entry outside the sample's blocks")
    return p


def keep_tokens(n_tokens: int, ratio: float) -> int:
    """Tokens kept by saliency pruning: clamp(ceil(ratio * n - 1e-9), 1, n)."""
    return int(_load().oracle_keep_tokens(int(n_tokens), float(ratio)))


def token_prune(x, valid_len=None, ratio: float = 0.5, npad_out: int | None = None):
    """Token pruning by feature-norm saliency (page "Sol Video Inference Engine", LTX-2.3
    appendix, stage 2: keep 50% of the video tokens by feat_norm).  x: bf16 bits
    [B, N, C].  Keeps the keep_tokens(L_b, ratio) tokens of largest squared norm
    (channel-order fp64 sum), ties to the lower index, in their original order.
    Returns (idx int32 [B, npad_out] ascending then -1, valid_out int32 [B],
    norm2 fp64 [B, N])."""
    x = np.ascontiguousarray(x)
    assert x.dtype == np.uint16 and x.ndim == 3, "bf16 bit patterns [B, N, C] expected"
    B, N, C = x.shape
    vl = np.full(B, N, dtype=np.int32) if valid_len is None else np.ascontiguousarray(valid_len, dtype=np.int32)
    if npad_out is None:
        npad_out = max(keep_tokens(int(L), ratio) for L in vl)
    idx = np.empty((B, npad_out), dtype=np.int32)
    vout = np.empty(B, dtype=np.int32)
    norm2 = np.empty((B, N))
    st = _load().oracle_token_prune(_p(x), B, N, C, _p(vl), float(ratio), int(npad_out), _p(norm2), _p(idx),
                                    _p(vout))
    if st != 0:
        raise ValueError("npad_out smaller than a kept count")
    return idx, vout, norm2
