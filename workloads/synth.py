"""Seeded smooth-field + noise video-token workloads.

Each of Q, K and V, for every sample b, head h and channel c, is the field

    x(t, y, w) = sum_{m=1..8} 0.5 * sin(2*pi*(f_t*t/T + f_y*y/Hg + f_w*w/Wg) + phi_m) + sigma * eps

evaluated on the latent grid (t, y, w) in T x Hg x Wg, flattened in raster order
n = (t*Hg + y)*Wg + w (the spatio-temporal token lattice is left unpermuted), then
rounded to bf16 with round-to-nearest-even.  Eight sinusoids of amplitude 0.5 give the
field unit variance; eps ~ N(0, 1).

Draw recipe (every stream is its own numpy PCG64 generator keyed by a SeedSequence):
  * frequencies f ~ U[0, 3) cycles per axis extent, 8 x 3 per channel, keyed by
    (seed, 1, tensor, b) when shared across heads, or (seed, 2, tensor, b, h) per head;
  * phases phi ~ U[0, 2*pi), 8 per channel, keyed by (seed, 3, tensor, b, h);
  * noise eps, [N, D] float32 standard normals, keyed by (seed, 4, tensor, b, h);
  * token pruning (long clips): token n of sample b is dropped when a U[0,1) draw from
    the generator seeded with seed*31 + b is below the drop rate; kept tokens are
    compacted in raster order, and every sample is padded with zeros to
    Npad = 64*ceil(max_b L_b / 64).
Because every (tensor, b, h) stream is independent, a subset of heads is bit-identical
to the same heads of the full draw.

Nothing here computes any part of the attention method.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np

BLOCK = 64

TENSORS = ("q", "k", "v")

# name -> (B, H, D, (T, Hg, Wg), sparsity, sigma, per_head_freq, drop_rate, index)
CONFIGS = {
    "tiny": dict(B=1, H=2, D=64, grid=(4, 16, 16), sparsity=0.5, sigma=0.5,
                 per_head_freq=False, drop_rate=0.0, index=0),
    "480p_dense": dict(B=1, H=24, D=128, grid=(21, 30, 52), sparsity=0.0, sigma=0.5,
                       per_head_freq=False, drop_rate=0.0, index=1),
    "480p_sparse": dict(B=1, H=24, D=128, grid=(21, 30, 52), sparsity=0.75, sigma=0.5,
                        per_head_freq=True, drop_rate=0.0, index=2),
    "720p": dict(B=1, H=40, D=128, grid=(21, 45, 80), sparsity=0.80, sigma=0.3,
                 per_head_freq=False, drop_rate=0.0, index=3),
    "long_clip": dict(B=2, H=32, D=128, grid=(31, 34, 60), sparsity=0.75, sigma=0.5,
                      per_head_freq=False, drop_rate=0.15, index=4),
}

BASE_SEED = 20261202


@dataclasses.dataclass
class Workload:
    """Host-side bf16 inputs of one problem.

    q, k, v: uint16 bf16 bit patterns, [B, H, Npad, D], C-contiguous.
    valid_len: int32 [B]; rows n >= valid_len[b] are padding.
    """
    name: str
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    valid_len: np.ndarray
    sparsity: float
    block: int = BLOCK
    grid: tuple = ()
    seed: int = 0
    # int32 [B, Npad, 3]: (t, y, x) latent-grid position of each kept token (raster
    # order n = (t*Hg + y)*Wg + x before pruning); padding rows are (0, 0, 0)
    positions: np.ndarray | None = None

    @property
    def B(self):
        return self.q.shape[0]

    @property
    def H(self):
        return self.q.shape[1]

    @property
    def Npad(self):
        return self.q.shape[2]

    @property
    def D(self):
        return self.q.shape[3]


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 with round-to-nearest-even, directly from the
    binary64 encoding (no intermediate float32 rounding).  Normal-range values only."""
    b = np.ascontiguousarray(x, dtype=np.float64).view(np.uint64)
    keep = b >> np.uint64(45)                       # sign | 11-bit exponent | 7 mantissa bits
    low = b & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    keep += (low > half) | ((low == half) & (keep & np.uint64(1)).astype(bool))
    # re-bias the exponent (1023 -> 127) in the combined exponent|mantissa field
    em = (keep & np.uint64(0x3FFFF)).astype(np.int64) - ((1023 - 127) << 7)
    zero = (b << np.uint64(1)) == np.uint64(0)
    if np.any(~zero & ((em < (1 << 7)) | (em > (254 << 7) + 127))):
        raise ValueError("value outside the bf16 normal range")
    em[zero] = 0
    return (((keep >> np.uint64(18)) << np.uint64(15)) | em.astype(np.uint64)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(*key):
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _field(grid, freqs, phases):
    """Smooth part of one (tensor, b, h) field, float64 [T*Hg*Wg, D].

    freqs [D, 8, 3] (cycles per axis extent), phases [D, 8].  Uses
    sin(a + b) = sin a cos b + cos a sin b with a = (t, y) part + phase and
    b = w part, so the sum over the 8 sinusoids is one small matmul per channel."""
    T, Hg, Wg = grid
    t = np.arange(T, dtype=np.float64)[:, None] / T
    y = np.arange(Hg, dtype=np.float64)[None, :] / Hg
    w = np.arange(Wg, dtype=np.float64) / Wg
    ty = 2 * np.pi * (freqs[:, :, 0, None, None] * t + freqs[:, :, 1, None, None] * y)
    a = (ty + phases[:, :, None, None]).reshape(freqs.shape[0], 8, T * Hg)      # [D, 8, TH]
    bw = 2 * np.pi * freqs[:, :, 2, None] * w                                    # [D, 8, W]
    lhs = np.concatenate([np.sin(a), np.cos(a)], axis=1).transpose(0, 2, 1)      # [D, TH, 16]
    rhs = np.concatenate([np.cos(bw), np.sin(bw)], axis=1)                      # [D, 16, W]
    x = 0.5 * np.matmul(lhs, rhs)                                                # [D, TH, W]
    return x.reshape(freqs.shape[0], T * Hg * Wg).T                             # [N, D]


def _build(name, B, H, D, grid, sparsity, sigma, per_head_freq, drop_rate, seed,
           heads=None, pad_value=0.0):
    T, Hg, Wg = grid
    N = T * Hg * Wg
    hsel = list(range(H)) if heads is None else list(range(heads))
    keep_rows = []
    for b in range(B):
        if drop_rate > 0.0:
            u = _rng(seed * 31 + b).random(N)
            keep_rows.append(np.nonzero(u >= drop_rate)[0])
        else:
            keep_rows.append(np.arange(N))
    valid_len = np.array([len(r) for r in keep_rows], dtype=np.int32)
    Npad = BLOCK * int(math.ceil(valid_len.max() / BLOCK))
    pad_bits = f64_to_bf16_bits(np.array([pad_value]))[0]
    out = {t: np.full((B, len(hsel), Npad, D), pad_bits, dtype=np.uint16) for t in TENSORS}

    def one(job):
        ti, b, hi, h = job
        if per_head_freq:
            fr = _rng(seed, 2, ti, b, h).uniform(0.0, 3.0, size=(D, 8, 3))
        else:
            fr = _rng(seed, 1, ti, b).uniform(0.0, 3.0, size=(D, 8, 3))
        ph = _rng(seed, 3, ti, b, h).uniform(0.0, 2 * np.pi, size=(D, 8))
        eps = _rng(seed, 4, ti, b, h).standard_normal((N, D), dtype=np.float32)
        x = _field(grid, fr, ph) + sigma * eps.astype(np.float64)
        rows = keep_rows[b]
        out[TENSORS[ti]][b, hi, :len(rows)] = f64_to_bf16_bits(x[rows])

    jobs = [(ti, b, hi, h) for ti in range(3) for b in range(B) for hi, h in enumerate(hsel)]
    # numpy releases the GIL in the heavy kernels: threads give real parallelism, and
    # every job owns its own generators, so the result does not depend on scheduling.
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        list(ex.map(one, jobs))
    pos = np.zeros((B, Npad, 3), dtype=np.int32)
    for b in range(B):
        r = keep_rows[b]
        pos[b, :len(r)] = np.stack([r // (Hg * Wg), (r // Wg) % Hg, r % Wg], axis=1)
    return Workload(name=name, q=out["q"], k=out["k"], v=out["v"], valid_len=valid_len,
                    sparsity=float(sparsity), grid=tuple(grid), seed=seed, positions=pos)


def make_hidden(B: int, grid, C: int, seed: int = 5, sigma: float = 0.5, chunk: int = 256) -> np.ndarray:
    """Token feature vectors of the whole latent grid (before any pruning), the input
    of saliency pruning: bf16 bits [B, T*Hg*Wg, C], each channel the same smooth field +
    sigma N(0,1) recipe as Q, K and V, in raster order.  Channels are drawn in chunks of
    `chunk` from generators of their own, so the result does not depend on threading."""
    T, Hg, Wg = grid
    N = T * Hg * Wg
    out = np.empty((B, N, C), dtype=np.uint16)

    def one(job):
        b, c0 = job
        c1 = min(C, c0 + chunk)
        fr = _rng(seed, 21, b, c0).uniform(0.0, 3.0, size=(c1 - c0, 8, 3))
        ph = _rng(seed, 22, b, c0).uniform(0.0, 2 * np.pi, size=(c1 - c0, 8))
        eps = _rng(seed, 23, b, c0).standard_normal((N, c1 - c0), dtype=np.float32)
        out[b, :, c0:c1] = f64_to_bf16_bits(_field(grid, fr, ph) + sigma * eps.astype(np.float64))

    jobs = [(b, c0) for b in range(B) for c0 in range(0, C, chunk)]
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        list(ex.map(one, jobs))
    return out


def make_norm_weights(D: int, seed: int = 7):
    """Per-channel RMSNorm weights for Q and K: bf16 bits [D] each, drawn from
    U[0.5, 1.5) (learned QK-norm scales sit near 1)."""
    wq = f64_to_bf16_bits(_rng(seed, 11).uniform(0.5, 1.5, size=D))
    wk = f64_to_bf16_bits(_rng(seed, 12).uniform(0.5, 1.5, size=D))
    return wq, wk


def make_workload(name: str, heads: int | None = None, pad_value: float = 0.0) -> Workload:
    """One of the five named problems; `heads` keeps only the first `heads` heads."""
    c = CONFIGS[name]
    return _build(name, c["B"], c["H"], c["D"], c["grid"], c["sparsity"], c["sigma"],
                  c["per_head_freq"], c["drop_rate"], BASE_SEED + c["index"],
                  heads=heads, pad_value=pad_value)


def make_custom(B, H, D, grid, sparsity, sigma=0.5, per_head_freq=False, drop_rate=0.0,
                seed=1, pad_value=0.0, name="custom") -> Workload:
    """A problem of any shape drawn with the same recipe (for parity sweeps)."""
    return _build(name, B, H, D, grid, sparsity, sigma, per_head_freq, drop_rate, seed,
                  pad_value=pad_value)
