"""Shared helpers of the GPU parity tests (no method arithmetic here)."""
import numpy as np

# Output tolerance against the fp64 oracle fed the GPU routing, for bf16 inputs.
MAX_ABS = 2e-2
MEAN_ABS = 2e-3
# Score gap below which a routing difference counts as a tie (relative).
TIE_REL = 1e-6


def to_device(w, dev):
    import torch
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev).view(torch.bfloat16)
    return t(w.q), t(w.k), t(w.v), torch.from_numpy(np.ascontiguousarray(w.valid_len)).to(dev)


def compare_routing(idx_g, cnt_g, idx_o, cnt_o, scores=None):
    """Row-by-row comparison of two routings.  Returns (bad_rows, excused_rows).

    A row whose kept sets differ is excused only when every differing block's
    oracle score lies within TIE_REL (relative) of the oracle's k-th score."""
    bad, excused = [], []
    if not np.array_equal(cnt_g, cnt_o):
        rows = np.argwhere(cnt_g != cnt_o)
        return [tuple(r) for r in rows], []
    for r in np.ndindex(cnt_o.shape):
        c = int(cnt_o[r])
        a = set(idx_o[r][:c].tolist())
        g = set(idx_g[r][:c].tolist())
        if a == g and list(idx_g[r][:c]) == sorted(g):
            continue
        if scores is None or list(idx_g[r][:c]) != sorted(g):
            bad.append(r)
            continue
        row = scores[r]
        tau = np.sort(row[np.isfinite(row)])[::-1][c - 1]
        diff = (a - g) | (g - a)
        if all(abs(row[j] - tau) <= TIE_REL * max(abs(row[j]), abs(tau)) for j in diff):
            excused.append(r)
        else:
            bad.append(r)
    return bad, excused


def output_errors(o_gpu, o_ref, rows_mask=None):
    """(max_abs, mean_abs) of the GPU bf16 output against the fp64 oracle."""
    o = o_gpu.astype(np.float64)
    if rows_mask is not None:
        o, o_ref = o[rows_mask], o_ref[rows_mask]
    e = np.abs(o - o_ref)
    return float(e.max()) if e.size else 0.0, float(e.mean()) if e.size else 0.0
