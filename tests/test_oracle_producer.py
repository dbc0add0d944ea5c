"""Pins of the oracle's producer step: QK RMSNorm + 3D RoPE, rounding after the norm
and after the rotation (page "MiniMax-H3 on 8xH200 benchmark", the kernel layer:
fused QK RMSNorm and 3D RoPE, head dimension 128, RoPE dimension 96, norm rounded
before RoPE).  Each pin rests on something other than the oracle's own formula:
a brute-force nearest-bf16 search, rotation invariants, exact power-of-two
scalings, and the axis/frequency structure read back from the outputs."""
import math

import numpy as np
import pytest

from workloads import bf16_bits_to_f32, f64_to_bf16_bits, make_custom

D, RD = 128, 96
DA = RD // 3


def bf(x):
    return f64_to_bf16_bits(np.asarray(x, dtype=np.float64))


def f64(bits):
    return bf16_bits_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


def nearest_bf16(v):
    """Nearest bf16 value to v by search over neighbouring bit patterns (ties: even)."""
    u = np.array([v], dtype=np.float32).view(np.uint32)[0] >> 16
    best = None
    for c in range(max(0, int(u) - 2), int(u) + 3):
        if c > 0xFFFF:
            continue
        for sgn in (0, 0x8000):
            bits = (c & 0x7FFF) | sgn
            val = float(f64(bits).ravel()[0])
            if not math.isfinite(val):
                continue
            key = (abs(val - v), bits & 1)
            if best is None or key < best[0]:
                best = (key, bits)
    return best[1]


def one_row(xrow, w=None, pos=(0, 0, 0), rope_dim=RD, eps=1e-6, oracle_mod=None):
    x = bf(np.asarray(xrow)[None, None, None, :])
    w = bf(np.ones(D)) if w is None else bf(w)
    p = np.array(pos, dtype=np.int32)[None, None, :]
    o, o64 = oracle_mod.qk_norm_rope(x, w, p, rope_dim=rope_dim, eps=eps, return_unrounded=True)
    return o[0, 0, 0], o64[0, 0, 0]


@pytest.mark.parametrize("a", [1.0, -3.5, 0.001, 250.0])
def test_constant_row_norm_is_nearest_bf16(oracle_mod, a):
    """A constant row normalises to a / sqrt(a^2 + eps), rounded to the nearest bf16."""
    o, _ = one_row(np.full(D, a), rope_dim=0, oracle_mod=oracle_mod)
    aa = float(f64(bf(a)).ravel()[0])
    want = nearest_bf16(aa / math.sqrt(aa * aa + 1e-6))
    assert np.all(o == want)


def test_rounding_is_nearest_even_on_random_values(oracle_mod):
    rng = np.random.default_rng(0)
    xr = rng.normal(size=D) * 3
    o, o64 = one_row(xr, rope_dim=0, oracle_mod=oracle_mod)
    # with no rotation the unrounded output is the (already rounded) norm; check the norm's rounding
    xs = f64(bf(xr))
    inv = 1.0 / math.sqrt(np.mean(xs * xs) + 1e-6)
    for d in range(0, D, 7):
        assert o[d] == nearest_bf16(xs[d] * inv)


def test_position_zero_is_no_rotation(oracle_mod):
    rng = np.random.default_rng(1)
    xr = rng.normal(size=D)
    o_rot, _ = one_row(xr, pos=(0, 0, 0), oracle_mod=oracle_mod)
    o_norot, _ = one_row(xr, rope_dim=0, oracle_mod=oracle_mod)
    np.testing.assert_array_equal(o_rot, o_norot)


def test_rotation_preserves_pair_norms_and_angles(oracle_mod):
    rng = np.random.default_rng(2)
    xr = rng.normal(size=D)
    y, _ = one_row(xr, rope_dim=0, oracle_mod=oracle_mod)
    y = f64(y)
    pos = (3, 5, 7)
    _, o64 = one_row(xr, pos=pos, oracle_mod=oracle_mod)
    for d in range(0, D, 2):
        r0, r1 = np.hypot(y[d], y[d + 1]), np.hypot(o64[d], o64[d + 1])
        assert abs(r0 - r1) <= 1e-12 * max(1.0, r0)
        if d >= RD:
            assert o64[d] == y[d] and o64[d + 1] == y[d + 1]
            continue
        a, i = d // DA, (d % DA) // 2
        theta = pos[a] * 10000.0 ** (-2.0 * i / DA)
        got = math.atan2(y[d] * o64[d + 1] - y[d + 1] * o64[d], y[d] * o64[d] + y[d + 1] * o64[d + 1])
        diff = (got - theta + math.pi) % (2 * math.pi) - math.pi
        assert abs(diff) < 1e-9, (d, got, theta)


def test_single_axis_position_moves_only_that_axis(oracle_mod):
    rng = np.random.default_rng(3)
    xr = rng.normal(size=D)
    y, _ = one_row(xr, rope_dim=0, oracle_mod=oracle_mod)
    for axis in range(3):
        pos = [0, 0, 0]
        pos[axis] = 4
        o, _ = one_row(xr, pos=tuple(pos), oracle_mod=oracle_mod)
        moved = np.nonzero(o != y)[0]
        assert moved.size > 0
        assert moved.min() >= axis * DA and moved.max() < (axis + 1) * DA


def test_dot_products_depend_on_relative_position(oracle_mod):
    rng = np.random.default_rng(4)
    xq, xk = rng.normal(size=D), rng.normal(size=D)
    for (pq, pk, s) in [((2, 3, 4), (0, 1, 9), (5, -1, 2)), ((7, 0, 0), (1, 6, 2), (-3, 4, 10))]:
        _, q1 = one_row(xq, pos=pq, oracle_mod=oracle_mod)
        _, k1 = one_row(xk, pos=pk, oracle_mod=oracle_mod)
        _, q2 = one_row(xq, pos=tuple(a + b for a, b in zip(pq, s)), oracle_mod=oracle_mod)
        _, k2 = one_row(xk, pos=tuple(a + b for a, b in zip(pk, s)), oracle_mod=oracle_mod)
        assert abs(q1 @ k1 - q2 @ k2) <= 1e-11 * (1 + abs(q1 @ k1))


def test_power_of_two_scalings_are_exact(oracle_mod):
    rng = np.random.default_rng(5)
    xr = rng.normal(size=D)
    base, _ = one_row(xr, pos=(1, 2, 3), eps=0.0, oracle_mod=oracle_mod)
    scaled, _ = one_row(4.0 * f64(bf(xr)), pos=(1, 2, 3), eps=0.0, oracle_mod=oracle_mod)
    np.testing.assert_array_equal(base, scaled)  # RMSNorm is scale-free when eps = 0
    wt = rng.uniform(0.5, 1.5, size=D)
    o1, _ = one_row(xr, w=wt, pos=(1, 2, 3), oracle_mod=oracle_mod)
    o2, _ = one_row(xr, w=2.0 * f64(bf(wt)), pos=(1, 2, 3), oracle_mod=oracle_mod)
    np.testing.assert_array_equal(f64(o2), 2.0 * f64(o1))  # a doubled weight doubles every output


def test_workload_positions():
    w = make_custom(2, 1, 64, (2, 3, 4), 0.5, drop_rate=0.3, seed=9)
    for b in range(2):
        L = int(w.valid_len[b])
        t, y, x = w.positions[b, :L].T
        n = (t * 3 + y) * 4 + x
        assert np.all(np.diff(n) > 0) and n.max() < 24  # kept tokens, raster order
        assert np.all(w.positions[b, L:] == 0)


def test_bad_rope_dim_rejected(oracle_mod):
    w = make_custom(1, 1, 128, (1, 4, 16), 0.5, seed=1)
    with pytest.raises(ValueError):
        oracle_mod.qk_norm_rope(w.q, bf(np.ones(128)), w.positions, rope_dim=100)
