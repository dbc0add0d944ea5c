"""The seeded synthetic inputs: bf16 rounding of the generator, the five configurations'
shapes, padding and lengths, determinism, and the scale of the field."""
import math
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from workloads import CONFIGS, bf16_bits_to_f32, f64_to_bf16_bits, make_workload  # noqa: E402


def _normal_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    exp = (bits >> 7) & 0xFF
    return bits[(exp > 0) & (exp < 255)]


def test_bf16_exact_values_round_trip():
    bits = _normal_bf16()
    v = bf16_bits_to_f32(bits).astype(np.float64)
    assert np.array_equal(f64_to_bf16_bits(v), bits)


def test_bf16_round_to_nearest_even():
    pos = np.sort(_normal_bf16()[(_normal_bf16() & 0x8000) == 0])   # positive, ascending
    lo = bf16_bits_to_f32(pos[:-1]).astype(np.float64)
    hi = bf16_bits_to_f32(pos[1:]).astype(np.float64)
    mid = (lo + hi) / 2                                               # exact in fp64
    even = np.where((pos[:-1] & 1) == 0, pos[:-1], pos[1:])
    assert np.array_equal(f64_to_bf16_bits(mid), even)
    step = (hi - lo) * 2.0 ** -20
    assert np.array_equal(f64_to_bf16_bits(mid - step), pos[:-1])
    assert np.array_equal(f64_to_bf16_bits(mid + step), pos[1:])
    assert np.array_equal(f64_to_bf16_bits(-mid), even | 0x8000)
    assert f64_to_bf16_bits(np.array([0.0]))[0] == 0


@pytest.mark.parametrize("name", list(CONFIGS))
def test_config_shapes_and_padding(name):
    c = CONFIGS[name]
    w = make_workload(name, heads=1)
    T, Hg, Wg = c["grid"]
    N = T * Hg * Wg
    assert w.q.shape[:2] == (c["B"], 1) and w.q.shape[3] == c["D"]
    assert w.q.shape == w.k.shape == w.v.shape
    assert w.Npad == 64 * math.ceil(int(w.valid_len.max()) / 64)
    if c["drop_rate"] == 0.0:
        assert np.all(w.valid_len == N)
    else:
        # Bernoulli(0.15) drops per token: about N * 0.85, within 5 sigma, and ragged
        mu, sd = N * (1 - c["drop_rate"]), math.sqrt(N * c["drop_rate"] * (1 - c["drop_rate"]))
        assert np.all(np.abs(w.valid_len - mu) < 5 * sd)
        assert len(set(w.valid_len.tolist())) == c["B"]
    for b in range(c["B"]):
        assert np.all(w.q[b, :, w.valid_len[b]:] == 0) and np.all(w.v[b, :, w.valid_len[b]:] == 0)


def test_deterministic_and_scaled():
    a = make_workload("480p_dense", heads=1)
    b = make_workload("480p_dense", heads=1)
    assert np.array_equal(a.q, b.q) and np.array_equal(a.k, b.k) and np.array_equal(a.v, b.v)
    # eight sinusoids of amplitude 0.5 give the field unit variance; noise sigma 0.5 adds 0.25
    x = bf16_bits_to_f32(a.q[0, 0, :a.valid_len[0]]).astype(np.float64)
    assert 0.9 < x.var() < 1.6
    assert abs(x.mean()) < 0.2
