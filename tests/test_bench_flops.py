"""bench.py's host arithmetic on the CPU.  The metric's FLOP count (kept_flops): 4 D for
every (query token, kept key token) pair of valid tokens, pinned by the dense closed form --
including the 480p dense figure of 4 * 128 * 24 * 32760^2 = 1.319e13 FLOPs -- and by
brute-force enumeration of token pairs; the whole-job value; and the clock summary read
from nvidia-smi lines."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def dense_routing(B, H, nQ):
    idx = np.broadcast_to(np.arange(nQ, dtype=np.int32), (B, H, nQ, nQ)).copy()
    return idx, np.full((B, H, nQ), nQ, dtype=np.int32)


def test_dense_closed_form_480p():
    nQ, L = 512, 32760
    idx, cnt = dense_routing(1, 24, nQ)
    assert bench.kept_flops(idx, cnt, np.array([L]), 128) == 4 * 128 * 24 * L * L
    assert abs(4 * 128 * 24 * L * L - 1.319e13) / 1.319e13 < 1e-3


def test_ragged_partial_block():
    # one sample of 100 tokens: blocks of 64 and 36 valid tokens; a second of 64
    idx, cnt = dense_routing(2, 1, 2)
    cnt[1, :, 1] = 0                      # block 1 of sample 1 lies past its length
    cnt[1, :, 0] = 1
    f = bench.kept_flops(idx, cnt, np.array([100, 64]), 64)
    assert f == 4 * 64 * (100 * 100 + 64 * 64)


def test_brute_force_token_pairs():
    rng = np.random.default_rng(5)
    B, H, nQ, D, kmax = 2, 3, 5, 64, 3
    vl = np.array([300, 201])
    idx = np.zeros((B, H, nQ, kmax), dtype=np.int32)
    cnt = np.zeros((B, H, nQ), dtype=np.int32)
    for b in range(B):
        nb = (vl[b] + 63) // 64
        for h in range(H):
            for I in range(nb):
                k = int(rng.integers(1, min(kmax, nb) + 1))
                sel = np.sort(rng.choice(nb, size=k, replace=False))
                idx[b, h, I, :k] = sel
                cnt[b, h, I] = k
    pairs = 0
    for b in range(B):
        for h in range(H):
            for i in range(vl[b]):
                kept = set(idx[b, h, i // 64, :cnt[b, h, i // 64]].tolist())
                pairs += sum(1 for j in range(vl[b]) if j // 64 in kept)
    assert bench.kept_flops(idx, cnt, vl, D) == 4 * D * pairs


def test_whole_job_value_sums_replicas():
    assert bench.whole_job_value(2e12, 4.0, 1) == 2e12 / 4e-3 / 1e12
    assert bench.whole_job_value(2e12, 4.0, 8) == 8 * 2e12 / 4e-3 / 1e12


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


class _FakeThread:
    def join(self, timeout=None):
        pass


def test_clock_sampler_window_and_reasons():
    """Only samples inside the timed window (widened by one interval) count; throttle
    reasons are read from their columns; malformed lines are skipped."""
    cs = bench.ClockSampler(0)
    cs.proc, cs.thread = _FakeProc(), _FakeThread()
    active = "Active"
    idle = "Not Active"
    cs.lines = [
        (0.50, f"0, 900, 1965, 400.0, 0x1, {active}, {idle}, {idle}, {idle}"),      # before the window
        (1.00, f"0, 1965, 1965, 700.0, 0x4, {idle}, {idle}, {idle}, {active}"),
        (1.05, f"0, 1800, 1965, 950.5, 0x4, {idle}, {idle}, {idle}, {active}"),
        (1.08, "0, [N/A], 1965"),                                                    # malformed
        (1.10, f"0, 1700, 1965, [N/A], 0x40, {idle}, {active}, {idle}, {idle}"),
        (3.00, f"0, 500, 1965, 100.0, 0x8, {idle}, {idle}, {active}, {idle}"),     # after the window
    ]
    cs.mark(0.95, 1.05)
    r = cs.stop()
    assert r["samples"] == 3
    assert r["sm_mhz"] == 1800.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]


def test_clock_sampler_without_nvidia_smi():
    cs = bench.ClockSampler(0)
    r = cs.stop()
    assert r["sm_mhz"] is None and r["reasons"] == ["nvidia-smi unavailable"]
