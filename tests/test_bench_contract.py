"""bench.py's JSON line carries the keys and types its consumers rely on: the reference
arm on the CPU, our arm on the GPU (tiny workload, a few steps)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric": str, "value": float, "unit": str, "n_gpus": int, "steps": int, "warmup": int,
             "ms_per_step": float, "higher_is_better": bool, "scaling": str, "dtype": str, "data": str,
             "config": dict}


def _run(args, timeout):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def _check_base(d):
    for k, t in BASE_KEYS.items():
        assert k in d, k
        assert isinstance(d[k], t) or (t is float and isinstance(d[k], int)), (k, type(d[k]))
    assert "vs_baseline" in d and d["vs_baseline"] is None
    assert d["config"]["workload"] == "tiny"
    assert d["higher_is_better"] is True and d["scaling"] == "weak"


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--config", "tiny", "--steps", "1", "--warmup", "0"], 600)
    _check_base(d)
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["value"] > 0
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.gpu
def test_our_arm_line():
    d = _run(["--config", "tiny", "--steps", "3", "--warmup", "3"], 900)
    _check_base(d)
    assert "impl" not in d and d["dtype"] == "bf16" and d["n_gpus"] == 1 and d["value"] > 0
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert "traffic" in r
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["unit"] == d["unit"] and cb["cores"] >= 1 and cb["sample"]
    e = d["e2e"]
    assert e["unit"] == d["unit"] and e["value"] > 0
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert isinstance(d["gpu_launches"], int) and d["gpu_launches"] > 0
    c = d["clocks"]
    assert "sm_mhz" in c and "sm_max_mhz" in c and isinstance(c["reasons"], list)
    p = d["parity"]
    assert p["mask_rows"] > 0 and p["mask_mismatch"] == 0 and p["ok"] is True
    assert p["max_abs"] <= 2e-2 and p["mean_abs"] <= 2e-3 and p["out_rows"] > 0
    m = d["median_ms"]
    assert m["step"] > 0 and m["attn"] > 0 and m["select"] > 0
    r = m["rounds"]
    assert r["n"] >= 1 and r["steps_each"] >= 1 and r["step"] > 0 and r["attn"] > 0
    f = m["l2_flushed"]
    assert f["n"] == r["n"] and f["flush_bytes"] >= 4 * 126 * 10**6
    assert f["step"] > 0 and f["attn"] > 0 and f["routing_call"] > 0 and f["attn_tflops"] > 0
    assert d["routing"]["pool_select_ms"] > 0 and d["routing"]["pair_ms"] > 0


@pytest.mark.gpu
def test_our_arm_line_with_pruning():
    """--prune: saliency pruning and the gathers inside every step; the parity block
    also checks the pruned index lists against the oracle."""
    d = _run(["--config", "tiny", "--steps", "3", "--warmup", "3", "--prune", "0.5", "--no-cpu-baseline"], 900)
    _check_base(d)
    assert d["prune_ms"] > 0 and d["config"]["pruning"]["ratio"] == 0.5
    assert d["config"]["pruning"]["valid_len_after"] == [512]
    p = d["parity"]
    assert p["prune_index_exact"] is True and p["ok"] is True and p["mask_mismatch"] == 0
