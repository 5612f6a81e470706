"""The JSON line bench.py prints is what the driver reads: its keys and
their types. The reference arm (the CPU oracle) runs here without a GPU; the
GPU arm is checked on the small workload on a GPU."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=600):
    r = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True, text=True,
                       timeout=timeout)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def check_common(d):
    for key, typ in (("metric", str), ("value", float), ("unit", str), ("n_gpus", int), ("steps", int),
                     ("warmup", int), ("higher_is_better", bool), ("scaling", str), ("dtype", str),
                     ("data", str), ("config", dict)):
        assert key in d and isinstance(d[key], typ), f"{key}: {d.get(key)!r}"
    assert d["value"] > 0 and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["vs_baseline"] is None
    assert d["config"]["workload"] and d["data"] == "synthetic"
    e2e = d["e2e"]
    assert e2e["unit"] == d["unit"] and e2e["value"] > 0
    assert isinstance(e2e["h2d_bytes_per_step"], int) and isinstance(e2e["d2h_bytes_per_step"], int)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0 and cb["sample"]


def test_reference_arm_line():
    d = run_bench("--impl", "reference", "--config", "tiny_mha", "--steps", "1", "--warmup", "1")
    check_common(d)
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["n_gpus"] == 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["cpu_baseline"]["value"] == d["value"]


@pytest.mark.gpu
def test_gpu_arm_line():
    d = run_bench("--config", "tiny_mha", "--steps", "5", "--warmup", "3", "--cpu-seconds", "2",
                  "--no-clock-window")
    check_common(d)
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] >= 3 and d["scaling"] == "weak"
    assert d["dtype"] == "bf16" and d["ms_per_step"] > 0
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert r["traffic"] is None or r["traffic"] > 0
    assert isinstance(d["gpu_launches"], int) and d["gpu_launches"] >= d["steps"]
    clocks = d["clocks"]
    assert set(("sm_mhz", "sm_max_mhz", "reasons")) <= set(clocks)
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    p = d["parity"]
    assert p["max_abs_err_out"] <= p["tolerance"]["out_abs"] and p["max_rel_err_lse"] <= p["tolerance"]["lse_rel"]
    assert d["per_call"]["median_us"] > 0 and d["read_probe"]["gbs"] > 0


def test_launch_bytes_average_the_rotated_copies():
    """The timed calls alternate over input copies; on a ragged workload the
    copies' lengths differ, so one launch's algorithmic bytes are their mean.
    K/V bytes are counted inside the sequences only (2 bytes per bf16
    element, K and V)."""
    import numpy as np

    import bench
    from decode_attention_07_b200.configs import WORKLOADS

    w = WORKLOADS["ragged_64k"]
    a = np.array([1, 65536] + [4096] * (w.B - 2), dtype=np.int32)
    b = np.array([777] * w.B, dtype=np.int32)
    S = 148
    kv = lambda lens: int(lens.astype(np.int64).sum()) * w.Hkv * w.D * 2 * 2
    one = bench.launch_bytes(w, [a], S)
    assert one == bench.byte_counts(w, a, S) and one["kv"] == kv(a)
    two = bench.launch_bytes(w, [a, b], S)
    assert two["kv"] == (kv(a) + kv(b)) / 2
    assert two["total"] == (bench.byte_counts(w, a, S)["total"] + bench.byte_counts(w, b, S)["total"]) / 2
    assert two["q"] == w.B * w.Hq * w.D * 2
