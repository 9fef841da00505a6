"""bench.py's reference arm (the fp64 oracle on a bounded sample) runs on the
CPU and prints one JSON line with the fields the benchmark contract asks for."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["value"] > 0 and d["unit"] == "weights/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert "workload" in d["config"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["e2e"]["d2h_bytes_per_step"] == 0


def test_stage_rooflines_arithmetic():
    sys.path.insert(0, ROOT)
    import bench
    r = bench.stage_rooflines({"hessian": 3.0, "prepare_hinv": 2.0, "quantize_layer": 1.0, "pack": 0.01},
                              rows=4096, n=4096, bits=4, ng=32, sms=148, mhz=2000.0, hbm_gbs=6000.0)
    assert abs(r["factorization"]["peak"] - 148 * 256 * 2.0e9 / 1e12) < 1e-9
    assert abs(r["factorization"]["achieved"] - 2 * 4096 ** 3 / 3 / 2e-3 / 1e12) < 1e-6
    # codes and zeros read (1 byte each), 512 + 4 packed words per row written
    assert r["pack"]["algorithmic_bytes"] == 4096 * 4096 + 4096 * 32 + 4 * 4096 * (512 + 4)
    assert abs(r["pack"]["frac"] - r["pack"]["achieved"] / 6000.0) < 1e-12
