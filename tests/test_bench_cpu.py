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
    pk = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    r = bench.stage_rooflines({"hessian": 3.0, "prepare_hinv": 2.0, "quantize_layer": 1.0, "pack": 0.01},
                              rows=4096, n=4096, bits=4, ng=32, pk=pk)
    assert r["factorization"]["peak"] == 1600.0
    assert abs(r["factorization"]["achieved"] - 2 * 4096 ** 3 / 3 / 2e-3 / 1e12) < 1e-6
    assert abs(r["factorization"]["tf32_issue_frac"] - 3 * r["factorization"]["achieved"] / (1600 * 1.1 / 2.25)) < 1e-12
    # codes and zeros read (1 byte each), 512 + 4 packed words per row written
    assert r["pack"]["algorithmic_bytes"] == 4096 * 4096 + 4096 * 32 + 4 * 4096 * (512 + 4)
    assert abs(r["pack"]["frac"] - r["pack"]["achieved"] / 6000.0) < 1e-12


def test_trailing_flops_is_the_sum_over_blocks():
    sys.path.insert(0, ROOT)
    import bench
    # square, block-divisible: rows * n * (n - B)
    assert bench.trailing_flops(4096, 4096, 128) == 4096 * 4096 * (4096 - 128)
    # ragged: blocks of 128, 128, 44 -> 2 rows (128 * 172 + 128 * 44)
    assert bench.trailing_flops(10, 300, 128) == 2 * 10 * (128 * 172 + 128 * 44)


def test_kernel_rooflines_from_a_trace():
    sys.path.insert(0, ROOT)
    import bench
    pk = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    trace = {"syrk_tc_kernel": (2, 6.0), "chol_tc_kernel": (2, 2.0), "trailing_tc_kernel": (62, 1.0),
             "gptq_block_kernel<16>": (64, 1.8), "pack_kernel<4>": (4, 0.03)}
    r = bench.kernel_rooflines(trace, 2, rows=4096, n=4096, n_tok=262144, bits=4, ng=32, block=128, pk=pk,
                               sms=148, mhz=1965.0)
    assert r["syrk_tc_kernel"]["ms"] == 3.0 and r["syrk_tc_kernel"]["launches"] == 1
    assert abs(r["syrk_tc_kernel"]["achieved"] - 4096 * 4097 * 262144 / 3e-3 / 1e12) < 1e-6
    assert r["gptq_block_kernel"]["launches"] == 32 and abs(r["gptq_block_kernel"]["ms"] - 0.9) < 1e-12
    assert abs(r["trailing_tc_kernel"]["achieved"] - 4096 * 4096 * 3968 / 0.5e-3 / 1e12) < 1e-6
    assert r["pack_kernel"]["launches"] == 2
