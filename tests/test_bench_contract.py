"""The JSON line bench.py prints: the reference arm (the CPU oracle) on CPU,
and a one-layer run of the GPU arm on a GPU, checked for the keys and units
the benchmark contract asks for."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, timeout):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args,
                         capture_output=True, text=True, timeout=timeout, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


COMMON = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
          "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
          "cpu_baseline", "e2e"}


def test_reference_arm_line():
    d = _run(["--impl", "reference", "--steps", "1", "--warmup", "0"], 300)
    assert COMMON <= set(d) and d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == "stack28_m16384"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s",
                        "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


@pytest.mark.gpu
def test_gpu_arm_line_one_layer():
    d = _run(["--layers", "1", "--linears", "qkv", "--steps", "2", "--warmup", "3",
              "--no-cpu-baseline"], 600)
    assert COMMON <= set(d) and "impl" not in d
    assert d["value"] > 0 and d["gpu_launches"] == 6 * 2
    r = d["roofline"]
    assert r["bound"] in ("tensor", "hbm") and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert d["config"]["workload"] == "partial"        # one layer is not the workload
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["clocks"] is None or d["clocks"]["sm_mhz"] > 0
    assert set(d["next_rows"]) == {"wgrad_f32_accumulate", "gemm_fused_rowwise_quant",
                                   "gemm_fused_rowcol_quant", "pow2_step", "configs"}
    rows = d["next_rows"]["configs"]["rows"]
    assert set(rows) == {"qkv_m8192_quant_x_rowwise", "qkv_m8192_fprop"}
    assert rows["qkv_m8192_fprop"]["shape"] == [8192, 4096, 2048]
    assert all(r["achieved"] > 0 and ("frac_of_fp8_peak" in r or "frac_of_hbm" in r)
               for r in rows.values())
