"""bench.py's GPU arm at small sizes: one JSON line per run, with the keys the benchmark driver
reads (roofline of the dominant kernel, end-to-end number, launch count, clocks)."""
import json
import subprocess
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent


def run_bench(*args):
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), *args], capture_output=True, text=True,
                         cwd=ROOT, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def check_common(line, steps):
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "gpu_launches", "clocks"):
        assert key in line, key
    assert line["n_gpus"] == 1 and line["steps"] == steps and line["value"] > 0 and line["ms_per_step"] > 0
    assert line["scaling"] == "weak" and line["data"] == "synthetic" and "workload" in line["config"]
    rf = line["roofline"]
    assert rf["bound"] in ("tensor", "hbm") and rf["peak"] > 0 and rf["achieved"] > 0
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-9
    assert line["gpu_launches"] >= steps
    assert "sm_mhz" in line["clocks"] and "reasons" in line["clocks"]


@pytest.mark.gpu
def test_step_line_with_e2e():
    line = run_bench("--steps", "2", "--warmup", "3", "--seqlen", "512", "--headdim", "64", "--no-cpu-baseline")
    check_common(line, 2)
    assert line["dtype"] == "bf16" and line["gpu_launches"] == 4 * 2
    e2e = line["e2e"]
    B, H, N, d = (line["config"][k] for k in ("B", "H", "N", "d"))
    assert e2e["h2d_bytes_per_step"] == 4 * B * H * N * d * 2  # q, k, v, dO
    assert e2e["d2h_bytes_per_step"] == 4 * B * H * N * d * 2 + B * H * N * 4  # o, dq, dk, dv, lse
    assert 0 < e2e["value"] < line["value"]  # the host copies make the end-to-end step slower
    assert set(line["kernels"]) == {"fwd", "bwd_preprocess", "bwd_main", "bwd_dq_finish"}
    # the metric's curve: every sweep point and the named configurations, each timed on its own
    sw = line["sweep"]
    pts = {(p["N"], p["d"], p["causal"]) for p in sw["points"]}
    assert pts == {(n, d, c) for n in (512, 1024, 2048, 4096, 8192, 16384) for d in (64, 128) for c in (False, True)}
    for p in sw["points"]:
        assert p["B"] * p["N"] == 16384 and p["H"] * p["d"] == 2048
        assert 0 < p["fwd_tflops"] and 0 < p["fwd_bwd_tflops"]
        assert abs(p["pct_of_peak_fwd"] - 100 * p["fwd_tflops"] / sw["peak"]) < 0.1
    assert set(sw["configs"]) == {"bert_large_shape", "gpt2_shape_causal", "block_sparse", "head_dim_256",
                                  "head_dim_256_causal"}
    assert 0.2 < sw["configs"]["block_sparse"]["block_density"] < 0.35
    assert "sm_mhz" in sw["clocks"]


@pytest.mark.gpu
def test_forward_only_and_decode_lines():
    line = run_bench("--forward-only", "--headdim", "256", "--seqlen", "1024", "--steps", "2", "--warmup", "3")
    check_common(line, 2)
    assert line["config"]["d"] == 256 and line["roofline"]["bound"] == "tensor"
    line = run_bench("--decode", "1", "--seqlen", "4096", "--steps", "2", "--warmup", "3")
    check_common(line, 2)
    assert line["roofline"]["bound"] == "hbm" and line["unit"] == "GB/s"
