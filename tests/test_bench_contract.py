"""bench.py's output contract, checked on CPU through the reference arm (the fp64 oracle on
host cores): one JSON line with the keys the benchmark driver reads."""
import json
import subprocess
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parent.parent


def run_bench(*args):
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), *args], capture_output=True, text=True,
                         cwd=ROOT, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


def test_reference_arm_prints_one_contract_line():
    line = run_bench("--impl", "reference", "--steps", "1", "--warmup", "3", "--seqlen", "512", "--headdim", "64")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and "head" in cb["sample"]
    assert line["config"]["workload"].startswith("seq-len sweep")


def test_warmup_below_three_is_refused():
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), "--warmup", "2"], capture_output=True, text=True,
                         cwd=ROOT, timeout=120)
    assert out.returncode != 0 and "warmup" in out.stderr


def test_traffic_record_matches_the_current_backward_code(tmp_path, monkeypatch):
    # The roofline's DRAM traffic comes from profiles/traffic.json, keyed to a hash of the
    # backward's code without comments: the committed record must match the committed code,
    # a comment edit must keep the key, and a code edit must retire it.
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", ROOT / "bench.py")
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    key = "bwd_main N=4096 d=128 causal=0 bs=0"
    assert bench.recorded_traffic(key) is not None
    h0 = bench.kernel_source_hash()
    src = tmp_path / "exact_attention_110_b200" / "csrc"
    src.mkdir(parents=True)
    for f in ("fa_bwd.cu", "ptx.cuh"):
        (src / f).write_text((ROOT / "exact_attention_110_b200" / "csrc" / f).read_text())
    monkeypatch.setattr(bench, "ROOT", tmp_path)
    assert bench.kernel_source_hash() == h0
    bwd = src / "fa_bwd.cu"
    bwd.write_text(bwd.read_text() + "\n// a comment\n/* and a block\n comment */\n")
    assert bench.kernel_source_hash() == h0
    bwd.write_text(bwd.read_text() + "\nstatic int fa_unused_probe = 1;\n")
    assert bench.kernel_source_hash() != h0
