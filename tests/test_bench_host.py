"""bench.py's host-side contract on CPU: the reference arm (the oracle timed on
the host cores) prints one JSON line with the contract's keys, ranks other
than 0 print nothing, and the roofline inputs (measured peaks, stored DRAM
counters tied to the kernel source) are read as documented."""
import hashlib
import json
import os
import subprocess
import sys

from conftest import ROOT

BENCH = os.path.join(ROOT, "bench.py")


def _load_bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_under_test", BENCH)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_reference_arm_prints_the_contract_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, BENCH, "--impl", "reference", "--steps", "1", "--warmup", "0",
                          "--ref-tokens", "16"], capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["warmup"] >= 3 and d["steps"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["config"]["workload"].startswith("gdn_layer_prefill_B1_T32768")


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, BENCH, "--impl", "reference", "--steps", "1", "--warmup", "0"],
                         capture_output=True, text=True, timeout=300, env=env, cwd=ROOT)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_roofline_inputs():
    b = _load_bench()
    pk = b.peaks()
    measured = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    assert pk["source"] == "measured" and pk["hbm_gbs"] == measured["hbm_gbs"]
    assert pk["bf16_tflops"] == measured["bf16_tflops"]
    # the stored scan counters hold for the committed scan source only
    stored = [ln.split() for ln in open(os.path.join(ROOT, "profiles", "dram_traffic.txt"))
              if ln.strip() and not ln.startswith("#")]
    scan = [f for f in stored if f[0] == "scan"]
    assert len(scan) == 1
    # stored counters are used only while the kernel source still matches them
    src = os.path.join(ROOT, "nvfp4_w4a4_gated_b200", "csrc", "scan.cu")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    t0 = int(scan[0][3])
    assert b.traffic_for("scan", t0) == (float(scan[0][1]) if scan[0][2] == sha else None)
    # at 8x the tokens, 8x the bytes (the figure is scaled by the tokens processed)
    assert b.traffic_for("scan", 8 * t0) == (8 * float(scan[0][1]) if scan[0][2] == sha else None)
    assert b.traffic_for("gates", t0) is None

