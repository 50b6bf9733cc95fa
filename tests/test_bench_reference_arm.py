"""The benchmark's reference arm (the CPU oracle on the host cores) keeps the
one-JSON-line contract: a whole sweep per step, a measured step time, and the
cpu_baseline / e2e objects describing this run.  Runs on the CPU only."""
import json
import os
import subprocess
import sys

from nvfp4_block_scaled_gemm_b200 import accounting, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["steps"] == 1 and d["warmup"] == 3 and d["n_gpus"] == 1
    assert d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["ms_per_step"] > 0
    # GB/s = algorithmic bytes of the six-GEMM sweep / measured step time
    step_bytes = sum(accounting.gemm_bytes(m, synth.ATTN_N, synth.HIDDEN_K) for m in synth.ATTN_SWEEP_M)
    assert abs(d["value"] - step_bytes / (d["ms_per_step"] * 1e6)) / d["value"] < 0.01
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    assert d["config"]["M"] == [1, 16, 64, 128, 256, 512] and d["config"]["N"] == 768 and d["config"]["K"] == 6144
