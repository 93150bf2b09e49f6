"""bench.py's reference arm (the CPU oracle timed on bounded samples of the
step) prints the contract's JSON line; runs on the CPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in line, k
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"] == "gpt175b_block_linears_fp8_train_step"
    assert line["extrapolated"] is True and line["ms_per_full_step_extrapolated"] > line["ms_per_step"]
    # the reference arm's config is the GPU arm's (one function builds both)
    sys.path.insert(0, ROOT)
    import bench

    assert line["config"] == bench.config_of(bench.WORKLOADS["gpt175b_block"], "overlap", 1)
