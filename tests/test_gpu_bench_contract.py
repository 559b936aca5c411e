"""bench.py's JSON line on a short run: every key the benchmark contract names, with sane values.

Runs the benchmark once in a subprocess (few steps, no extra workloads) and checks the line rank 0
prints: the headline metric, its roofline with the measured peak, the end-to-end number with the
bytes it copies, the decode and speculative-decode objects, the launch count and the clocks."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "3", "--warmup", "3",
                        "--no-extra", "--no-cpu-baseline", "--decode-steps", "8"],
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_headline_keys(line):
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in line, k
    assert line["n_gpus"] == 1 and line["steps"] == 3 and line["warmup"] >= 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["config"]["workload"] == "prefill_B1_T8192_H32_d128_bf16"
    assert line["gpu_launches"] > 0


def test_roofline_and_e2e(line):
    rf = line["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in rf, k
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s"
    assert 0 < rf["frac"] < 1.5 and abs(rf["achieved"] / rf["peak"] - rf["frac"]) < 1e-9
    e = line["e2e"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert 0 < e["value"] < line["value"]  # the copies are inside its timed region
    assert 0 < e["frac_of_upload_bound"] <= 1.05


def test_decode_objects(line):
    d = line["decode"]
    assert d["ms_per_step"] > 0 and 0 < d["roofline"]["frac"] < 1.5
    s = line["speculative_decode"]
    for k in ("verify_ms", "commit_ms", "ms_per_step", "speedup_vs_single_steps"):
        assert s[k] > 0, k


def test_clocks_sampled(line):
    c = line["clocks"]  # nvidia-smi samples every 200 ms: a very short timed region may get none
    assert c is None or ("sm_mhz" in c and "reasons" in c and "sm_max_mhz" in c)
