"""The JSON line of bench.py's CUDA arm, one short run per kind of step
(prefill, decode, backward): exactly one line on stdout with every key of
the contract, a positive whole-job value, a roofline whose fraction is
achieved / peak and whose traffic is the recorded ncu figure for the current
kernel sources (or null), the launch count per step, the end-to-end figure
with its copied bytes, and the clocks sampled during the timed region."""
import json
import os
import subprocess
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu

KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks")
STEPS = 3

CASES = [
    # workload, kind, roofline bound, kernel launches per step
    ("bf16_causal_b4h16_n2048_d128", "prefill", "tensor", 1),
    ("decode_b8h32kv8_nq1_nk16384_d128", "decode", "hbm", 2),
    ("bwd_bf16_causal_b4h16_n2048_d128", "backward", "tensor", 3),
]


@pytest.fixture(scope="module", autouse=True)
def _gpu(lib_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[1])
def test_bench_line(case):
    name, kind, bound, launches = case
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", name, "--steps", str(STEPS),
           "--warmup", "3", "--no-cpu-baseline"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=280, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [l for l in proc.stdout.splitlines() if l.lstrip().startswith("{")]
    assert len(lines) == 1, proc.stdout
    j = json.loads(lines[0])
    for key in KEYS:
        assert key in j, key
    assert j["n_gpus"] == 1 and j["steps"] == STEPS and j["warmup"] == 3
    assert j["value"] > 0 and j["ms_per_step"] > 0 and j["higher_is_better"] is True
    assert j["scaling"] == "weak" and j["data"] == "synthetic"
    assert j["config"]["workload"] == name

    r = j["roofline"]
    assert r["bound"] == bound and r["unit"] == ("GB/s" if bound == "hbm" else "TFLOP/s")
    assert r["peak"] > 0 and r["achieved"] > 0
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-9)
    assert 0.0 < r["frac"] < 1.5
    assert r["kernel_source_hash"] == bench.kernel_source_hash(kind)
    assert r["traffic"] == bench.load_traffic(name)
    assert r["traffic"] is None or r["traffic"] > 0

    assert j["gpu_launches"] == STEPS * launches
    e = j["e2e"]
    assert e["value"] > 0 and e["unit"] == j["unit"]
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    # a few samples at most in so short a run; the key is always present
    assert j["clocks"] is None or j["clocks"]["sm_mhz"] > 0


def test_default_line_carries_the_curve():
    """The default run times the largest forward configuration and adds
    per_config: all five forward configurations, shortest sequence first,
    each with its own value, roofline and probed SM clock."""
    from exact_io_aware_78_b200.inputs import CURVE_WORKLOADS, DEFAULT_BENCH_WORKLOAD
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--steps", str(STEPS), "--warmup", "3",
           "--no-cpu-baseline"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=280, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [l for l in proc.stdout.splitlines() if l.lstrip().startswith("{")]
    assert len(lines) == 1, proc.stdout
    j = json.loads(lines[0])
    assert j["config"]["workload"] == DEFAULT_BENCH_WORKLOAD
    curve = j["per_config"]
    assert [c["workload"] for c in curve] == list(CURVE_WORKLOADS)
    for c in curve:
        r = c["roofline"]
        assert c["value"] > 0 and c["ms_per_step"] > 0 and r["achieved"] > 0
        assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], rel=1e-9)
        assert c["clocks"]["sm_mhz_probe_median"] > 100
    top = curve[list(CURVE_WORKLOADS).index(DEFAULT_BENCH_WORKLOAD)]
    assert top["value"] == j["value"] and top["roofline"] == j["roofline"]
