"""Host-side logic of bench.py without a GPU: the reference arm's JSON line,
the whole-job throughput formula, and the multi-rank reduction and barrier
run as two gloo ranks on the CPU."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_job_tflops_is_weak_scaling_over_the_slowest_rank():
    # 2 ranks x 10 steps x 1e12 FLOP in 4 ms (slowest rank) = 5000 TFLOP/s
    assert bench.job_tflops(1e12, 10, 2, 4.0) == pytest.approx(5000.0)
    assert bench.job_tflops(1e12, 10, 1, 4.0) == pytest.approx(2500.0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        m = bench.dist_max(10.0 + 5.0 * rank, world, torch.device("cpu"))
        out[rank] = m
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_reference_arm_prints_one_contract_line():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "fp32_n128_d64",
           "--steps", "3", "--warmup", "3", "--ref-seconds", "1.5"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr
    lines = [l for l in proc.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in j, key
    assert j["impl"] == "reference" and j["unit"] == "TFLOP/s" and j["value"] > 0
    assert j["config"]["workload"] == "fp32_n128_d64"
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference", "--workload",
           "fp32_n128_d64", "--steps", "3", "--warmup", "3", "--ref-seconds", "1.5"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert proc.returncode == 0 and proc.stdout.strip() == ""


# ---- head-sharded multi-GPU layout (each rank owns a block of KV heads and
# their query heads; no data moves between ranks)

from exact_io_aware_78_b200 import accounting  # noqa: E402
from exact_io_aware_78_b200.inputs import WORKLOADS, head_shard, make_inputs, shard_inputs  # noqa: E402
from dataclasses import replace as dataclasses_replace  # noqa: E402


@pytest.mark.parametrize("name", ["bf16_causal_b4h16_n2048_d128", "bf16_gqa_causal_b2h32kv8_n4096_d128_q3",
                                  "fp8_causal_b2h16_n8192_d128"])
@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_head_shards_partition_the_heads(name, world):
    w = WORKLOADS[name]
    q_seen, kv_seen, flops = [], [], 0.0
    for rank in range(world):
        sub, q_lo, q_hi, kv_lo, kv_hi = head_shard(w, world, rank)
        q_seen += list(range(q_lo, q_hi))
        kv_seen += list(range(kv_lo, kv_hi))
        # every query head of the shard reads a KV head of the same shard
        assert all(kv_lo <= h // w.group < kv_hi for h in range(q_lo, q_hi))
        assert sub.group == w.group and sub.Hq == q_hi - q_lo and sub.Hkv == kv_hi - kv_lo
        flops += accounting.flops(sub)
    assert q_seen == list(range(w.Hq)) and kv_seen == list(range(w.Hkv))
    assert flops == pytest.approx(accounting.flops(w))


def test_head_shard_rejects_uneven_splits():
    with pytest.raises(ValueError):
        head_shard(WORKLOADS["bf16_gqa_causal_b2h32kv8_n4096_d128_q3"], 3, 0)
    with pytest.raises(ValueError):
        head_shard(WORKLOADS["bf16_causal_b4h16_n2048_d128"], 2, 2)


def test_sharded_results_are_the_full_results():
    """Attention per (b, h) involves no other head, so the oracle run on each
    shard's slices and concatenated along the heads equals the oracle on the
    whole problem (GQA, e4m3 scales included)."""
    import oracle
    w = dataclasses_replace(WORKLOADS["fp8_causal_b2h16_n8192_d128"], B=1, Hq=4, Hkv=2, N=40, d=128)
    inp = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, 77)

    def run(x):
        q, k, v = (oracle.dequantize_per_head(x[n].view(torch.uint8).numpy(), x[n + "_scale"].numpy())
                   for n in "qkv")
        return oracle.attention_ref(q, k, v, w.causal, w.window, w.scale)

    full_o, full_l = run(inp)
    parts = []
    for rank in range(2):
        _, q_lo, q_hi, kv_lo, kv_hi = head_shard(w, 2, rank)
        parts.append(run(shard_inputs(inp, q_lo, q_hi, kv_lo, kv_hi)))
    o = np.concatenate([p[0] for p in parts], axis=2)
    l = np.concatenate([p[1] for p in parts], axis=1)
    assert np.array_equal(o, full_o) and np.array_equal(l, full_l)


def test_sharded_tflops_is_strong_scaling_over_the_slowest_rank():
    # the whole problem (1e12 FLOP per step) x 10 steps in 4 ms (slowest rank)
    assert bench.sharded_tflops(1e12, 10, 4.0) == pytest.approx(2500.0)


def _shard_rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WORKLOADS["bf16_gqa_causal_b2h32kv8_n4096_d128_q3"]
        sub, q_lo, q_hi, kv_lo, kv_hi = head_shard(w, world, rank)
        f = torch.tensor([accounting.flops(sub)], dtype=torch.float64)
        dist.all_reduce(f)
        slowest = bench.dist_max(2.0 + rank, world, torch.device("cpu"))
        out[rank] = (q_lo, q_hi, float(f.item()), bench.sharded_tflops(accounting.flops(w), 10, slowest))
    finally:
        dist.destroy_process_group()


def test_head_shards_over_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_shard_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    w = WORKLOADS["bf16_gqa_causal_b2h32kv8_n4096_d128_q3"]
    total = accounting.flops(w)
    assert out[0][:2] == (0, 16) and out[1][:2] == (16, 32)
    for rank in range(world):
        assert out[rank][2] == pytest.approx(total)
        assert out[rank][3] == pytest.approx(total * 10 / 3e-3 / 1e12)  # slowest rank: 3 ms


def test_reference_arm_on_a_decode_workload():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "decode_b4h32kv8_nq2_nk8192_d128_window2048", "--steps", "3", "--warmup", "3", "--ref-seconds", "1.5"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr
    lines = [l for l in proc.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["config"]["Nq"] == 2 and j["config"]["Nk"] == 8192
    assert j["value"] > 0 and j["cpu_baseline"]["kind"] == "oracle"


def test_reference_arm_on_the_document_mask_workload():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "bf16_doccausal_b2h16_n16384_d128", "--steps", "3", "--warmup", "3", "--ref-seconds", "3"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr
    lines = [l for l in proc.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["config"]["row_ranges"].startswith("documents")
    assert j["value"] > 0


def test_pairs_for_rows_with_ranges_brute_force():
    from exact_io_aware_78_b200.inputs import make_row_ranges
    N = 60
    lo, hi = make_row_ranges("random", 1, N, 8)
    lo, hi = lo[0].numpy(), hi[0].numpy()
    rows = [0, 3, 17, 59, 30]
    for causal in (False, True):
        for window in (0, 5):
            want = 0
            for i in rows:
                for j in range(N):
                    if lo[i] <= j < hi[i] and (not causal or j <= i) and (window <= 0 or j > i - window):
                        want += 1
            assert bench.pairs_for_rows(rows, N, causal, window, lo, hi) == want


def test_reference_arm_on_a_backward_workload():
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
           "bwd_bf16_causal_b4h16_n2048_d128", "--steps", "3", "--warmup", "3", "--ref-seconds", "3"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr
    lines = [l for l in proc.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["metric"].startswith("attention bwd") and j["value"] > 0


def test_backward_accounting():
    from exact_io_aware_78_b200.inputs import BWD_WORKLOADS
    w = BWD_WORKLOADS["bwd_bf16_causal_b4h16_n2048_d128"]
    assert accounting.bwd_flops(w) == pytest.approx(10 * 4 * 16 * 128 * (2048 * 2049 // 2))
    # Q, K, V, O, dO read; dQ, dK, dV written (bf16); LSE read (fp32)
    assert accounting.bwd_bytes(w) == 8 * (4 * 2048 * 16 * 128 * 2) + 4 * 16 * 2048 * 4


# ---- --gpus N: the launcher and the shared config object

def test_resolve_launch():
    assert bench.resolve_launch(1, {}) == "run"
    assert bench.resolve_launch(4, {}) == "spawn"
    assert bench.resolve_launch(2, {"WORLD_SIZE": "2"}) == "run"
    assert bench.resolve_launch(1, {"WORLD_SIZE": "1"}) == "run"
    with pytest.raises(ValueError):
        bench.resolve_launch(8, {"WORLD_SIZE": "1"})  # torchrun job of another size
    with pytest.raises(ValueError):
        bench.resolve_launch(1, {"WORLD_SIZE": "2"})
    with pytest.raises(ValueError):
        bench.resolve_launch(0, {})


def test_gpus_mismatch_with_torchrun_is_an_error():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference", "--workload",
           "fp32_n128_d64", "--steps", "3", "--warmup", "3", "--ref-seconds", "1.5"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert proc.returncode != 0 and "WORLD_SIZE" in proc.stderr


def test_gpus_two_spawns_two_ranks_and_prints_one_line():
    """--gpus 2 without a torchrun environment relaunches the command as a
    two-rank torchrun job: rank 0 prints the one JSON line with n_gpus 2,
    rank 1 reports that it exits without work."""
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                                                          "MASTER_PORT")}
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "2", "--impl", "reference", "--workload",
           "fp32_n128_d64", "--steps", "3", "--warmup", "3", "--ref-seconds", "1.5"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert proc.returncode == 0, proc.stderr[-2000:]
    lines = [l for l in proc.stdout.splitlines() if l.lstrip().startswith("{")]
    assert len(lines) == 1, proc.stdout
    j = json.loads(lines[0])
    assert j["n_gpus"] == 2 and j["impl"] == "reference"
    assert "rank 1 of 2 exits without work" in proc.stderr


@pytest.mark.parametrize("name", ["bf16_causal_window4096_b1h16_n16384_d128", "decode_b4h32kv8_nq2_nk8192_d128_window2048",
                                  "bwd_bf16_causal_b4h16_n2048_d128"])
def test_reference_arm_config_is_the_cuda_arms(name):
    """Both arms print the same `config` object for a workload."""
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", name,
           "--steps", "3", "--warmup", "3", "--ref-seconds", "1.5"]
    proc = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert proc.returncode == 0, proc.stderr[-2000:]
    j = json.loads([l for l in proc.stdout.splitlines() if l.lstrip().startswith("{")][0])
    from exact_io_aware_78_b200.inputs import BWD_WORKLOADS, DECODE_WORKLOADS
    w = {**WORKLOADS, **DECODE_WORKLOADS, **BWD_WORKLOADS}[name]
    assert j["config"] == json.loads(json.dumps(bench.any_line_config(w, 1, "replicas")))


def test_default_workload_is_the_largest_forward_configuration():
    from exact_io_aware_78_b200.inputs import CURVE_WORKLOADS, DEFAULT_BENCH_WORKLOAD
    assert DEFAULT_BENCH_WORKLOAD in CURVE_WORKLOADS and len(CURVE_WORKLOADS) == 5
    ws = [WORKLOADS[n] for n in CURVE_WORKLOADS]
    assert [w.N for w in ws] == [128, 2048, 4096, 16384, 8192]
    # the longest sequence (the curve's axis); C3, C4 and C5 hold equally many Q elements
    assert max(ws, key=lambda w: w.N).name == DEFAULT_BENCH_WORKLOAD
