"""GPU check of the head-sharded multi-GPU layout on one GPU: each rank's
shard (a block of KV heads and their query heads, as bench.py --shard heads
gives it) runs through the C ABI one after another, and the shards' O and
LSE, put back together along the heads, must match the oracle on the whole
problem -- bitwise equal to one whole-problem launch, since attention of one
(b, h) involves no other head."""
import numpy as np
import pytest
import torch

import exact_io_aware_78_b200 as ea
from exact_io_aware_78_b200.inputs import WORKLOADS, head_shard, sample_rows, shard_inputs, workload_inputs
from oracle import attention_ref

from gpu_helpers import assert_close, oracle_view, ranges_view, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(lib_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.set_device(0)
    ea.load_library(lib_path)
    yield


@pytest.mark.parametrize("name,world", [("bf16_gqa_causal_b2h32kv8_n4096_d128_q3", 2),
                                        ("bf16_gqa_causal_b2h32kv8_n4096_d128_q3", 8),
                                        ("fp8_causal_b2h16_n8192_d128", 4),
                                        ("bf16_doccausal_b2h16_n16384_d128", 2)])
def test_head_shards_concatenate_to_the_whole_problem(name, world):
    w = WORKLOADS[name]
    inp = workload_inputs(w)
    whole_o, whole_l = run_gpu(inp, w.causal, w.window, w.scale)
    parts = []
    for rank in range(world):
        _, q_lo, q_hi, kv_lo, kv_hi = head_shard(w, world, rank)
        parts.append(run_gpu(shard_inputs(inp, q_lo, q_hi, kv_lo, kv_hi), w.causal, w.window, w.scale))
    o = np.concatenate([p[0] for p in parts], axis=2)
    lse = np.concatenate([p[1] for p in parts], axis=1)
    # a shard's heads are computed exactly as in the whole launch
    assert np.array_equal(o, whole_o) and np.array_equal(lse, whole_l)
    rows = sample_rows(w.N, w.window, 24, seed=w.seed + 7)
    q, k, v = oracle_view(inp, w.dtype)
    lo, hi = ranges_view(inp)
    Oref, Lref = attention_ref(q, k, v, w.causal, w.window, w.scale, rows=rows, key_lo=lo, key_hi=hi)
    assert_close(o[:, rows], lse[:, :, rows], Oref, Lref, w.dtype, f"{name} as {world} head shards")
