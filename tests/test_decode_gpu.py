"""Parity of the decode / split-KV forward (attn_fwd_decode, through the C
ABI: the tensor-core kernel for num_splits = 0, the CUDA-core kernel for an
explicit split count) with the float64 oracle attention_kv_ref, on seeded
bf16 inputs:
small shapes covering GQA groups, d = 64 and 128, causal and windowed masks,
ragged key counts, a single key, Nq > 1 (new tokens causal among
themselves) and explicit split counts from one to more ranges than key
batches; the two named decode workloads at full size (every query row:
Nq is small); results across split counts and across repeated runs."""
import numpy as np
import pytest
import torch

import exact_io_aware_78_b200 as ea
from exact_io_aware_78_b200 import _binding as Bn
from exact_io_aware_78_b200.inputs import DECODE_WORKLOADS, decode_workload_inputs, make_decode_inputs
from oracle import attention_kv_ref

from gpu_helpers import TOL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib(lib_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability(0)[0] != 10:
        pytest.skip("needs an sm_100 GPU")
    torch.cuda.set_device(0)
    return ea.load_library(lib_path)


def run(inp, causal, window, splits=0):
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    o, lse = ea.forward_decode(q, k, v, causal=causal, window=window, num_splits=splits)
    torch.cuda.synchronize()
    return o, lse


def check(inp, o, lse, causal, window, what):
    q, k, v = (inp[n].to(torch.float64).numpy() for n in "qkv")
    ref_o, ref_l = attention_kv_ref(q, k, v, causal, window)
    d_o = np.abs(o.double().cpu().numpy() - ref_o)
    d_l = np.abs(lse.double().cpu().numpy() - ref_l)
    tmax, tmean, tlse = TOL["bf16"]
    msg = f"{what}: max {d_o.max():.3e} (<= {tmax}), mean {d_o.mean():.3e} (<= {tmean}), lse {d_l.max():.3e}"
    print(msg)
    assert np.isfinite(o.float().cpu().numpy()).all() and np.isfinite(lse.cpu().numpy()).all(), msg
    assert d_o.max() <= tmax and d_o.mean() <= tmean and d_l.max() <= tlse, msg


CASES = [
    # B, Hq, Hkv, Nq, Nk, d, causal, window, splits
    (1, 1, 1, 1, 1, 128, True, 0, 0),        # a single key
    (1, 4, 1, 1, 31, 128, True, 0, 0),       # less than one key batch
    (2, 8, 2, 1, 300, 128, True, 0, 0),      # GQA 4:1, ragged
    (2, 8, 2, 1, 300, 128, True, 0, 1),      # one key range
    (2, 8, 2, 1, 300, 128, True, 0, 3),
    (2, 8, 2, 1, 300, 128, True, 0, 1000),   # more ranges than batches (clamped)
    (1, 8, 1, 1, 1000, 128, False, 0, 0),    # 8 query rows per KV head
    (1, 8, 2, 2, 1000, 128, True, 0, 0),     # two new tokens, causal among themselves
    (1, 4, 2, 4, 513, 64, True, 0, 0),       # d = 64, four new tokens
    (3, 4, 4, 1, 4097, 64, False, 0, 5),     # MHA, d = 64
    (1, 8, 8, 1, 129, 128, True, 50, 0),     # window
    (1, 4, 1, 2, 700, 128, True, 1, 0),      # window 1: each query sees only itself
    (1, 4, 2, 4, 4, 128, True, 0, 0),        # Nq == Nk: self-attention of a short sequence
    (1, 2, 2, 3, 3, 128, False, 0, 2),
    # tensor-core kernel only (more than 8 rows per kv head), ragged stream-K ranges
    (2, 16, 1, 2, 1500, 128, True, 0, 0),    # 32 rows per kv head
    (3, 12, 2, 3, 777, 64, True, 0, 0),      # 18 rows, d = 64
    (1, 8, 1, 4, 300, 128, True, 100, 0),    # 32 rows, window
    (4, 32, 8, 1, 16500, 128, False, 0, 0),  # many pairs, ragged last tile
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}h{}kv{}nq{}nk{}d{}c{}w{}s{}".format(*c))
def test_small_shapes(lib, case):
    B, Hq, Hkv, Nq, Nk, d, causal, window, splits = case
    inp = make_decode_inputs(B, Hq, Hkv, Nq, Nk, d, seed=Nk + 7 * Nq + Hq)
    o, lse = run(inp, causal, window, splits)
    check(inp, o, lse, causal, window, str(case))


@pytest.mark.parametrize("name", sorted(DECODE_WORKLOADS))
def test_workloads_full_size(lib, name):
    w = DECODE_WORKLOADS[name]
    inp = decode_workload_inputs(w)
    o, lse = run(inp, w.causal, w.window)
    check(inp, o, lse, w.causal, w.window, name)


def test_tensor_core_and_cuda_core_kernels_agree(lib):
    """The two key-range kernels compute the same rows (within rounding)."""
    inp = make_decode_inputs(2, 8, 2, 2, 3000, 128, seed=41)
    a_o, a_l = run(inp, True, 0, 0)
    b_o, b_l = run(inp, True, 0, 5)
    check(inp, a_o, a_l, True, 0, "tensor-core kernel")
    assert (a_o.float() - b_o.float()).abs().max().item() <= 1.6e-2
    assert (a_l - b_l).abs().max().item() <= 1e-4


def test_split_counts_agree_and_runs_repeat(lib):
    inp = make_decode_inputs(2, 8, 2, 1, 5000, 128, seed=31)
    results = {s: run(inp, True, 0, s) for s in (1, 2, 7, 40, 0)}
    base_o, base_l = results[1]
    for s, (o, lse) in results.items():
        check(inp, o, lse, True, 0, f"splits={s}")
        assert (o.float() - base_o.float()).abs().max().item() <= 1.6e-2
        assert (lse - base_l).abs().max().item() <= 1e-4
    # a given split count is deterministic
    for s in (7, 0):
        o, lse = run(inp, True, 0, s)
        assert torch.equal(o, results[s][0]) and torch.equal(lse, results[s][1])


def test_decode_matches_the_prefill_kernel_on_the_last_row(lib):
    """The decode step's result for the last token equals the last row of the
    tcgen05 prefill kernel run over the whole sequence (two independent GPU
    paths for the same rows)."""
    B, H, N, d = 2, 8, 1000, 128
    full = make_decode_inputs(B, H, H, N, N, d, seed=5)
    dev = torch.device("cuda:0")
    q, k, v = (full[n].to(dev) for n in "qkv")
    o_full, l_full = ea.forward(q, k, v, causal=True)
    o_dec, l_dec = ea.forward_decode(q[:, N - 1:].contiguous(), k, v, causal=True)
    torch.cuda.synchronize()
    assert (o_dec.float() - o_full[:, N - 1:].float()).abs().max().item() <= 1.6e-2
    assert (l_dec - l_full[:, :, N - 1:]).abs().max().item() <= 1e-4


def test_bad_arguments_return_codes(lib):
    dev = torch.device("cuda:0")
    q = torch.zeros(1, 2, 8, 128, device=dev, dtype=torch.bfloat16)
    k = torch.zeros(1, 1, 2, 128, device=dev, dtype=torch.bfloat16)  # Nk = 1 < Nq = 2
    o = torch.empty_like(q)
    lse = torch.empty(1, 8, 2, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    assert lib.attn_fwd_decode(q.data_ptr(), k.data_ptr(), k.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 8, 2, 2,
                               1, 128, 1, 0, 0.1, Bn.EA_BF16, 0, s) == Bn.EA_EINVAL
    # a host pointer is rejected before any launch
    h = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16)
    assert lib.attn_fwd_decode(q.data_ptr(), h.data_ptr(), h.data_ptr(), o.data_ptr(), lse.data_ptr(), 1, 8, 2, 2,
                               4, 128, 1, 0, 0.1, Bn.EA_BF16, 0, s) == Bn.EA_EINVAL
