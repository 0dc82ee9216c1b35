"""Host-side checks of the seeded input recipe and the FLOP/byte accounting."""
import numpy as np
import pytest
import torch

from exact_io_aware_78_b200 import accounting
from exact_io_aware_78_b200.inputs import (E4M3_MAX, WORKLOADS, make_inputs,
                                           quantize_e4m3_per_head, sample_rows)


def test_generation_is_deterministic_and_seeded():
    a = make_inputs(1, 2, 1, 33, 8, "bf16", 99)
    b = make_inputs(1, 2, 1, 33, 8, "bf16", 99)
    c = make_inputs(1, 2, 1, 33, 8, "bf16", 100)
    for n in "qkv":
        assert torch.equal(a[n], b[n])
    assert not torch.equal(a["q"], c["q"])
    assert a["q"].dtype == torch.bfloat16 and a["q"].shape == (1, 33, 2, 8)
    assert a["k"].shape == (1, 33, 1, 8)


def test_q_multiplier_applies_before_cast():
    a = make_inputs(1, 1, 1, 16, 8, "fp32", 5, q_mult=3.0)
    b = make_inputs(1, 1, 1, 16, 8, "fp32", 5)
    assert torch.equal(a["q"], b["q"] * 3.0)
    assert torch.equal(a["k"], b["k"])


def test_fp8_per_head_scale_definition():
    x = torch.randn(2, 64, 3, 16, generator=torch.Generator().manual_seed(1))
    codes, s = quantize_e4m3_per_head(x)
    amax = x.abs().amax(dim=(0, 1, 3))
    torch.testing.assert_close(s, amax / E4M3_MAX)
    deq = codes.to(torch.float32) * s.view(1, 1, -1, 1)
    # the largest element of each head maps to +-448 exactly
    assert torch.all(codes.to(torch.float32).abs().amax(dim=(0, 1, 3)) == E4M3_MAX)
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 for normal codes
    big = x.abs() > 2 ** -6 * s.view(1, 1, -1, 1) * 4
    rel = ((deq - x).abs() / x.abs())[big]
    assert rel.max() <= 2 ** -4 + 1e-6


def test_workload_table():
    assert len(WORKLOADS) == 6
    assert WORKLOADS["bf16_doccausal_b2h16_n16384_d128"].mask == "documents"
    w = WORKLOADS["bf16_gqa_causal_b2h32kv8_n4096_d128_q3"]
    assert (w.B, w.Hq, w.Hkv, w.N, w.d, w.causal, w.q_mult) == (2, 32, 8, 4096, 128, True, 3.0)
    assert w.group == 4


@pytest.mark.parametrize("N", list(range(1, 30)) + [128, 257])
def test_attended_pairs_brute_force(N):
    for causal in (False, True):
        for window in (0, 1, 2, 5, 17, 64):
            i = np.arange(N)[:, None]
            j = np.arange(N)[None, :]
            ok = np.ones((N, N), bool)
            if causal:
                ok &= j <= i
            if window > 0:
                ok &= j > i - window
            assert accounting.attended_pairs(N, causal, window) == int(ok.sum())


@pytest.mark.parametrize("kind", ["documents", "prefix", "random"])
def test_range_pairs_brute_force(kind):
    from exact_io_aware_78_b200.inputs import make_row_ranges
    N = 50
    lo, hi = make_row_ranges(kind, 3, N, 4, 3, 17)
    lo, hi = lo.numpy(), hi.numpy()
    for causal in (False, True):
        for window in (0, 1, 6):
            i = np.arange(N)[None, :, None]
            j = np.arange(N)[None, None, :]
            ok = (j >= lo[:, :, None]) & (j < hi[:, :, None])
            if causal:
                ok &= j <= i
            if window > 0:
                ok &= j > i - window
            assert accounting.range_pairs(lo, hi, causal, window) == int(ok.sum())
    # ranges that cover every key reduce to the mask-free count
    full_lo, full_hi = np.zeros((2, N), np.int64), np.full((2, N), N)
    assert accounting.range_pairs(full_lo, full_hi, True, 7) == 2 * accounting.attended_pairs(N, True, 7)


def test_flop_counts_of_the_workloads():
    w = WORKLOADS["bf16_causal_b4h16_n2048_d128"]
    # 4*B*H*N^2*d / 2 for causal, and the exact pair count is N(N+1)/2
    assert accounting.flops_half_square(w) == 4 * 4 * 16 * 2048 ** 2 * 128 / 2
    assert accounting.flops(w) == 4 * 4 * 16 * 128 * (2048 * 2049 // 2)
    w4 = WORKLOADS["bf16_causal_window4096_b1h16_n16384_d128"]
    assert abs(accounting.flops(w4) / 1e9 - 481.05) < 0.01
    assert abs(accounting.flops_half_square(w4) / 1e9 - 1099.51) < 0.01


def test_sample_rows_cover_edges():
    r = sample_rows(4096, 0, 64, 3)
    assert r[0] == 0 and r[-1] == 4095 and 128 in r and 127 in r
    assert r == sorted(set(r))
    rw = sample_rows(16384, 4096, 16, 3)
    assert 4095 in rw and 4096 in rw


# ---- decode steps

from exact_io_aware_78_b200.accounting import decode_bytes, decode_flops, decode_pairs  # noqa: E402
from exact_io_aware_78_b200.inputs import DECODE_WORKLOADS, make_decode_inputs  # noqa: E402


@pytest.mark.parametrize("Nq,Nk,causal,window", [(1, 1, True, 0), (1, 100, True, 0), (3, 100, True, 0),
                                                  (3, 100, False, 0), (4, 50, True, 7), (2, 9, False, 3),
                                                  (5, 5, True, 0)])
def test_decode_pairs_by_brute_force(Nq, Nk, causal, window):
    n = 0
    for i in range(Nq):
        pos = Nk - Nq + i
        for j in range(Nk):
            if (not causal or j <= pos) and (window <= 0 or j > pos - window):
                n += 1
    assert decode_pairs(Nq, Nk, causal, window) == n


def test_decode_workload_accounting():
    w = DECODE_WORKLOADS["decode_b8h32kv8_nq1_nk16384_d128"]
    assert decode_flops(w) == 4 * 128 * 8 * 32 * 16384
    # K and V of every cached row read once dominate the bytes
    assert decode_bytes(w) == 2 * 8 * 1 * 32 * 128 * 2 + 2 * 8 * 16384 * 8 * 128 * 2 + 8 * 32 * 4
    ww = DECODE_WORKLOADS["decode_b4h32kv8_nq2_nk8192_d128_window2048"]
    # only the last window + Nq - 1 keys can be seen
    assert decode_bytes(ww) == 2 * 4 * 2 * 32 * 128 * 2 + 2 * 4 * (2048 + 1) * 8 * 128 * 2 + 4 * 32 * 2 * 4


def test_decode_inputs_are_seeded_bf16():
    a = make_decode_inputs(2, 4, 2, 1, 33, 64, seed=3)
    b = make_decode_inputs(2, 4, 2, 1, 33, 64, seed=3)
    assert all(torch.equal(a[n], b[n]) for n in "qkv")
    assert a["q"].shape == (2, 1, 4, 64) and a["k"].shape == (2, 33, 2, 64) and a["q"].dtype == torch.bfloat16


def test_head_shards_keep_the_row_ranges_whole():
    """Row ranges are shared by all heads: every shard carries them unchanged."""
    import torch
    from exact_io_aware_78_b200.inputs import WORKLOADS, head_shard, shard_inputs, workload_inputs
    w = WORKLOADS["bf16_doccausal_b2h16_n16384_d128"]
    inp = workload_inputs(w)
    sw, q_lo, q_hi, kv_lo, kv_hi = head_shard(w, 4, 1)
    sub = shard_inputs(inp, q_lo, q_hi, kv_lo, kv_hi)
    assert sub["q"].shape[2] == sw.Hq == 4 and sub["k"].shape[2] == sw.Hkv == 4
    assert torch.equal(sub["key_lo"], inp["key_lo"]) and torch.equal(sub["key_hi"], inp["key_hi"])
    assert sw.mask == w.mask and sw.mask_min == w.mask_min
