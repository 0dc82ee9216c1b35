"""Parity of the attention backward (attn_bwd, through the C ABI) with the
float64 oracle attention_bwd_ref on seeded bf16 inputs: every element of
dQ, dK, dV for small shapes (GQA groups, d = 64 and 128, causal and windowed
masks, ragged N), both with the oracle's own O and LSE fed to the kernels
(the backward alone) and end to end after the tcgen05 forward; sampled
checks at a benchmark size; determinism; the invariants of the softmax
Jacobian (dK sums to zero over the keys of a head).  With per-row key ranges
(attn_bwd_masked): documents, prefix-LM and random ranges (empty rows, key
tiles no row sees), and bit-identity with the causal backward when the
ranges reproduce the causal mask."""
import numpy as np
import pytest
import torch

import exact_io_aware_78_b200 as ea
from exact_io_aware_78_b200.inputs import make_grad_output, make_inputs, make_row_ranges
from oracle import attention_bwd_ref, attention_ref

pytestmark = pytest.mark.gpu

# Bars, relative to the size of each reference gradient: max |err| <= 1.2e-2
# * max |ref| and mean |err| <= 6e-3 * mean |ref|, about twice the largest
# errors measured on a B200 over every case in this file (relative max
# 6.0e-3, relative mean 3.1e-3).  The kernels round P and dS to bf16
# (relative step 2^-9) before the products that consume them and store bf16
# gradients, accumulating in fp32, so each gradient element carries errors
# of a few 2^-9 of the typical element size; a dropped term or a wrong
# scale moves the mean by far more.
TOL_MAX, TOL_MEAN = 1.2e-2, 6e-3


@pytest.fixture(scope="module", autouse=True)
def _gpu(lib_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability(0)[0] != 10:
        pytest.skip("needs an sm_100 GPU")
    torch.cuda.set_device(0)
    ea.load_library(lib_path)


def inputs(B, Hq, Hkv, N, d, seed):
    inp = make_inputs(B, Hq, Hkv, N, d, "bf16", seed)
    inp["do"] = make_grad_output(B, N, Hq, d, seed + 3)
    return inp


def compare(got, ref, what):
    out = []
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        g = g.double().cpu().numpy()
        assert np.isfinite(g).all(), f"{what}: non-finite {name}"
        err = np.abs(g - r)
        mx, mean = err.max() / np.abs(r).max(), err.mean() / np.abs(r).mean()
        out.append(f"{name} max {mx:.2e} mean {mean:.2e}")
        assert mx <= TOL_MAX and mean <= TOL_MEAN, f"{what}: {name} relative max {mx:.3e}, mean {mean:.3e}"
    print(what, "; ".join(out))


def run_case(B, Hq, Hkv, N, d, causal, window, seed, end_to_end):
    inp = inputs(B, Hq, Hkv, N, d, seed)
    dev = torch.device("cuda:0")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    scale = d ** -0.5
    q64, k64, v64, do64 = (inp[n].double().numpy() for n in ("q", "k", "v", "do"))
    o_ref, l_ref = attention_ref(q64, k64, v64, causal, window, scale)
    if end_to_end:
        o, lse = ea.forward(q, k, v, causal=causal, window=window, scale=scale)
    else:
        o = torch.from_numpy(o_ref).to(torch.bfloat16).to(dev)
        lse = torch.from_numpy(l_ref).float().to(dev)
    grads = ea.backward(q, k, v, o, lse, do, causal=causal, window=window, scale=scale)
    st, code, site = ea.attn_get_last_error()
    assert st == 0, f"device error code {code} at wait site {site}"
    ref = attention_bwd_ref(q64, k64, v64, do64, causal, window, scale, o=o_ref, lse=l_ref)
    compare(grads, ref, f"B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} c{int(causal)} w{window} e2e{int(end_to_end)}")
    return grads


CASES = [
    # B, Hq, Hkv, N, d, causal, window
    (1, 1, 1, 128, 128, False, 0),
    (1, 2, 2, 128, 128, True, 0),
    (1, 2, 1, 300, 128, True, 0),        # ragged, GQA 2:1
    (2, 4, 1, 257, 64, True, 0),         # GQA 4:1, d = 64
    (1, 2, 2, 520, 128, False, 0),
    (1, 2, 2, 700, 128, True, 100),      # window
    (1, 4, 2, 384, 64, False, 50),       # window without causal
    (1, 1, 1, 17, 128, True, 0),         # one partial tile
    (2, 8, 8, 1024, 128, True, 0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}h{}kv{}n{}d{}c{}w{}".format(*c))
def test_backward_alone(case):
    run_case(*case, seed=5000 + case[3] + case[4], end_to_end=False)


@pytest.mark.parametrize("case", CASES[1::3], ids=lambda c: "B{}h{}kv{}n{}d{}c{}w{}".format(*c))
def test_forward_then_backward(case):
    run_case(*case, seed=6000 + case[3], end_to_end=True)


def test_benchmark_shape_sampled():
    """B4 H16 N2048 d128 causal (the backward benchmark's shape): full GPU run,
    the oracle on four (b, h) heads, every element of those heads' dQ and of
    dK, dV."""
    B, H, N, d = 4, 16, 2048, 128
    inp = inputs(B, H, H, N, d, 2048)
    dev = torch.device("cuda:0")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = ea.forward(q, k, v, causal=True)
    dq, dk, dv = ea.backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (1, 7), (2, 15), (3, 3)):
        sl = (slice(b, b + 1), slice(None), slice(h, h + 1))
        ref = attention_bwd_ref(*(inp[n][sl].double().numpy() for n in ("q", "k", "v", "do")), True, 0,
                                d ** -0.5)
        compare((dq[sl], dk[sl], dv[sl]), ref, f"b{b} h{h}")


def test_deterministic_and_dk_sums_to_zero():
    B, Hq, Hkv, N, d = 2, 4, 2, 600, 128
    inp = inputs(B, Hq, Hkv, N, d, 77)
    dev = torch.device("cuda:0")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = ea.forward(q, k, v, causal=True)
    a = ea.backward(q, k, v, o, lse, do, causal=True)
    b = ea.backward(q, k, v, o, lse, do, causal=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    dk = a[1].double()
    # rows of dS sum to zero: sum over keys of dK is ~0 relative to its terms
    assert (dk.sum(dim=1).abs().max() / dk.abs().sum(dim=1).max()).item() < 2e-2


# ------------------------------------------------------------- row ranges
def run_ranges(kind, B, Hq, Hkv, N, d, causal, window, mn, mx, seed, end_to_end=False, lo=None, hi=None):
    inp = inputs(B, Hq, Hkv, N, d, seed)
    if lo is None:
        lo, hi = make_row_ranges(kind, B, N, seed + 5, mn, mx)
    lo = torch.as_tensor(lo, dtype=torch.int32)
    hi = torch.as_tensor(hi, dtype=torch.int32)
    dev = torch.device("cuda:0")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    klo, khi = lo.to(dev), hi.to(dev)
    scale = d ** -0.5
    q64, k64, v64, do64 = (inp[n].double().numpy() for n in ("q", "k", "v", "do"))
    o_ref, l_ref = attention_ref(q64, k64, v64, causal, window, scale, key_lo=lo.numpy(), key_hi=hi.numpy())
    if end_to_end:
        o, lse = ea.forward(q, k, v, causal=causal, window=window, scale=scale, key_lo=klo, key_hi=khi)
    else:
        o = torch.from_numpy(o_ref).to(torch.bfloat16).to(dev)
        lse = torch.from_numpy(l_ref).float().to(dev)
    grads = ea.backward(q, k, v, o, lse, do, causal=causal, window=window, scale=scale, key_lo=klo, key_hi=khi)
    st, code, site = ea.attn_get_last_error()
    assert st == 0, f"device error code {code} at wait site {site}"
    ref = attention_bwd_ref(q64, k64, v64, do64, causal, window, scale, key_lo=lo.numpy(), key_hi=hi.numpy(),
                            o=o_ref, lse=l_ref)
    compare(grads, ref, f"{kind} B{B} Hq{Hq} Hkv{Hkv} N{N} d{d} c{int(causal)} w{window} e2e{int(end_to_end)}")
    return grads, ref


RANGE_CASES = [
    # kind, B, Hq, Hkv, N, d, causal, window, min, max
    ("documents", 2, 4, 2, 1000, 128, True, 0, 40, 400),
    ("documents", 1, 2, 2, 700, 64, False, 0, 100, 300),
    ("prefix", 2, 2, 1, 600, 128, False, 0, 1, 500),
    ("random", 1, 2, 2, 520, 128, False, 0, 1, 1),
    ("random", 1, 4, 2, 450, 64, True, 0, 1, 1),
    ("documents", 1, 2, 1, 900, 128, True, 64, 150, 600),
]


@pytest.mark.parametrize("c", RANGE_CASES, ids=lambda c: "{}_B{}h{}kv{}n{}d{}c{}w{}".format(*c[:8]))
def test_backward_with_row_ranges(c):
    run_ranges(*c, seed=7000 + c[4] + c[5])


def test_backward_with_row_ranges_end_to_end():
    run_ranges("documents", 2, 4, 2, 1100, 128, True, 0, 50, 500, seed=7100, end_to_end=True)


def test_backward_ranges_unseen_key_tiles_and_empty_query_tiles():
    """Keys [256, 384) seen by no row (their dK, dV rows are zero), query rows
    [512, 640) that see no key (their dQ rows are zero, a whole query tile)."""
    B, H, N, d = 1, 2, 768, 128
    lo = np.zeros((B, N), np.int64)
    hi = np.full((B, N), 256, np.int64)
    hi[0, 384:] = N
    lo[0, 384:] = 384
    lo[0, 512:640] = hi[0, 512:640] = 5
    grads, ref = run_ranges("custom", B, H, H, N, d, False, 0, 0, 0, seed=7200, lo=lo, hi=hi)
    dq, dk, dv = (g.float().cpu() for g in grads)
    assert torch.all(dk[:, 256:384] == 0) and torch.all(dv[:, 256:384] == 0)
    assert torch.all(dq[:, 512:640] == 0)


def test_ranges_reproducing_causal_give_the_causal_backward_bitwise():
    B, H, N, d = 2, 4, 800, 128
    inp = inputs(B, H, H, N, d, 7300)
    dev = torch.device("cuda:0")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = ea.forward(q, k, v, causal=True)
    a = ea.backward(q, k, v, o, lse, do, causal=True)
    i = torch.arange(N, dtype=torch.int32).view(1, N).repeat(B, 1)
    b = ea.backward(q, k, v, o, lse, do, causal=False, key_lo=torch.zeros_like(i).to(dev), key_hi=(i + 1).to(dev))
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_range_backward_dynamic_and_static_deals_agree_bitwise():
    """With row ranges both backward kernels take their work items from a
    counter (dynamic deal) by default: the gradients are bit-identical to the
    static deal's and to any CTA count's, on documents of unequal lengths
    (one key tile's or query tile's work is the same wherever it runs)."""
    from exact_io_aware_78_b200 import _binding as Bn
    B, Hq, Hkv, N, d = 3, 4, 2, 1500, 128
    inp = inputs(B, Hq, Hkv, N, d, 7400)
    lo, hi = make_row_ranges("documents", B, N, 7401, 30, 700)
    dev = torch.device("cuda:0")
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    klo, khi = lo.to(dev), hi.to(dev)
    o, lse = ea.forward(q, k, v, causal=True, key_lo=klo, key_hi=khi)
    ref = ea.backward(q, k, v, o, lse, do, causal=True, key_lo=klo, key_hi=khi)
    lib = ea.load_library()
    try:
        for deal, ctas in [(1, 0), (0, 1), (0, 6), (1, 6), (0, 0)]:
            assert lib.attn_set_option(Bn.EA_OPT_ITEM_DEAL, deal) == 0
            assert lib.attn_set_option(Bn.EA_OPT_MAX_CTAS, ctas) == 0
            got = ea.backward(q, k, v, o, lse, do, causal=True, key_lo=klo, key_hi=khi)
            for x, y in zip(ref, got):
                assert torch.equal(x, y), (deal, ctas)
    finally:
        lib.attn_set_option(Bn.EA_OPT_ITEM_DEAL, 0)
        lib.attn_set_option(Bn.EA_OPT_MAX_CTAS, 0)
    scale = d ** -0.5
    q64, k64, v64, do64 = (inp[n].double().numpy() for n in ("q", "k", "v", "do"))
    O, L = attention_ref(q64, k64, v64, True, 0, scale, key_lo=lo.numpy(), key_hi=hi.numpy())
    bref = attention_bwd_ref(q64, k64, v64, do64, True, 0, scale, key_lo=lo.numpy(), key_hi=hi.numpy(), o=O, lse=L)
    compare(ref, bref, "documents, dynamic deal")
