"""Parity of the forward with per-row key ranges (attn_fwd_masked, through
the C ABI) with the float64 oracle on seeded inputs: packed documents with
causal masking inside each document, prefix-LM masks, random ranges (empty
rows, ranges past either end, single keys), whole query tiles with no
visible key, tiles whose ranges leave a gap of K/V tiles, every element
format (bf16 d = 64 / 128, e4m3, fp32), GQA and ragged N.  Invariants: ranges
that reproduce the causal mask give results bit-identical to the causal
kernel, and ranges that cover every key give the unmasked kernel's results."""
import numpy as np
import pytest
import torch

import exact_io_aware_78_b200 as ea
from exact_io_aware_78_b200.inputs import make_inputs, make_row_ranges
from oracle import attention_ref

from gpu_helpers import assert_close, oracle_view, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(lib_path):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if torch.cuda.get_device_capability(0)[0] != 10:
        pytest.skip("needs an sm_100 GPU")
    torch.cuda.set_device(0)
    ea.load_library(lib_path)


def check(inp, causal, window, dtype, what):
    d = inp["q"].shape[3]
    scale = d ** -0.5
    O, L = run_gpu(inp, causal, window, scale)
    q, k, v = oracle_view(inp, dtype)
    lo, hi = inp["key_lo"].numpy(), inp["key_hi"].numpy()
    Oref, Lref = attention_ref(q, k, v, causal, window, scale, key_lo=lo, key_hi=hi)
    assert_close(O, L, Oref, Lref, dtype, what)
    return O, L


CASES = [
    # kind, B, Hq, Hkv, N, d, causal, window, dtype, (min_len, max_len)
    ("documents", 2, 4, 2, 1000, 128, True, 0, "bf16", (40, 300)),
    ("documents", 1, 2, 2, 777, 128, False, 0, "bf16", (100, 500)),
    ("documents", 2, 4, 4, 640, 64, True, 0, "bf16", (1, 200)),
    ("documents", 1, 4, 1, 1300, 128, True, 100, "bf16", (200, 900)),   # window inside documents
    ("prefix", 2, 4, 2, 900, 128, False, 0, "bf16", (1, 700)),
    ("prefix", 1, 2, 2, 513, 64, False, 0, "bf16", (300, 300)),
    ("random", 2, 2, 1, 600, 128, False, 0, "bf16", (0, 0)),
    ("random", 1, 4, 2, 700, 128, True, 0, "bf16", (0, 0)),
    ("random", 1, 2, 2, 450, 64, False, 37, "bf16", (0, 0)),
    ("documents", 2, 4, 4, 1024, 128, True, 0, "fp8", (64, 512)),
    ("random", 1, 2, 2, 500, 128, False, 0, "fp8", (0, 0)),
    ("documents", 1, 2, 1, 400, 64, True, 0, "fp32", (30, 150)),
    ("random", 1, 2, 2, 300, 64, False, 0, "fp32", (0, 0)),
]


@pytest.mark.parametrize("c", CASES, ids=lambda c: "{}_B{}h{}kv{}n{}d{}c{}w{}_{}".format(*c[:9]))
def test_small_shapes(c):
    kind, B, Hq, Hkv, N, d, causal, window, dtype, (mn, mx) = c
    seed = 3000 + N + d + Hq
    inp = make_inputs(B, Hq, Hkv, N, d, dtype, seed)
    inp["key_lo"], inp["key_hi"] = make_row_ranges(kind, B, N, seed + 3, max(mn, 1), mx)
    check(inp, causal, window, dtype, str(c))


def _with_ranges(inp, lo, hi):
    out = dict(inp)
    out["key_lo"] = torch.as_tensor(lo, dtype=torch.int32).contiguous()
    out["key_hi"] = torch.as_tensor(hi, dtype=torch.int32).contiguous()
    return out


def test_empty_tiles_and_gaps():
    """Query tiles no row of which sees a key (the second tile of a work
    item, the first, both), rows that see no key inside live tiles, and two
    tiles of one work item whose key ranges leave a gap of K/V tiles."""
    B, H, N, d = 1, 2, 1280, 128
    inp = make_inputs(B, H, H, N, d, "bf16", 91)
    lo = np.zeros((B, N), np.int64)
    hi = np.full((B, N), N, np.int64)
    lo[0, 128:256] = hi[0, 128:256] = 0          # tile 1 of item 0 empty
    lo[0, 256:384] = 5                           # tile 2 empty (lo >= hi)
    hi[0, 256:384] = 5
    lo[0, 512:768] = N                           # item 2: both tiles empty (ranges past the end)
    hi[0, 512:768] = N + 10
    lo[0, 768:896] = 0                           # item 3, tile 0: keys [0, 200)
    hi[0, 768:896] = 200
    lo[0, 896:1024] = 1000                       # item 3, tile 1: keys [1000, 1100): a gap of K/V tiles
    hi[0, 896:1024] = 1100
    hi[0, 1024:1280:3] = -1                      # scattered empty rows in a live item
    check(_with_ranges(inp, lo, hi), False, 0, "bf16", "empty tiles and gaps")
    check(_with_ranges(inp, lo, hi), True, 0, "bf16", "empty tiles and gaps, causal")


def _raw(inp, causal, window, lo=None, hi=None):
    dev = torch.device("cuda:0")
    q, k, v = (inp[n].to(dev) for n in "qkv")
    kw = {}
    if lo is not None:
        kw = dict(key_lo=torch.as_tensor(lo, dtype=torch.int32).to(dev),
                  key_hi=torch.as_tensor(hi, dtype=torch.int32).to(dev))
    o, lse = ea.forward(q, k, v, causal=causal, window=window, **kw)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def test_ranges_reproducing_causal_are_bit_identical():
    """Ranges [0, i + 1) without the causal flag, and [i - W + 1, i + 1) for a
    window, visit the same K/V tiles and mask the same scores as the causal /
    window kernel: the results are bit-identical."""
    B, H, N, d = 2, 4, 1100, 128
    inp = make_inputs(B, H, H, N, d, "bf16", 92)
    i = np.arange(N)[None, :].repeat(B, 0)
    o1, l1 = _raw(inp, True, 0)
    o2, l2 = _raw(inp, False, 0, np.zeros_like(i), i + 1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o1, l1 = _raw(inp, True, 300)
    o2, l2 = _raw(inp, False, 0, i - 299, i + 1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_full_ranges_equal_the_unmasked_kernel():
    B, Hq, Hkv, N, d = 1, 4, 2, 900, 64
    inp = make_inputs(B, Hq, Hkv, N, d, "bf16", 93)
    lo = np.full((B, N), -5)
    hi = np.full((B, N), N + 5)
    o1, l1 = _raw(inp, False, 0)
    o2, l2 = _raw(inp, False, 0, lo, hi)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    o1, l1 = _raw(inp, True, 0)
    o2, l2 = _raw(inp, True, 0, lo, hi)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_masked_runs_repeat_bitwise():
    B, H, N, d = 2, 4, 2000, 128
    inp = make_inputs(B, H, H, N, d, "bf16", 94)
    lo, hi = make_row_ranges("documents", B, N, 97, 50, 600)
    a = _raw(inp, True, 0, lo, hi)
    b = _raw(inp, True, 0, lo, hi)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_ranked_and_unranked_schedules_agree_bitwise():
    """The schedule (default, lightest first, or (batch, query block) pairs
    ranked by cost; items taken from a counter or dealt statically; any CTA
    count) only changes which CTA takes which item: all give bit-identical
    results, on a batch of many pairs with unequal costs."""
    from exact_io_aware_78_b200 import _binding as Bn
    B, H, N, d = 24, 2, 1536, 64
    inp = make_inputs(B, H, H, N, d, "bf16", 95)
    lo, hi = make_row_ranges("documents", B, N, 96, 30, 1500)
    a = _raw(inp, True, 0, lo, hi)
    lib = ea.load_library()
    for order in (1, 2):
        assert lib.attn_set_option(Bn.EA_OPT_SCHEDULE_ORDER, order) == 0
        try:
            b = _raw(inp, True, 0, lo, hi)
        finally:
            lib.attn_set_option(Bn.EA_OPT_SCHEDULE_ORDER, 0)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    # the dynamic deal (the default with ranges) against the static one, and
    # under CTA counts that make each CTA take many items from the counter
    for deal, ctas in [(1, 0), (0, 1), (0, 5), (1, 5), (0, 0)]:
        assert lib.attn_set_option(Bn.EA_OPT_ITEM_DEAL, deal) == 0
        assert lib.attn_set_option(Bn.EA_OPT_MAX_CTAS, ctas) == 0
        try:
            b = _raw(inp, True, 0, lo, hi)
        finally:
            lib.attn_set_option(Bn.EA_OPT_ITEM_DEAL, 0)
            lib.attn_set_option(Bn.EA_OPT_MAX_CTAS, 0)
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]), (deal, ctas)
    q, k, v = oracle_view(inp, "bf16")
    rows = list(range(0, N, 97)) + [N - 1]
    Oref, Lref = attention_ref(q, k, v, True, 0, d ** -0.5, rows=rows, key_lo=lo.numpy(), key_hi=hi.numpy())
    assert_close(a[0].double().numpy()[:, rows], a[1].double().numpy()[:, :, rows], Oref, Lref, "bf16",
                 "ranked schedule, 24 batches")
