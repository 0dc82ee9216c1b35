"""Pins for the oracle's per-row key ranges (key_lo <= j < key_hi per query
row, intersected with the causal and window masks).  Each pin ties the
oracle to something other than itself: independent sub-problems (a document
mask equals attention run on each document alone), the already-pinned
causal/window mask it must reproduce, closed forms (a single visible key, no
visible key), scalar-Python brute force, torch's float64 scaled dot-product
attention with an explicit boolean mask, and the blockwise recurrence.  The
mutation tests plant plausible slips in the oracle's mask and check that a
pin catches each.  CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle.attention as oa
from oracle import attention_ref, online_ref
from exact_io_aware_78_b200.inputs import make_row_ranges

RNG = np.random.default_rng(2024)


def rand(*shape):
    return RNG.standard_normal(shape)


def ranges(kind, B, N, seed, lo=1, hi=0):
    a, b = make_row_ranges(kind, B, N, seed, lo, hi)
    return a.numpy(), b.numpy()


def doc_bounds(lo_row):
    """Start indices of the documents of one batch row of a "documents" mask."""
    starts = sorted(set(int(x) for x in lo_row))
    return starts + [len(lo_row)]


# ---------------------------------------------------------------- pins

def pin_documents_equal_separate_runs():
    """A document mask is block-diagonal: each document's rows equal the
    oracle run on that document's slice of Q, K, V alone (no row ranges),
    with and without causal masking inside the document."""
    B, N, Hq, Hkv, d = 2, 37, 4, 2, 8
    q, k, v = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d)
    lo, hi = ranges("documents", B, N, 7, 3, 11)
    for causal in (False, True):
        o, l = attention_ref(q, k, v, causal, 0, key_lo=lo, key_hi=hi)
        for b in range(B):
            bounds = doc_bounds(lo[b])
            assert len(bounds) > 3
            for s, e in zip(bounds[:-1], bounds[1:]):
                o2, l2 = attention_ref(q[b:b + 1, s:e], k[b:b + 1, s:e], v[b:b + 1, s:e], causal, 0)
                np.testing.assert_allclose(o[b:b + 1, s:e], o2, atol=1e-13)
                np.testing.assert_allclose(l[b:b + 1, :, s:e], l2, atol=1e-13)


def pin_ranges_reproduce_causal_window():
    """Row ranges [i - W + 1, i + 1) with no causal flag reproduce the causal
    + window mask, and [0, i + 1) reproduces causal alone."""
    q, k, v = rand(1, 29, 2, 8), rand(1, 29, 2, 8), rand(1, 29, 2, 8)
    i = np.arange(29).reshape(1, -1)
    for W in (1, 4, 40):
        o, l = attention_ref(q, k, v, False, 0, key_lo=i - W + 1, key_hi=i + 1)
        o2, l2 = attention_ref(q, k, v, True, W)
        np.testing.assert_allclose(o, o2, atol=1e-13)
        np.testing.assert_allclose(l, l2, atol=1e-13)
    o, l = attention_ref(q, k, v, False, 0, key_lo=np.zeros_like(i), key_hi=i + 1)
    o2, l2 = attention_ref(q, k, v, True, 0)
    np.testing.assert_allclose(o, o2, atol=1e-13)


def pin_single_key_and_empty_rows():
    """A row that sees one key j returns V[j] with LSE = scale q.k_j; a row
    that sees none (lo >= hi, a range outside [0, N), or a range that the
    causal mask removes) returns O = 0 and LSE = -inf."""
    B, N, d = 1, 12, 8
    q, k, v = rand(B, N, 1, d), rand(B, N, 1, d), rand(B, N, 1, d)
    j = RNG.integers(0, N, N)
    lo = j.reshape(1, -1)
    o, l = attention_ref(q, k, v, False, 0, key_lo=lo, key_hi=lo + 1)
    for i in range(N):
        np.testing.assert_allclose(o[0, i, 0], v[0, j[i], 0], atol=1e-14)
        assert abs(l[0, 0, i] - q[0, i, 0] @ k[0, j[i], 0] / math.sqrt(d)) < 1e-13
    empty_lo = np.array([[5, 3, -4, N, N + 3, 0, 7, 2, 9, 11, 6, 1]])
    empty_hi = np.array([[5, 2, 0, N + 2, N + 9, 0, 7, 1, 9, 11, 6, 1]])
    o, l = attention_ref(q, k, v, False, 0, key_lo=empty_lo, key_hi=empty_hi)
    assert np.all(o == 0) and np.all(np.isneginf(l))
    # causal removes every key of ranges that start after the row
    i = np.arange(N).reshape(1, -1)
    o, l = attention_ref(q, k, v, True, 0, key_lo=i + 1, key_hi=i + 4)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def pin_brute_force_random_ranges():
    """Scalar Python over explicit key lists, random ranges (including empty
    and out-of-range ones), GQA, causal and window on top."""
    B, N, Hq, Hkv, d = 2, 9, 4, 2, 3
    q, k, v = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d)
    lo, hi = ranges("random", B, N, 11)
    for causal, window in [(False, 0), (True, 0), (True, 3), (False, 4)]:
        o, l = attention_ref(q, k, v, causal, window, key_lo=lo, key_hi=hi)
        for b in range(B):
            for h in range(Hq):
                for i in range(N):
                    keys = [jj for jj in range(N) if lo[b, i] <= jj < hi[b, i] and (not causal or jj <= i)
                            and (window <= 0 or jj > i - window)]
                    if not keys:
                        assert np.isneginf(l[b, h, i]) and np.all(o[b, i, h] == 0)
                        continue
                    s = [sum(q[b, i, h, t] * k[b, jj, h // 2, t] for t in range(d)) / math.sqrt(d) for jj in keys]
                    mx = max(s)
                    w = [math.exp(x - mx) for x in s]
                    assert abs(l[b, h, i] - (mx + math.log(sum(w)))) < 1e-12
                    for c in range(d):
                        ref = sum(wi * v[b, jj, h // 2, c] for wi, jj in zip(w, keys)) / sum(w)
                        assert abs(o[b, i, h, c] - ref) < 1e-12


def pin_torch_sdpa_boolean_mask():
    """torch's float64 scaled dot-product attention on CPU with the boolean
    mask built from the ranges (rows with at least one visible key)."""
    B, N, H, d = 2, 40, 3, 16
    q, k, v = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    for kind, causal in [("documents", True), ("prefix", False), ("random", False)]:
        lo, hi = ranges(kind, B, N, 5, 4, 15)
        o, l = attention_ref(q, k, v, causal, 0, key_lo=lo, key_hi=hi)
        jj = torch.arange(N).view(1, 1, N)
        ii = torch.arange(N).view(1, N, 1)
        m = (jj >= torch.from_numpy(lo).view(B, N, 1)) & (jj < torch.from_numpy(hi).view(B, N, 1))
        if causal:
            m &= jj <= ii
        has = m.any(-1)
        t = lambda x: torch.from_numpy(x).permute(0, 2, 1, 3)
        ref = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m.unsqueeze(1))
        ref = ref.permute(0, 2, 1, 3).numpy()
        sel = has.numpy()
        np.testing.assert_allclose(o[sel], ref[sel], atol=1e-12)
        assert np.all(o[~sel] == 0)


def pin_online_equals_two_pass_with_ranges():
    """The blockwise recurrence with blocks that a row's range covers fully,
    partly or not at all gives the two-pass result."""
    B, N, Hq, Hkv, d = 1, 23, 2, 1, 5
    q, k, v = rand(B, N, Hq, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d)
    for kind in ("documents", "random"):
        lo, hi = ranges(kind, B, N, 3, 2, 9)
        o, l = attention_ref(q, k, v, True, 0, key_lo=lo, key_hi=hi)
        for bq, bk in [(1, 1), (4, 3), (8, 5)]:
            o2, l2 = online_ref(q, k, v, True, 0, block_q=bq, block_k=bk, key_lo=lo, key_hi=hi)
            np.testing.assert_allclose(o, o2, atol=1e-13)
            fin = np.isfinite(l)
            assert np.array_equal(fin, np.isfinite(l2))
            np.testing.assert_allclose(l[fin], l2[fin], atol=1e-13)


PINS = [pin_documents_equal_separate_runs, pin_ranges_reproduce_causal_window, pin_single_key_and_empty_rows,
        pin_brute_force_random_ranges, pin_torch_sdpa_boolean_mask, pin_online_equals_two_pass_with_ranges]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_ranges_are_checked():
    q = rand(1, 4, 1, 2)
    with pytest.raises(ValueError):
        attention_ref(q, q, q, key_lo=np.zeros((1, 4), dtype=np.int64))
    with pytest.raises(ValueError):
        attention_ref(q, q, q, key_lo=np.zeros((1, 3), dtype=np.int64), key_hi=np.ones((1, 3), dtype=np.int64))


def test_range_generators():
    lo, hi = make_row_ranges("documents", 3, 1000, 1, 50, 200)
    for b in range(3):
        starts = doc_bounds(lo[b].numpy())
        assert starts[0] == 0 and starts[-1] == 1000
        lens = np.diff(starts)
        assert np.all(lens[:-1] >= 50) and np.all(lens <= 200)
        for s, e in zip(starts[:-1], starts[1:]):
            assert torch.all(lo[b, s:e] == s) and torch.all(hi[b, s:e] == e)
    lo, hi = make_row_ranges("prefix", 1, 30, 2, 5, 9)
    P = int(hi[0, 0])
    assert 5 <= P <= 9 and torch.all(lo == 0)
    assert torch.all(hi[0, :P] == P) and torch.all(hi[0, P:] == torch.arange(P, 30) + 1)
    a1, b1 = make_row_ranges("random", 2, 64, 9)
    a2, b2 = make_row_ranges("random", 2, 64, 9)
    assert torch.equal(a1, a2) and torch.equal(b1, b2)
    assert (b1 <= a1).any() and (a1 < 0).any() and (b1 > 64).any()


# ---------------------------------------------------------------- mutants

def _mask_hi_inclusive(rows, N, causal, window, key_lo=None, key_hi=None):
    return _orig(rows, N, causal, window, key_lo, None if key_hi is None else np.asarray(key_hi) + 1)


def _mask_ignores_lo(rows, N, causal, window, key_lo=None, key_hi=None):
    return _orig(rows, N, causal, window, None if key_lo is None else np.zeros_like(key_lo), key_hi)


def _mask_ranges_replace_causal(rows, N, causal, window, key_lo=None, key_hi=None):
    return _orig(rows, N, causal and key_lo is None, window, key_lo, key_hi)


def _mask_ranges_by_column(rows, N, causal, window, key_lo=None, key_hi=None):
    """Ranges applied per key column instead of per query row."""
    ok = _orig(rows, N, causal, window)
    if key_lo is not None:
        i = np.asarray(rows).reshape(-1, 1)
        j = np.arange(N).reshape(1, -1)
        ok &= (i >= np.asarray(key_lo)[j]) & (i < np.asarray(key_hi)[j])
    return ok


_orig = oa.allowed_mask


@pytest.mark.parametrize("mutant", [_mask_hi_inclusive, _mask_ignores_lo, _mask_ranges_replace_causal,
                                    _mask_ranges_by_column], ids=lambda f: f.__name__)
def test_mutant_is_caught(monkeypatch, mutant):
    monkeypatch.setattr(oa, "allowed_mask", mutant)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught {mutant.__name__}"
