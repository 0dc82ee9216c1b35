"""Pins for the decode / split-KV oracle (Nq query rows at the end of Nk
keys; merging results over disjoint key sets).  Each pin ties the oracle to
something other than itself: the already-pinned self-attention oracle it must
reduce to, brute force written with scalar Python arithmetic, closed forms, and
the algebra of log-sum-exp.  The mutation tests plant plausible slips in the
oracle and check that a pin catches each.  CPU only."""
import math
import sys

import numpy as np
import pytest

from oracle import attention_kv_ref, attention_ref, merge_partials_ref
from oracle import decode as od

RNG = np.random.default_rng(99)


def rand(*shape):
    return RNG.standard_normal(shape)


def brute_force(q, k, v, causal, window, scale):
    """Scalar-Python definition, independent of the oracle's array code."""
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    g = Hq // Hkv
    o = np.zeros((B, Nq, Hq, v.shape[3]))
    lse = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            for i in range(Nq):
                pos = Nk - Nq + i
                keys = [j for j in range(Nk) if (not causal or j <= pos) and (window <= 0 or j > pos - window)]
                logits = [scale * sum(q[b, i, h, t] * k[b, j, h // g, t] for t in range(d)) for j in keys]
                mx = max(logits)
                ws = [math.exp(x - mx) for x in logits]
                tot = sum(ws)
                lse[b, h, i] = mx + math.log(tot)
                for c in range(v.shape[3]):
                    o[b, i, h, c] = sum(w * v[b, j, h // g, c] for w, j in zip(ws, keys)) / tot
    return o, lse


# ---------------------------------------------------------------- pins

def pin_reduces_to_self_attention():
    """Nq == Nk is ordinary self-attention (already pinned elsewhere)."""
    for causal, window in [(False, 0), (True, 0), (True, 5)]:
        q, k, v = rand(2, 13, 4, 8), rand(2, 13, 2, 8), rand(2, 13, 2, 8)
        o1, l1 = attention_kv_ref(q, k, v, causal, window)
        o2, l2 = attention_ref(q, k, v, causal, window)
        np.testing.assert_allclose(o1, o2, atol=1e-13)
        np.testing.assert_allclose(l1, l2, atol=1e-13)


def pin_decode_rows_are_the_last_rows_of_self_attention():
    """New queries are the last tokens of the sequence: their results equal
    the last Nq rows of causal self-attention over a query sequence that ends
    with them."""
    Nk, Nq = 21, 3
    q, k, v = rand(1, Nq, 4, 8), rand(1, Nk, 2, 8), rand(1, Nk, 2, 8)
    q_full = np.concatenate([rand(1, Nk - Nq, 4, 8), q], axis=1)
    for window in (0, 6):
        o1, l1 = attention_kv_ref(q, k, v, True, window)
        o2, l2 = attention_ref(q_full, k, v, True, window)
        np.testing.assert_allclose(o1, o2[:, Nk - Nq:], atol=1e-13)
        np.testing.assert_allclose(l1, l2[:, :, Nk - Nq:], atol=1e-13)


def pin_brute_force():
    for causal, window, Nq in [(False, 0, 1), (True, 0, 4), (True, 3, 2), (False, 4, 3)]:
        q, k, v = rand(1, Nq, 4, 3), rand(1, 9, 2, 3), rand(1, 9, 2, 2)
        o1, l1 = attention_kv_ref(q, k, v, causal, window, 0.7)
        o2, l2 = brute_force(q, k, v, causal, window, 0.7)
        np.testing.assert_allclose(o1, o2, atol=1e-12)
        np.testing.assert_allclose(l1, l2, atol=1e-12)


def pin_closed_forms():
    # all keys equal: uniform weights, O = mean of the allowed V rows, LSE = s + ln(count)
    Nk, d = 10, 4
    kk = np.tile(rand(1, 1, 1, d), (1, Nk, 1, 1))
    v = rand(1, Nk, 1, 3)
    q = rand(1, 2, 1, d)
    o, l = attention_kv_ref(q, kk, v, True, 0, 0.5)
    for i in range(2):
        pos = Nk - 2 + i
        np.testing.assert_allclose(o[0, i, 0], v[0, :pos + 1, 0].mean(axis=0), atol=1e-13)
        s = 0.5 * float(q[0, i, 0] @ kk[0, 0, 0])
        np.testing.assert_allclose(l[0, 0, i], s + np.log(pos + 1), atol=1e-13)
    # window 1: each query sees only the key at its own position
    q, k, v = rand(1, 3, 2, 4), rand(1, 8, 1, 4), rand(1, 8, 1, 5)
    o, _ = attention_kv_ref(q, k, v, True, 1)
    for i in range(3):
        np.testing.assert_allclose(o[0, i, :], np.tile(v[0, 8 - 3 + i, 0], (2, 1)), atol=1e-14)


def pin_merge_of_key_splits_is_the_whole():
    """Attention over disjoint key blocks, merged by their LSEs, equals
    attention over all keys (non-causal so every block is a plain slice)."""
    q, k, v = rand(2, 3, 4, 8), rand(2, 30, 2, 8), rand(2, 30, 2, 8)
    full_o, full_l = attention_kv_ref(q, k, v)
    for cuts in ([0, 30], [0, 7, 30], [0, 1, 2, 17, 29, 30]):
        parts = [attention_kv_ref(q, k[:, a:b], v[:, a:b]) for a, b in zip(cuts[:-1], cuts[1:])]
        # each part's LSE is over its own keys; rows of o are [B, Nq, Hq, dv], LSE [B, Hq, Nq]
        o_p = np.stack([p[0] for p in parts])
        l_p = np.stack([p[1].transpose(0, 2, 1) for p in parts])  # to [B, Nq, Hq]
        o, l = merge_partials_ref(o_p, l_p)
        np.testing.assert_allclose(o, full_o, atol=1e-12)
        np.testing.assert_allclose(l, full_l.transpose(0, 2, 1), atol=1e-12)


def pin_merge_closed_forms():
    o_a, o_b = rand(5, 3), rand(5, 3)
    l = rand(5)
    o, m = merge_partials_ref(np.stack([o_a, o_b]), np.stack([l, l]))
    np.testing.assert_allclose(o, (o_a + o_b) / 2, atol=1e-14)
    np.testing.assert_allclose(m, l + np.log(2.0), atol=1e-14)
    # a part with no keys (LSE -inf) contributes nothing; all parts empty gives -inf and O = 0
    o, m = merge_partials_ref(np.stack([o_a, o_b]), np.stack([l, np.full(5, -np.inf)]))
    np.testing.assert_allclose(o, o_a, atol=1e-14)
    np.testing.assert_allclose(m, l, atol=1e-14)
    o, m = merge_partials_ref(np.stack([o_a]), np.stack([np.full(5, -np.inf)]))
    assert np.all(o == 0) and np.all(np.isneginf(m))


PINS = [pin_reduces_to_self_attention, pin_decode_rows_are_the_last_rows_of_self_attention, pin_brute_force,
        pin_closed_forms, pin_merge_of_key_splits_is_the_whole, pin_merge_closed_forms]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


# ---------------------------------------------------------------- mutants

def _fails_some_pin():
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            return True
    return False


def _no_offset(q, k, v, causal=False, window=0, scale=None, rows=None):
    # queries placed at the START of the key sequence instead of its end
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Nq, Hq, d = q.shape
    Hkv = k.shape[2]
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out = np.zeros((B, Nq, Hq, v.shape[3]))
    lse = np.zeros((B, Hq, Nq))
    for b in range(B):
        for h in range(Hq):
            kh = h // (Hq // Hkv)
            o, l, _ = od._row_block(q[b, :, h], k[b, :, kh], v[b, :, kh], np.arange(Nq), causal, window, scale)
            out[b, :, h] = o
            lse[b, h] = l
    return out, lse


def _merge_unnormalised(o_parts, lse_parts):
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    w = np.exp(lse_parts - m)
    return (w[..., None] * o_parts).sum(axis=0), m + np.log(w.sum(axis=0))


def _merge_plain_mean(o_parts, lse_parts):
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    return o_parts.mean(axis=0), m + np.log(np.exp(lse_parts - m).sum(axis=0))


@pytest.mark.parametrize("target,mutant", [("attention_kv_ref", _no_offset),
                                           ("merge_partials_ref", _merge_unnormalised),
                                           ("merge_partials_ref", _merge_plain_mean)])
def test_mutant_is_caught(monkeypatch, target, mutant):
    monkeypatch.setattr(od, target, mutant)
    monkeypatch.setattr(sys.modules[__name__], target, mutant)
    assert _fails_some_pin()
