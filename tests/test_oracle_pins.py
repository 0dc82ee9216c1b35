"""Pins for the float64 oracle: facts fixed by the pages and by mathematics,
each chosen so that a plausible slip in the oracle (a dropped term, a wrong
sign or index, a transposed operand, an off-by-one mask) breaks at least one
of them.  The mutation tests at the end plant such slips in the oracle and
check that the pins catch them.  CPU only."""
import json
import os

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import (allowed_mask, attention_ref, decode_e4m3, dequantize_per_head,
                    online_ref, probabilities_ref)

HERE = os.path.dirname(os.path.abspath(__file__))
RNG = np.random.default_rng(20240711)


def rand(*shape, rng=RNG):
    return rng.standard_normal(shape)


# ---------------------------------------------------------------- pin helpers
# Each helper raises AssertionError when its fact does not hold, so that the
# mutation tests can reuse them.

def pin_rows_sum_to_one():
    for causal, window in [(False, 0), (True, 0), (True, 3), (False, 4)]:
        q, k = rand(2, 11, 3, 5), rand(2, 11, 3, 5)
        P = probabilities_ref(q, k, causal, window)
        np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-12)
        # and nothing outside the mask carries weight
        ok = allowed_mask(range(11), 11, causal, window)
        assert np.all(P[..., ~ok] == 0.0)


def pin_equal_keys_give_mean():
    """All keys equal: every allowed logit in a row is the same, so P is
    uniform over the allowed keys, O_i is the mean of those V rows and
    LSE_i = s_i + ln(count_i)."""
    N, d = 13, 6
    for causal, window in [(False, 0), (True, 0), (True, 4)]:
        q = rand(1, N, 2, d)
        k = np.repeat(rand(1, 1, 2, d), N, axis=1)
        v = rand(1, N, 2, 3)
        O, L = attention_ref(q, k, v, causal, window, scale=0.7)
        ok = allowed_mask(range(N), N, causal, window)
        for h in range(2):
            s = 0.7 * q[0, :, h, :] @ k[0, 0, h, :]
            for i in range(N):
                js = np.nonzero(ok[i])[0]
                np.testing.assert_allclose(O[0, i, h], v[0, js, h].mean(0), atol=1e-12)
                np.testing.assert_allclose(L[0, h, i], s[i] + np.log(len(js)), atol=1e-12)


def pin_single_allowed_key():
    """Causal with window 1: row i sees only key i, so O_i = V_i and LSE_i = S_ii."""
    N, d = 9, 4
    q, k, v = rand(2, N, 3, d), rand(2, N, 3, d), rand(2, N, 3, 7)
    O, L = attention_ref(q, k, v, causal=True, window=1, scale=0.3)
    np.testing.assert_allclose(O, v, atol=1e-12)
    s_diag = 0.3 * np.einsum("bnhd,bnhd->bhn", q, k)
    np.testing.assert_allclose(L, s_diag, atol=1e-12)


def pin_causal_row0():
    q, k, v = rand(3, 17, 2, 8), rand(3, 17, 2, 8), rand(3, 17, 2, 8)
    O, L = attention_ref(q, k, v, causal=True)
    np.testing.assert_allclose(O[:, 0], v[:, 0], atol=1e-12)
    s00 = np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]) / np.sqrt(8)
    np.testing.assert_allclose(L[:, :, 0], s00, atol=1e-12)


def pin_torch_sdpa():
    """Agreement with torch's float64 CPU scaled_dot_product_attention (a
    library routine used only as a comparator), with GQA expanded by
    repeating each key/value head over its group."""
    for causal, window, g in [(False, 0, 1), (True, 0, 2), (True, 5, 4), (False, 3, 1)]:
        B, N, Hkv, d = 2, 23, 2, 16
        q, k, v = rand(B, N, Hkv * g, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d)
        O, L = attention_ref(q, k, v, causal, window, scale=0.21)
        qt = torch.tensor(q).permute(0, 2, 1, 3)
        kt = torch.tensor(k).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
        vt = torch.tensor(v).permute(0, 2, 1, 3).repeat_interleave(g, dim=1)
        mask = torch.ones(N, N, dtype=torch.bool)
        if causal:
            mask &= torch.ones(N, N, dtype=torch.bool).tril()
        if window > 0:
            mask &= torch.ones(N, N, dtype=torch.bool).triu(-(window - 1))
        ot = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=0.21)
        np.testing.assert_allclose(O, ot.permute(0, 2, 1, 3).numpy(), atol=1e-10)
        s = torch.einsum("bhid,bhjd->bhij", qt, kt) * 0.21
        lt = torch.logsumexp(s.masked_fill(~mask, float("-inf")), dim=-1)
        np.testing.assert_allclose(L, lt.numpy(), atol=1e-10)


def pin_golden():
    with open(os.path.join(HERE, "golden", "hand_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q, k, v = (np.array(c[x])[None] for x in "qkv")
        O, L = attention_ref(q, k, v, c["causal"], c["window"], c["scale"])
        np.testing.assert_allclose(O[0], np.array(c["o"]), atol=1e-12, err_msg=c["name"])
        np.testing.assert_allclose(L[0], np.array(c["lse"]), atol=1e-12, err_msg=c["name"])


def pin_gqa_equals_repeated_heads():
    B, N, Hkv, g, d = 2, 10, 3, 4, 5
    q, k, v = rand(B, N, Hkv * g, d), rand(B, N, Hkv, d), rand(B, N, Hkv, d)
    O, L = attention_ref(q, k, v, True, 0)
    for h in range(Hkv * g):
        O1, L1 = attention_ref(q[:, :, h:h + 1], k[:, :, h // g:h // g + 1],
                               v[:, :, h // g:h // g + 1], True, 0)
        np.testing.assert_allclose(O[:, :, h], O1[:, :, 0], atol=1e-13)
        np.testing.assert_allclose(L[:, h], L1[:, 0], atol=1e-13)


PINS = [pin_rows_sum_to_one, pin_equal_keys_give_mean, pin_single_allowed_key, pin_causal_row0,
        pin_torch_sdpa, pin_golden, pin_gqa_equals_repeated_heads]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin()


# ------------------------------------------------------- online vs two-pass
def test_online_equals_two_pass_exhaustive_tiny():
    """The tiled online recurrence reaches the two-pass result on every tiny
    shape, mask and block size (brute force over the combinations)."""
    rng = np.random.default_rng(7)
    count = 0
    for N in range(1, 10):
        for d in (1, 2, 4):
            q, k, v = (rng.standard_normal((1, N, 1, d)) * 2 for _ in range(3))
            for causal in (False, True):
                for window in range(0, N + 2):
                    O, L = attention_ref(q, k, v, causal, window)
                    for bq in range(1, N + 1):
                        for bk in range(1, N + 1):
                            O2, L2 = online_ref(q, k, v, causal, window, block_q=bq, block_k=bk)
                            np.testing.assert_allclose(O2, O, atol=1e-12, rtol=0)
                            np.testing.assert_allclose(L2, L, atol=1e-12, rtol=0)
                            count += 1
    assert count > 1000


def test_online_equals_two_pass_gqa_ragged_blocks():
    q, k, v = rand(2, 45, 8, 16), rand(2, 45, 2, 16), rand(2, 45, 2, 16)
    for causal, window in [(False, 0), (True, 0), (True, 7)]:
        O, L = attention_ref(q, k, v, causal, window)
        O2, L2 = online_ref(q, k, v, causal, window, block_q=16, block_k=13)
        np.testing.assert_allclose(O2, O, atol=1e-12)
        np.testing.assert_allclose(L2, L, atol=1e-12)


# ---------------------------------------------------------------- invariances
def test_shift_invariance_of_keys():
    """K_j -> K_j + c for every key adds scale * q_i . c to the whole row:
    O is unchanged and LSE shifts by exactly that amount."""
    q, k, v = rand(1, 12, 2, 6), rand(1, 12, 2, 6), rand(1, 12, 2, 6)
    c = rand(6)
    for causal, window in [(False, 0), (True, 0), (True, 5)]:
        O, L = attention_ref(q, k, v, causal, window, scale=0.4)
        O2, L2 = attention_ref(q, k + c, v, causal, window, scale=0.4)
        np.testing.assert_allclose(O2, O, atol=1e-12)
        np.testing.assert_allclose(L2 - L, 0.4 * np.einsum("bnhd,d->bhn", q, c), atol=1e-12)


def test_joint_key_value_permutation_noncausal():
    q, k, v = rand(2, 15, 3, 4), rand(2, 15, 3, 4), rand(2, 15, 3, 4)
    perm = np.random.default_rng(3).permutation(15)
    O, L = attention_ref(q, k, v)
    O2, L2 = attention_ref(q, k[:, perm], v[:, perm])
    np.testing.assert_allclose(O2, O, atol=1e-12)
    np.testing.assert_allclose(L2, L, atol=1e-12)


def test_affine_values():
    """Rows of P sum to 1, so O(a V + b) = a O + b."""
    q, k, v = rand(1, 14, 2, 4), rand(1, 14, 2, 4), rand(1, 14, 2, 4)
    b = rand(4)
    O, _ = attention_ref(q, k, v, True, 6)
    O2, _ = attention_ref(q, k, -2.5 * v + b, True, 6)
    np.testing.assert_allclose(O2, -2.5 * O + b, atol=1e-12)


def test_row_subset_matches_full():
    q, k, v = rand(2, 40, 4, 8), rand(2, 40, 2, 8), rand(2, 40, 2, 8)
    rows = [0, 3, 17, 39]
    O, L = attention_ref(q, k, v, True, 9)
    O2, L2 = attention_ref(q, k, v, True, 9, rows=rows, row_chunk=3)
    np.testing.assert_allclose(O2, O[:, rows], atol=1e-14)
    np.testing.assert_allclose(L2, L[:, :, rows], atol=1e-14)


def test_fully_masked_row_reading():
    """Non-causal with a window is the one mask where a row could see no key
    if the window were empty; with window >= 1 every row sees itself.  The
    defined fallback O = 0, LSE = -inf is exercised by an explicit empty
    mask on the two-pass helper."""
    qb, kb, vb = rand(2, 3), rand(4, 3), rand(4, 2)
    o, lse, p = oa._row_block(qb, kb, vb, np.array([0, 1]), True, 0, 1.0)
    assert np.isfinite(lse).all()
    o, lse, p = oa._row_block(qb, kb[:0], vb[:0], np.array([0, 1]), True, 0, 1.0)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


# ---------------------------------------------------------------- e4m3 decode
def test_e4m3_decode_matches_torch_cast_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_dequantize_per_head_broadcasts_over_heads():
    codes = np.full((1, 2, 3, 4), 0x38, dtype=np.uint8)  # 1.0
    x = dequantize_per_head(codes, np.array([1.0, 2.0, 0.5]))
    np.testing.assert_array_equal(x[0, 0, :, 0], [1.0, 2.0, 0.5])


# --------------------------------------------------------- planted mistakes
def _bad_mask_strict_causal(rows, N, causal, window, key_lo=None, key_hi=None):
    i = np.asarray(rows).reshape(-1, 1)
    j = np.arange(N).reshape(1, -1)
    ok = np.ones((i.shape[0], N), dtype=bool)
    if causal:
        ok &= j < i          # diagonal dropped
    if window > 0:
        ok &= j > i - window
    return ok


def _bad_mask_wide_window(rows, N, causal, window, key_lo=None, key_hi=None):
    i = np.asarray(rows).reshape(-1, 1)
    j = np.arange(N).reshape(1, -1)
    ok = np.ones((i.shape[0], N), dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j >= i - window  # one key too many
    return ok


def _bad_row_block_transposed_values(qb, kb, vb, rows, causal, window, scale, lo=None, hi=None):
    o, lse, p = _orig_row_block(qb, kb, vb, rows, causal, window, scale, lo, hi)
    # P^T V instead of P V (only shape-compatible when R == N)
    if p.shape[0] == p.shape[1]:
        o = p.T @ vb
    return o, lse, p


def _bad_row_block_log2_lse(qb, kb, vb, rows, causal, window, scale, lo=None, hi=None):
    o, lse, p = _orig_row_block(qb, kb, vb, rows, causal, window, scale, lo, hi)
    return o, lse / np.log(2.0), p


def _bad_row_block_no_scale(qb, kb, vb, rows, causal, window, scale, lo=None, hi=None):
    return _orig_row_block(qb, kb, vb, rows, causal, window, 1.0, lo, hi)


def _bad_row_block_column_softmax(qb, kb, vb, rows, causal, window, scale, lo=None, hi=None):
    s = scale * (qb @ kb.T)
    ok = allowed_mask(rows, kb.shape[0], causal, window, lo, hi)
    e = np.where(ok, np.exp(s), 0.0)
    den = e.sum(axis=0, keepdims=True)   # normalised over the wrong axis
    p = np.divide(e, den, out=np.zeros_like(e), where=den > 0)
    lse = np.log(e.sum(axis=1))
    return p @ vb, lse, p


def _bad_row_block_negated_logits(qb, kb, vb, rows, causal, window, scale, lo=None, hi=None):
    return _orig_row_block(-qb, kb, vb, rows, causal, window, scale, lo, hi)


_orig_row_block = oa._row_block

MUTANTS = {
    "causal_drops_diagonal": ("allowed_mask", _bad_mask_strict_causal),
    "window_one_key_too_wide": ("allowed_mask", _bad_mask_wide_window),
    "gqa_heads_interleaved": ("kv_head_of", lambda h, Hq, Hkv: h % Hkv),
    "values_transposed": ("_row_block", _bad_row_block_transposed_values),
    "lse_in_log2": ("_row_block", _bad_row_block_log2_lse),
    "scale_dropped": ("_row_block", _bad_row_block_no_scale),
    "softmax_over_queries": ("_row_block", _bad_row_block_column_softmax),
    "logit_sign_flipped": ("_row_block", _bad_row_block_negated_logits),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    attr, bad = MUTANTS[name]
    monkeypatch.setattr(oa, attr, bad)
    caught = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
