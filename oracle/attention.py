"""Float64 CPU oracle for the exact attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module; only the tests, the package's smoke check and the
benchmark's CPU-baseline leg do.  It shares no code with the CUDA path.

What it computes (per batch b and query head h, with g = Hq / Hkv query heads
per key/value head and key/value head h // g):

    S[i, j]   = scale * sum_t Q[b, i, h, t] * K[b, j, h // g, t]
    allowed   = (not causal or j <= i) and (window <= 0 or j > i - window)
                and (no row ranges or key_lo[b, i] <= j < key_hi[b, i])
    P[i, j]   = exp(S[i, j] - max_allowed S[i, :]) / sum_allowed exp(...)
    O[b,i,h]  = sum_j P[i, j] * V[b, j, h // g, :]
    LSE[b,h,i]= max_allowed S[i, :] + ln sum_allowed exp(S[i, j] - max)

Sources (the method is exact, so the oracle is the plain definition):
  * softmax(Q K^T) V as the quantity computed, with an attention mask that
    decides which queries see which keys, GQA changing only how the heads of
    Q, K, V are produced: Hacker News discussion (item 40939398), the answer
    on GQA and sliding-window attention.
  * The three steps S = Q K^T, P = softmax(S), O = P V: "Flash Attention"
    concept note (heepie.pages.dev), AS-IS sequence diagram (standard
    attention).
  * Exactness of the tiled method (same result as standard attention, not an
    approximation): same note, introduction; FlashAttention quiz
    (aiunderstanding.org), question 2; "FlashAttention-2 (PL)", opening
    paragraph.
  * Per-row key ranges (key_lo, key_hi): the mask is the thing that decides
    which queries see which keys (Hacker News discussion, same answer); the
    richer masks of the FlashMask work that "FlashAttention-2 (PL)" lists
    in its literature section are represented here by one contiguous range
    of visible keys per query row.
  * The blockwise recurrence in `online_ref`: the note's TO-BE diagram
    (per block a partial result plus a normalisation factor) and its
    "Tiling" section (scale each block's output by the right normalisation
    factors and add them up); quiz question 4 (online softmax with running
    rescaling).

Readings where the pages are silent (each listed in the design notes):
  * window: a query i sees keys j with i - window < j, i.e. at most `window`
    keys ending at itself when causal; window <= 0 means no window.
  * GQA mapping: query head h uses key/value head h // (Hq / Hkv).
  * A row with no allowed key (cannot happen with causal or no mask; it can
    with row ranges) gets O = 0 and LSE = -inf.
  * Row ranges: query row i of batch b sees keys key_lo[b, i] <= j <
    key_hi[b, i], intersected with the causal and window masks; one range
    per row, shared by all heads; any integers (lo >= hi: no key).
  * LSE is the natural-log log-sum-exp of the scaled, masked logits.
  * e4m3 inputs enter as code * per-head scale, decoded exactly here.

Parity pins (tests/test_oracle_pins.py): rows of P sum to 1; equal keys give
the mean of the attended V rows and LSE = s + ln(count); a single allowed key
returns that V row; causal row 0 equals V[0]; window 1 returns V row i;
`online_ref` equals the two-pass definition on exhaustive tiny inputs;
shift, permutation and affine invariances; the GQA reduction to repeated
heads; hand-derived golden cases; agreement with torch's float64 scaled
dot-product attention on CPU; e4m3 decoding against torch's cast.  Row
ranges (tests/test_oracle_mask_pins.py): a document mask equals separate
runs per document; ranges [i-W+1, i+1) reproduce causal + window; single
visible key and empty rows in closed form; scalar brute force; torch SDPA
with an explicit boolean mask; the blockwise recurrence.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "allowed_mask",
    "kv_head_of",
    "attention_ref",
    "probabilities_ref",
    "online_ref",
    "decode_e4m3",
    "dequantize_per_head",
]


# --------------------------------------------------------------------------
# Input decoding
# --------------------------------------------------------------------------

def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """Decode OCP FP8 E4M3 ("fn": no infinities) bytes to float64.

    Bit layout s.eeee.mmm, exponent bias 7.  e = 0 encodes subnormals
    m/8 * 2^-6; otherwise (1 + m/8) * 2^(e-7).  The pattern s.1111.111 is NaN;
    every other pattern with e = 15 is a finite normal (max 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c >> 7) & 1, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    sub = (m / 8.0) * 2.0 ** -6
    nor = (1.0 + m / 8.0) * np.power(2.0, (e - 7).astype(np.float64))
    val = sign * np.where(e == 0, sub, nor)
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return val


def dequantize_per_head(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """x = decode(code) * scale[h] for codes laid out [B, N, H, d]."""
    x = decode_e4m3(codes)
    return x * np.asarray(scale, dtype=np.float64).reshape(1, 1, -1, 1)


# --------------------------------------------------------------------------
# Mask
# --------------------------------------------------------------------------

def allowed_mask(rows: Sequence[int], N: int, causal: bool, window: int,
                 key_lo: Optional[np.ndarray] = None, key_hi: Optional[np.ndarray] = None) -> np.ndarray:
    """Boolean [len(rows), N]: which keys j each query row i may attend to.
    key_lo / key_hi, when given, are this batch's per-row bounds indexed by
    the absolute row number (length >= max(rows) + 1): row i then also needs
    key_lo[i] <= j < key_hi[i]."""
    i = np.asarray(rows, dtype=np.int64).reshape(-1, 1)
    j = np.arange(N, dtype=np.int64).reshape(1, -1)
    ok = np.ones((i.shape[0], N), dtype=bool)
    if causal:
        ok &= j <= i
    if window > 0:
        ok &= j > i - window
    if key_lo is not None:
        lo = np.asarray(key_lo, dtype=np.int64)[i[:, 0]].reshape(-1, 1)
        hi = np.asarray(key_hi, dtype=np.int64)[i[:, 0]].reshape(-1, 1)
        ok &= (j >= lo) & (j < hi)
    return ok


def kv_head_of(h: int, Hq: int, Hkv: int) -> int:
    """Key/value head used by query head h: consecutive groups of Hq / Hkv
    query heads share one key/value head."""
    return h // (Hq // Hkv)


def _check_shapes(q, k, v):
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, N, H, d]")
    B, N, Hq, d = q.shape
    if k.shape[:2] != (B, N) or v.shape[:3] != k.shape[:3]:
        raise ValueError("k, v must be [B, N, Hkv, d] with q's B and N")
    Hkv = k.shape[2]
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    if k.shape[3] != d:
        raise ValueError("q and k must share d")
    return B, N, Hq, Hkv, d


def _check_ranges(key_lo, key_hi, B, N):
    if (key_lo is None) != (key_hi is None):
        raise ValueError("key_lo and key_hi come together")
    if key_lo is None:
        return None, None
    lo = np.asarray(key_lo)
    hi = np.asarray(key_hi)
    if lo.shape != (B, N) or hi.shape != (B, N):
        raise ValueError("key_lo, key_hi must be [B, N]")
    if not (np.issubdtype(lo.dtype, np.integer) and np.issubdtype(hi.dtype, np.integer)):
        raise ValueError("key ranges are integers")
    return lo.astype(np.int64), hi.astype(np.int64)


# --------------------------------------------------------------------------
# Two-pass definition
# --------------------------------------------------------------------------

def _row_block(qb: np.ndarray, kb: np.ndarray, vb: np.ndarray, rows: np.ndarray,
               causal: bool, window: int, scale: float, lo=None, hi=None):
    """Plain definition for one (b, h) and a set of query rows.
    qb [R, d] holds those rows of Q; kb, vb are [N, d]; lo, hi are this
    batch's per-row key ranges (or None)."""
    N = kb.shape[0]
    s = scale * (qb @ kb.T)                       # S = scale * Q K^T
    ok = allowed_mask(rows, N, causal, window, lo, hi)
    s_masked = np.where(ok, s, -np.inf)
    m = s_masked.max(axis=1, keepdims=True, initial=-np.inf)  # row max, allowed keys
    any_ok = ok.any(axis=1, keepdims=True)
    m_safe = np.where(any_ok, m, 0.0)
    e = np.where(ok, np.exp(s - m_safe), 0.0)     # exp(S - max), 0 where masked
    den = e.sum(axis=1, keepdims=True)            # per-row normaliser
    p = np.divide(e, den, out=np.zeros_like(e), where=den > 0)
    o = p @ vb                                    # O = P V
    lse = np.where(any_ok[:, 0], m_safe[:, 0] + np.log(np.where(den[:, 0] > 0, den[:, 0], 1.0)),
                   -np.inf)
    return o, lse, p


def attention_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, causal: bool = False,
                  window: int = 0, scale: Optional[float] = None,
                  rows: Optional[Sequence[int]] = None,
                  row_chunk: int = 512, key_lo: Optional[np.ndarray] = None,
                  key_hi: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Exact attention forward in float64.

    q [B, N, Hq, d], k [B, N, Hkv, d], v [B, N, Hkv, dv] (any real dtype,
    upcast to float64).  Returns O [B, R, Hq, dv] and LSE [B, Hq, R] where R
    is N, or len(rows) when `rows` selects a subset of query rows (for
    sampled checks at full size).  key_lo, key_hi: optional integer [B, N]
    per-row key ranges (both or neither).  Work is chunked over rows to bound
    memory; each chunk is still the two-pass definition."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, Hq, Hkv, d = _check_shapes(q, k, v)
    key_lo, key_hi = _check_ranges(key_lo, key_hi, B, N)
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    sel = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    R = sel.shape[0]
    dv = v.shape[3]
    out = np.zeros((B, R, Hq, dv), dtype=np.float64)
    lse = np.zeros((B, Hq, R), dtype=np.float64)
    for b in range(B):
        for h in range(Hq):
            kb = k[b, :, kv_head_of(h, Hq, Hkv), :]
            vb = v[b, :, kv_head_of(h, Hq, Hkv), :]
            for c0 in range(0, R, row_chunk):
                r = sel[c0:c0 + row_chunk]
                o, l, _ = _row_block(q[b, r, h, :], kb, vb, r, causal, window, scale,
                                     None if key_lo is None else key_lo[b],
                                     None if key_hi is None else key_hi[b])
                out[b, c0:c0 + r.shape[0], h, :] = o
                lse[b, h, c0:c0 + r.shape[0]] = l
    return out, lse


def probabilities_ref(q: np.ndarray, k: np.ndarray, causal: bool = False, window: int = 0,
                      scale: Optional[float] = None, key_lo: Optional[np.ndarray] = None,
                      key_hi: Optional[np.ndarray] = None) -> np.ndarray:
    """The full probability matrix P [B, Hq, N, N] (small inputs only)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    key_lo, key_hi = _check_ranges(key_lo, key_hi, B, N)
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    P = np.zeros((B, Hq, N, N))
    rows = np.arange(N)
    for b in range(B):
        for h in range(Hq):
            kb = k[b, :, kv_head_of(h, Hq, Hkv), :]
            _, _, p = _row_block(q[b, :, h, :], kb, np.zeros((N, 1)), rows, causal, window, scale,
                                 None if key_lo is None else key_lo[b],
                                 None if key_hi is None else key_hi[b])
            P[b, h] = p
    return P


# --------------------------------------------------------------------------
# Blockwise online softmax (the tiled method, written independently)
# --------------------------------------------------------------------------

def online_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, causal: bool = False,
               window: int = 0, scale: Optional[float] = None,
               block_q: int = 1, block_k: int = 1, key_lo: Optional[np.ndarray] = None,
               key_hi: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """The tiled forward: for each block of query rows, walk the key/value
    blocks in order, keeping per row a running maximum m, a running
    normaliser l and an unnormalised partial output acc.  On each key block
    the old partial result is rescaled by exp(m_old - m_new) before the new
    block's contribution is added; at the end O = acc / l and
    LSE = m + ln l.  Float64, pure Python loops over blocks."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, N, Hq, Hkv, d = _check_shapes(q, k, v)
    key_lo, key_hi = _check_ranges(key_lo, key_hi, B, N)
    g = Hq // Hkv
    dv = v.shape[3]
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    out = np.zeros((B, N, Hq, dv))
    lse = np.zeros((B, Hq, N))
    for b in range(B):
        for h in range(Hq):
            kb_all = k[b, :, kv_head_of(h, Hq, Hkv), :]
            vb_all = v[b, :, kv_head_of(h, Hq, Hkv), :]
            for q0 in range(0, N, block_q):
                rows = np.arange(q0, min(N, q0 + block_q))
                qi = q[b, rows, h, :]
                m = np.full(rows.shape[0], -np.inf)
                l = np.zeros(rows.shape[0])
                acc = np.zeros((rows.shape[0], dv))
                for k0 in range(0, N, block_k):
                    cols = np.arange(k0, min(N, k0 + block_k))
                    s = scale * (qi @ kb_all[cols].T)
                    ok = allowed_mask(rows, N, causal, window,
                                      None if key_lo is None else key_lo[b],
                                      None if key_hi is None else key_hi[b])[:, cols]
                    s = np.where(ok, s, -np.inf)
                    m_new = np.maximum(m, s.max(axis=1))
                    # reference point for the exponentials: finite once any
                    # key of the row has been allowed
                    ref = np.where(np.isfinite(m_new), m_new, 0.0)
                    alpha = np.where(np.isfinite(m), np.exp(m - ref), 0.0)
                    p = np.where(ok, np.exp(s - ref[:, None]), 0.0)
                    acc = alpha[:, None] * acc + p @ vb_all[cols]
                    l = alpha * l + p.sum(axis=1)
                    m = m_new
                has = l > 0
                out[b, rows, h, :] = np.where(has[:, None], acc / np.where(has, l, 1.0)[:, None], 0.0)
                lse[b, h, rows] = np.where(has, m + np.log(np.where(has, l, 1.0)), -np.inf)
    return out, lse
