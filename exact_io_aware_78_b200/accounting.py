"""FLOP and byte accounting used to report throughput and roofline fractions.

The forward pass does two dense contractions per attended (query, key) pair,
S = Q K^T and O += P V, each 2*d FLOPs, so 4*d FLOPs per pair.  The
algorithmic bytes are those of the IO-aware schedule: Q, K, V read once and
O plus the per-row log-sum-exp written once; no N x N matrix ever moves
(FlashAttention concept note (heepie.pages.dev), "IO complexity" table).
"""
from __future__ import annotations

import numpy as np

from .inputs import Workload, make_row_ranges


def attended_pairs(N: int, causal: bool, window: int) -> int:
    """Count pairs (i, j), 0 <= i, j < N, with (not causal or j <= i) and
    (window <= 0 or j > i - window)."""
    if not causal and window <= 0:
        return N * N
    if causal and window <= 0:
        return N * (N + 1) // 2
    w = min(window, N)
    if causal:
        # rows i < w see i + 1 keys; rows i >= w see w keys
        return w * (w + 1) // 2 + (N - w) * w
    # non-causal with a left bound: row i sees keys j in (i - window, N)
    # rows i < w see all N keys; row i >= w sees N - (i - w + 1) keys
    tail = N - w
    return w * N + tail * N - (tail * (tail + 1)) // 2


def range_pairs(key_lo, key_hi, causal: bool, window: int) -> int:
    """Attended pairs over all batches of per-row key ranges ([B, N] integer
    arrays): row i sees keys [max(lo_i, 0, i - window + 1), min(hi_i, N, i + 1)),
    the window and causal bounds applying only when set."""
    lo = np.asarray(key_lo, dtype=np.int64)
    hi = np.asarray(key_hi, dtype=np.int64)
    N = lo.shape[-1]
    i = np.arange(N, dtype=np.int64)
    a = np.maximum(lo, 0)
    b = np.minimum(hi, N)
    if window > 0:
        a = np.maximum(a, i - window + 1)
    if causal:
        b = np.minimum(b, i + 1)
    return int(np.maximum(b - a, 0).sum())


def workload_pairs(w: Workload) -> int:
    """Attended pairs of one query head summed over the batch."""
    if w.mask:
        lo, hi = make_row_ranges(w.mask, w.B, w.N, w.seed + 3, w.mask_min, w.mask_max)
        return range_pairs(lo.numpy(), hi.numpy(), w.causal, w.window)
    return w.B * attended_pairs(w.N, w.causal, w.window)


def flops(w: Workload) -> float:
    """4 * d FLOPs per attended pair, summed over batch and query heads."""
    return 4.0 * w.Hq * w.d * workload_pairs(w)


def flops_half_square(w: Workload) -> float:
    """4*B*Hq*N^2*d, halved when causal; ignores the sliding window."""
    f = 4.0 * w.B * w.Hq * w.N * w.N * w.d
    return f / 2 if w.causal else f


def element_bytes(dtype: str) -> int:
    return {"fp32": 4, "bf16": 2, "fp8": 1}[dtype]


def out_bytes(dtype: str) -> int:
    """O is fp32 for fp32 inputs and bf16 otherwise."""
    return 4 if dtype == "fp32" else 2


def algorithmic_bytes(w: Workload) -> int:
    """Read Q, K, V (and fp8 scales) once; write O and the fp32 LSE once."""
    e = element_bytes(w.dtype)
    q = w.B * w.N * w.Hq * w.d * e
    kv = 2 * w.B * w.N * w.Hkv * w.d * e
    o = w.B * w.N * w.Hq * w.d * out_bytes(w.dtype)
    lse = w.B * w.Hq * w.N * 4
    scales = (w.Hq + 2 * w.Hkv) * 4 if w.dtype == "fp8" else 0
    return q + kv + o + lse + scales


def bwd_flops(w: Workload) -> float:
    """Backward FLOPs: five products of 2*d FLOPs per attended pair (S, dP,
    dV, dK, dQ), 2.5 x the forward's; the recomputation of S and dP in a
    second kernel is not counted."""
    return 2.5 * flops(w)


def bwd_bytes(w: Workload) -> int:
    """Algorithmic bytes of a backward step: Q, K, V, O, dO (bf16) and LSE
    read once; dQ, dK, dV written once."""
    q = w.B * w.N * w.Hq * w.d * 2
    kv = w.B * w.N * w.Hkv * w.d * 2
    lse = w.B * w.Hq * w.N * 4
    return 3 * q + 2 * kv + lse + q + 2 * kv


def decode_pairs(Nq: int, Nk: int, causal: bool, window: int) -> int:
    """Attended (query, key) pairs of one (b, h) in a decode step: query i
    sits at position Nk - Nq + i."""
    total = 0
    for i in range(Nq):
        pos = Nk - Nq + i
        hi = pos + 1 if causal else Nk
        lo = max(0, pos - window + 1) if window > 0 else 0
        total += max(0, hi - lo)
    return total


def decode_flops(w) -> float:
    """4 * d FLOPs per attended pair, over B * Hq."""
    return 4.0 * w.d * w.B * w.Hq * decode_pairs(w.Nq, w.Nk, w.causal, w.window)


def decode_bytes(w) -> int:
    """Algorithmic bytes of a decode step: Q read once, the K and V rows some
    query can see read once (with a window, only the last window + Nq - 1),
    O and LSE written once (bf16, LSE fp32)."""
    key_lo = max(0, w.Nk - w.Nq - w.window + 1) if w.window > 0 else 0
    q = w.B * w.Nq * w.Hq * w.d * 2
    kv = 2 * w.B * (w.Nk - key_lo) * w.Hkv * w.d * 2
    return q + kv + q + w.B * w.Hq * w.Nq * 4
