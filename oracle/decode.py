"""Float64 CPU oracle for the decode / split-KV attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module; only the tests and the benchmark's CPU-baseline leg do.
It shares no code with the CUDA path.

The quantity is the same exact attention as in `attention.py`, for Nq query
rows against Nk >= Nq keys (a decode step: new queries against the whole
key/value cache):

    S[i, j]   = scale * sum_t Q[b, i, h, t] * K[b, j, h // g, t]
    pos(i)    = Nk - Nq + i                      (query i's position)
    allowed   = (not causal or j <= pos(i)) and (window <= 0 or j > pos(i) - window)
    O, LSE    as in `attention.py`, over the allowed keys

Sources: the quantity is the pages' softmax(Q K^T) V with a mask (Hacker News
discussion, item 40939398; "Flash Attention" concept note, AS-IS diagram);
splitting the keys and combining the parts follows the method's own
blockwise combination of partial results with their normalisation factors
("Flash Attention" note, TO-BE diagram and "Tiling" section; FlashAttention
quiz, question 4), applied across parallel workers as in the decoding work the
pages list by title only (FlashDecoding++, PagedAttention).

Readings where the pages are silent (each listed in the design notes):
  * Query rows sit at the END of the key sequence (bottom-right alignment):
    query i is the token at position Nk - Nq + i, so with causal masking it
    sees keys 0 .. Nk - Nq + i.  With Nq == Nk this is self-attention.
  * The window and GQA readings are those of `attention.py`.
"""
from __future__ import annotations

from typing import Optional, Sequence, Tuple

import numpy as np

from .attention import _row_block, kv_head_of


def attention_kv_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, causal: bool = False,
                     window: int = 0, scale: Optional[float] = None,
                     rows: Optional[Sequence[int]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Exact attention of q [B, Nq, Hq, d] against k [B, Nk, Hkv, d],
    v [B, Nk, Hkv, dv] (Nq <= Nk when a mask uses the query positions), in
    float64.  Returns O [B, R, Hq, dv] and
    LSE [B, Hq, R], R = Nq or len(rows)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [B, N, H, d]")
    B, Nq, Hq, d = q.shape
    Nk, Hkv = k.shape[1], k.shape[2]
    if k.shape[0] != B or v.shape[:3] != k.shape[:3] or k.shape[3] != d:
        raise ValueError("k, v must be [B, Nk, Hkv, d] with q's B and d")
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    if Nq > Nk and (causal or window > 0):
        raise ValueError("query positions need Nq <= Nk")  # without a mask they do not matter
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    sel = np.arange(Nq) if rows is None else np.asarray(rows, dtype=np.int64)
    pos = sel + (Nk - Nq)  # positions in the key sequence
    dv = v.shape[3]
    out = np.zeros((B, sel.shape[0], Hq, dv))
    lse = np.zeros((B, Hq, sel.shape[0]))
    for b in range(B):
        for h in range(Hq):
            kh = kv_head_of(h, Hq, Hkv)
            o, l, _ = _row_block(q[b, sel, h, :], k[b, :, kh, :], v[b, :, kh, :], pos, causal, window, scale)
            out[b, :, h, :] = o
            lse[b, h, :] = l
    return out, lse


def merge_partials_ref(o_parts: np.ndarray, lse_parts: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Combine results over disjoint key sets into the result over their
    union.  o_parts [P, ...rows, dv] are each part's normalised outputs,
    lse_parts [P, ...rows] their log-sum-exps (-inf for a part with no
    allowed key).  With L = ln sum_p exp(LSE_p):
        O = sum_p exp(LSE_p - L) O_p,   LSE = L."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    m_safe = np.where(np.isfinite(m), m, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - m_safe), 0.0)  # [P, ...rows]
    tot = w.sum(axis=0)
    lse = np.where(tot > 0, m_safe + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    wn = np.divide(w, tot, out=np.zeros_like(w), where=tot > 0)
    o = (wn[..., None] * o_parts).sum(axis=0)
    return o, lse
