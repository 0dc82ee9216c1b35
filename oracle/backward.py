"""Float64 CPU oracle for the exact attention backward pass.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module; only the tests, the package's smoke check and the
benchmark's CPU-baseline leg do.  It shares no code with the CUDA path.

What it computes: for the forward O = softmax(S) V with S = scale * Q K^T
plus the mask (attention.py) and an upstream gradient dO = dL/dO of some
scalar loss L, the gradients dQ, dK, dV.  They follow from the forward's
definition by the chain rule; per (b, h), with g = Hq / Hkv query heads
sharing key/value head h // g:

    P      = exp(S - LSE)          (0 where masked; LSE the forward's row LSE)
    dV    += P^T dO                (summed over the g query heads of the group)
    dP     = dO V^T
    D_i    = sum_j P_ij dP_ij  =  sum_c dO_ic O_ic
    dS     = P * (dP - D)          (elementwise; the softmax Jacobian)
    dQ     = scale * dS K
    dK    += scale * dS^T Q

Sources: the forward it differentiates (see attention.py); the backward
recomputes S and P from Q, K and the saved per-row LSE instead of storing
the N x N probabilities, trading FLOPs for memory traffic ("Flash
Attention" concept note (heepie.pages.dev), "Tiling" section -- FLOPs grow
through recomputation yet the run is faster -- and "FLOP != speed").  The
pages print no backward formulas; the lines above are the calculus of the
forward definition, written out.

Readings (listed in the design notes): the loss is any L with dL/dO = dO;
masked pairs contribute nothing; a row with no visible key has P = 0 and so
contributes nothing to any gradient; LSE, when supplied, is the forward's
natural-log LSE (else it is computed here).

Parity pins (tests/test_oracle_backward_pins.py): central finite differences
of the forward oracle; torch float64 autograd through an explicit-mask
softmax; D computed both ways; rows of dS sum to zero, so dK sums to zero over
the keys of a (b, kv head) and dV sums to the sum of dO over rows that see a
key; keys that no query sees get zero gradients; GQA equals repeated heads
with the group's key/value gradients summed.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np

from .attention import _check_ranges, _check_shapes, allowed_mask, attention_ref, kv_head_of

__all__ = ["attention_bwd_ref"]


def attention_bwd_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, do: np.ndarray, causal: bool = False,
                      window: int = 0, scale: Optional[float] = None, key_lo: Optional[np.ndarray] = None,
                      key_hi: Optional[np.ndarray] = None, o: Optional[np.ndarray] = None,
                      lse: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """dQ [B, N, Hq, d], dK [B, N, Hkv, d], dV [B, N, Hkv, dv] in float64.

    q [B, N, Hq, d], k [B, N, Hkv, d], v [B, N, Hkv, dv], do [B, N, Hq, dv];
    o [B, N, Hq, dv] and lse [B, Hq, N] are the forward's outputs (computed
    here by the forward oracle when not given)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, N, Hq, Hkv, d = _check_shapes(q, k, v)
    key_lo, key_hi = _check_ranges(key_lo, key_hi, B, N)
    if do.shape != (B, N, Hq, v.shape[3]):
        raise ValueError("do must be [B, N, Hq, dv]")
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    if o is None or lse is None:
        o, lse = attention_ref(q, k, v, causal, window, scale, key_lo=key_lo, key_hi=key_hi)
    o = np.asarray(o, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    rows = np.arange(N)
    for b in range(B):
        ok = allowed_mask(rows, N, causal, window,
                          None if key_lo is None else key_lo[b], None if key_hi is None else key_hi[b])
        for h in range(Hq):
            kh = kv_head_of(h, Hq, Hkv)
            qb, kb, vb, dob = q[b, :, h], k[b, :, kh], v[b, :, kh], do[b, :, h]
            s = scale * (qb @ kb.T)                                   # recompute S
            fin = np.isfinite(lse[b, h])
            ref = np.where(fin, lse[b, h], 0.0)[:, None]
            p = np.where(ok & fin[:, None], np.exp(s - ref), 0.0)     # recompute P from LSE
            dv[b, :, kh] += p.T @ dob                                 # dV = P^T dO
            dp = dob @ vb.T                                           # dP = dO V^T
            D = (dob * o[b, :, h]).sum(axis=1, keepdims=True)         # D = rowsum(dO o O)
            ds = p * (dp - D)                                         # dS = P o (dP - D)
            dq[b, :, h] = scale * (ds @ kb)                           # dQ = scale dS K
            dk[b, :, kh] += scale * (ds.T @ qb)                       # dK = scale dS^T Q
    return dq, dk, dv
