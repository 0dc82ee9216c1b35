"""Seeded synthetic inputs for the attention forward workloads.

This module is shared by the CUDA path's callers (tests, bench) and by the
float64 oracle's tests.  It holds no attention arithmetic: it draws i.i.d.
normal tensors from a seeded CPU generator and stores them in the element
format a workload asks for (fp32, bf16, or e4m3 codes plus per-head fp32
scales).  Everything is generated on the CPU so that every consumer sees
bit-identical values.

Layout: Q is [B, N, Hq, d], K and V are [B, N, Hkv, d], all d-contiguous.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

E4M3_MAX = 448.0  # largest finite e4m3 (OCP FP8, "fn" variant) magnitude


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention-forward problem: shapes, mask, element format and seed."""

    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    d: int
    causal: bool
    window: int  # <= 0: no sliding window
    dtype: str  # "fp32" | "bf16" | "fp8"
    seed: int
    q_mult: float = 1.0  # Q drawn as q_mult * N(0, 1) before the format cast
    description: str = ""
    mask: str = ""       # per-row key ranges: "" (none), "documents" or "prefix" (make_row_ranges)
    mask_min: int = 0    # shortest document / prefix
    mask_max: int = 0    # longest document / prefix

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv


WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("fp32_n128_d64", 1, 1, 1, 128, 64, False, 0, "fp32", 1234,
                 description="non-causal, fp32 inputs, tiny"),
        Workload("bf16_causal_b4h16_n2048_d128", 4, 16, 16, 2048, 128, True, 0, "bf16", 2048,
                 description="causal self-attention"),
        Workload("bf16_gqa_causal_b2h32kv8_n4096_d128_q3", 2, 32, 8, 4096, 128, True, 0, "bf16", 4096,
                 q_mult=3.0, description="grouped-query causal, Q sharpened x3"),
        Workload("bf16_causal_window4096_b1h16_n16384_d128", 1, 16, 16, 16384, 128, True, 4096, "bf16",
                 16384, description="long context, causal + sliding window 4096"),
        Workload("fp8_causal_b2h16_n8192_d128", 2, 16, 16, 8192, 128, True, 0, "fp8", 8192,
                 description="e4m3 inputs with per-head fp32 scales"),
        Workload("bf16_doccausal_b2h16_n16384_d128", 2, 16, 16, 16384, 128, True, 0, "bf16", 1638,
                 description="packed documents of 512-4096 tokens, causal inside each document "
                             "(per-row key ranges)", mask="documents", mask_min=512, mask_max=4096),
    ]
}

# The five forward configurations of the throughput-vs-sequence-length curve,
# shortest sequence first: fp32 N=128 d=64; bf16 causal N=2048; bf16 GQA
# causal N=4096 (Q x 3); bf16 causal + window 4096 at N=16384; e4m3 causal
# N=8192.
CURVE_WORKLOADS = ("fp32_n128_d64", "bf16_causal_b4h16_n2048_d128", "bf16_gqa_causal_b2h32kv8_n4096_d128_q3",
                   "bf16_causal_window4096_b1h16_n16384_d128", "fp8_causal_b2h16_n8192_d128")

# The workload the benchmark times by default: the largest one-GPU
# configuration (causal + sliding window 4096, B=1, H=16, N=16384, d=128).
DEFAULT_BENCH_WORKLOAD = "bf16_causal_window4096_b1h16_n16384_d128"

# Backward-pass workloads: the forward's inputs plus dO = make_grad_output(seed + 3).
BWD_WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("bwd_bf16_causal_b4h16_n2048_d128", 4, 16, 16, 2048, 128, True, 0, "bf16", 2048,
                 description="backward of causal self-attention"),
        Workload("bwd_bf16_gqa_causal_b2h32kv8_n4096_d128", 2, 32, 8, 4096, 128, True, 0, "bf16", 4096,
                 description="backward of grouped-query causal attention"),
        Workload("bwd_bf16_doccausal_b2h16_n16384_d128", 2, 16, 16, 16384, 128, True, 0, "bf16", 1638,
                 description="backward of the packed-document mask (per-row key ranges)", mask="documents",
                 mask_min=512, mask_max=4096),
    ]
}


def _randn(seed: int, shape, mult: float = 1.0) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if mult != 1.0:
        x = x * mult
    return x


def quantize_e4m3_per_head(x: torch.Tensor):
    """Per-head scale s_h = amax over (B, N, d) of |x[..., h, :]| / 448, codes =
    round-to-nearest-even saturating cast of x / s_h to e4m3.  Returns
    (codes as torch.float8_e4m3fn [same shape], scales fp32 [H])."""
    amax = x.abs().amax(dim=(0, 1, 3)).to(torch.float32)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (x / scale.view(1, 1, -1, 1)).clamp(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return codes, scale


def make_inputs(B: int, Hq: int, Hkv: int, N: int, d: int, dtype: str, seed: int,
                q_mult: float = 1.0) -> Dict[str, Optional[torch.Tensor]]:
    """Draw Q, K, V (seeds seed, seed+1, seed+2) as fp32 N(0,1) on the CPU,
    multiply Q by q_mult, then store them in `dtype`.

    Returns a dict with CPU tensors q, k, v (dtype torch.float32,
    torch.bfloat16 or torch.float8_e4m3fn) and q_scale, k_scale, v_scale
    (fp32 per-head scales for fp8, else None)."""
    q = _randn(seed + 0, (B, N, Hq, d), q_mult)
    k = _randn(seed + 1, (B, N, Hkv, d))
    v = _randn(seed + 2, (B, N, Hkv, d))
    out: Dict[str, Optional[torch.Tensor]] = {"q_scale": None, "k_scale": None, "v_scale": None}
    if dtype == "fp32":
        out.update(q=q, k=k, v=v)
    elif dtype == "bf16":
        out.update(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16))
    elif dtype == "fp8":
        for name, x in (("q", q), ("k", k), ("v", v)):
            codes, s = quantize_e4m3_per_head(x)
            out[name] = codes
            out[name + "_scale"] = s
    else:
        raise ValueError(f"unknown dtype {dtype!r}")
    return out


def make_ramp_inputs(B: int, H: int, N: int, d: int, dtype: str, seed: int,
                     ramp: float) -> Dict[str, Optional[torch.Tensor]]:
    """Inputs whose scores grow along the keys: Q = N(0, 1) + 1 and
    K[j] = N(0, 1) / 2 + ramp * j / N in every dimension, V = N(0, 1) (one
    generator seeded with `seed`, drawn in that order), stored bf16 or as
    e4m3 codes with per-head scales.  Each row's running maximum then climbs
    from key tile to key tile, which exercises the rescaling of the running
    sums."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn(B, N, H, d, generator=g) + 1.0
    k = torch.randn(B, N, H, d, generator=g) * 0.5 + (ramp * torch.arange(N) / N).view(1, N, 1, 1)
    v = torch.randn(B, N, H, d, generator=g)
    out: Dict[str, Optional[torch.Tensor]] = {"q_scale": None, "k_scale": None, "v_scale": None}
    if dtype == "bf16":
        out.update(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16))
    elif dtype == "fp8":
        for name, x in (("q", q), ("k", k), ("v", v)):
            out[name], out[name + "_scale"] = quantize_e4m3_per_head(x)
    else:
        raise ValueError(f"unknown dtype {dtype!r}")
    return out


def workload_inputs(w: Workload) -> Dict[str, Optional[torch.Tensor]]:
    out = make_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.dtype, w.seed, w.q_mult)
    out["key_lo"] = out["key_hi"] = None
    if w.mask:
        out["key_lo"], out["key_hi"] = make_row_ranges(w.mask, w.B, w.N, w.seed + 3, w.mask_min, w.mask_max)
    return out


def make_grad_output(B: int, N: int, Hq: int, d: int, seed: int) -> torch.Tensor:
    """dO = dL/dO for backward runs: N(0, 1) drawn on the CPU, stored bf16
    [B, N, Hq, d]."""
    return _randn(seed, (B, N, Hq, d)).to(torch.bfloat16)


def make_row_ranges(kind: str, B: int, N: int, seed: int, min_len: int = 1, max_len: int = 0):
    """Seeded per-row key ranges: int32 CPU tensors key_lo, key_hi of shape
    [B, N] (query row i of batch b may see keys key_lo <= j < key_hi).

      "documents"  the N rows are packed documents whose lengths are drawn
                   uniformly from [min_len, max_len] (the last one cut at N);
                   a row sees the keys of its own document.  With causal
                   masking on top this is the packed-sequence training mask.
      "prefix"     per batch a prefix length P drawn from [min_len, max_len]:
                   rows i < P see keys [0, P), later rows keys [0, i]
                   (a prefix-LM mask; use without causal masking).
      "random"     lo drawn from [-2, N], hi = lo + a draw from [-2, N // 2]:
                   empty rows, ranges past either end and single keys, for
                   edge-case tests."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    lo = torch.zeros(B, N, dtype=torch.int32)
    hi = torch.zeros(B, N, dtype=torch.int32)
    max_len = max(max_len, min_len)
    for b in range(B):
        if kind == "documents":
            start = 0
            while start < N:
                n = int(torch.randint(min_len, max_len + 1, (1,), generator=g))
                end = min(N, start + n)
                lo[b, start:end] = start
                hi[b, start:end] = end
                start = end
        elif kind == "prefix":
            P = min(N, int(torch.randint(min_len, max_len + 1, (1,), generator=g)))
            i = torch.arange(N, dtype=torch.int32)
            hi[b] = torch.where(i < P, torch.full_like(i, P), i + 1)
        elif kind == "random":
            lo[b] = torch.randint(-2, N + 1, (N,), generator=g, dtype=torch.int32)
            hi[b] = lo[b] + torch.randint(-2, N // 2 + 1, (N,), generator=g, dtype=torch.int32)
        else:
            raise ValueError(f"unknown row-range kind {kind!r}")
    return lo, hi


def sample_rows(N: int, window: int, count: int, seed: int):
    """A seeded, sorted set of query rows for sampled checks at full size:
    `count` random rows plus the first, the last, the tile edges around
    128-row boundaries near the ends, and (with a window) the rows where the
    window starts to bind."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    rows = set(torch.randint(0, N, (count,), generator=g).tolist())
    rows.update({0, 1, N - 1, max(0, N - 2)})
    for r in (127, 128, 129, 255, 256, N - 129, N - 128, N - 127):
        if 0 <= r < N:
            rows.add(r)
    if window > 0:
        for r in (window - 2, window - 1, window, window + 1):
            if 0 <= r < N:
                rows.add(r)
    return sorted(rows)


def head_shard(w: Workload, world: int, rank: int):
    """Head-sharded multi-GPU layout: rank `rank` of `world` owns the
    contiguous block of KV heads [kv_lo, kv_hi) and their query heads
    [kv_lo * g, kv_hi * g) (g = Hq / Hkv), as a tensor-parallel model holds
    its own heads.  (b, h) problems are independent, so no data moves
    between ranks.  Returns (sub-workload, q_lo, q_hi, kv_lo, kv_hi)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    if w.Hkv % world != 0:
        raise ValueError(f"Hkv={w.Hkv} is not divisible by {world} ranks")
    per = w.Hkv // world
    kv_lo, kv_hi = rank * per, (rank + 1) * per
    q_lo, q_hi = kv_lo * w.group, kv_hi * w.group
    sub = dataclasses.replace(w, name=f"{w.name}_heads{rank}of{world}", Hq=q_hi - q_lo, Hkv=per)
    return sub, q_lo, q_hi, kv_lo, kv_hi


def shard_inputs(inp: Dict[str, Optional[torch.Tensor]], q_lo: int, q_hi: int, kv_lo: int, kv_hi: int):
    """This rank's contiguous slices of a workload's inputs (and per-head
    scales) along the head dimension."""
    out: Dict[str, Optional[torch.Tensor]] = {}
    for name, (lo, hi) in (("q", (q_lo, q_hi)), ("k", (kv_lo, kv_hi)), ("v", (kv_lo, kv_hi))):
        out[name] = inp[name][:, :, lo:hi, :].contiguous()
        s = inp[name + "_scale"]
        out[name + "_scale"] = None if s is None else s[lo:hi].contiguous()
    # per-row key ranges are shared by all heads: every shard keeps them whole
    out["key_lo"], out["key_hi"] = inp.get("key_lo"), inp.get("key_hi")
    return out


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """A decode step: Nq new query rows (the last tokens of the sequence)
    against a key/value cache of Nk rows; bf16 inputs."""

    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    Nk: int
    d: int
    causal: bool
    window: int
    seed: int
    description: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv


DECODE_WORKLOADS: Dict[str, DecodeWorkload] = {
    w.name: w
    for w in [
        DecodeWorkload("decode_b8h32kv8_nq1_nk16384_d128", 8, 32, 8, 1, 16384, 128, True, 0, 1601,
                       description="one new token per sequence, GQA 4:1, 16384-token cache"),
        DecodeWorkload("decode_b4h32kv8_nq2_nk8192_d128_window2048", 4, 32, 8, 2, 8192, 128, True, 2048, 1602,
                       description="two new tokens, causal within the step, sliding window 2048"),
    ]
}


def make_decode_inputs(B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int,
                       seed: int) -> Dict[str, Optional[torch.Tensor]]:
    """Q [B, Nq, Hq, d], K, V [B, Nk, Hkv, d]: seeded N(0, 1) on the CPU
    (seeds seed, seed+1, seed+2), stored as bf16 (no per-head scales)."""
    return {"q": _randn(seed + 0, (B, Nq, Hq, d)).to(torch.bfloat16),
            "k": _randn(seed + 1, (B, Nk, Hkv, d)).to(torch.bfloat16),
            "v": _randn(seed + 2, (B, Nk, Hkv, d)).to(torch.bfloat16),
            "q_scale": None, "k_scale": None, "v_scale": None}


def decode_workload_inputs(w: DecodeWorkload) -> Dict[str, Optional[torch.Tensor]]:
    return make_decode_inputs(w.B, w.Hq, w.Hkv, w.Nq, w.Nk, w.d, w.seed)
