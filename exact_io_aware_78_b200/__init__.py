"""Exact IO-aware attention for NVIDIA B200 (sm_100a): forward, decode, backward.

The compute path is the C-ABI library libexactattn.so (hand-written CUDA:
tcgen05 tensor cores, TMA and tensor memory for the prefill forward; a
split-KV tcgen05 kernel for decode steps; per-row key-range masks as a
variant of the prefill kernel; the backward pass as two tcgen05 kernels);
this package holds its ctypes binding, the seeded input generators and the
throughput accounting.
The library is loaded lazily on the first call, and calls raise if it is
missing: there is no CPU fallback.
"""
from ._binding import (AttnError, attn_bwd, attn_bwd_masked, attn_fwd, attn_fwd_decode, attn_fwd_masked,
                       attn_get_last_error, attn_set_option, attn_shutdown, attn_status_string, attn_version, backward,
                       forward, forward_decode, load_library)

__all__ = ["AttnError", "attn_bwd", "attn_bwd_masked", "attn_fwd", "attn_fwd_decode", "attn_fwd_masked", "attn_get_last_error",
           "attn_set_option", "attn_shutdown", "attn_status_string", "attn_version", "backward", "forward",
           "forward_decode", "load_library"]
