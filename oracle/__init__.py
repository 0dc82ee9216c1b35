"""Float64 CPU oracle for exact attention, forward and backward (test
infrastructure only).

Only tests/, the package smoke check and the benchmark's CPU-baseline leg may
import this package.  It shares no code with the CUDA path.
"""
from .attention import (allowed_mask, attention_ref, decode_e4m3, dequantize_per_head,
                        online_ref, probabilities_ref)
from .backward import attention_bwd_ref
from .decode import attention_kv_ref, merge_partials_ref

__all__ = ["allowed_mask", "attention_bwd_ref", "attention_kv_ref", "attention_ref", "decode_e4m3", "dequantize_per_head",
           "merge_partials_ref", "online_ref", "probabilities_ref"]
