"""SageAttention-style quantized attention forward for B200 (sm_100a).

INT8 QK^T on tcgen05 tensor cores with K smoothing, FP8 e4m3 PV with two-level
accumulation, exposed through the C ABI in include/sage.h and the thin binding
in ``api``.  Importing this package does not load the CUDA library; the first
call does, and raises if it is missing.
"""

from .api import (Problem, Quantized, attn_fwd, debug_qk_int32, poll_device_status, quant_qk,
                  quant_v, sageattn)

__all__ = ["Problem", "Quantized", "attn_fwd", "debug_qk_int32", "poll_device_status",
           "quant_qk", "quant_v", "sageattn"]
