"""ctypes view of the C ABI declared in include/sage.h (argument marshalling only)."""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
# SAGE_LIB_PATH may name another build of the same library (e.g. one built with
# different compile options); the default is the in-tree build.
LIB_PATH = os.environ.get("SAGE_LIB_PATH") or os.path.join(_PKG, "libsage.so")

SAGE_OK = 0
SAGE_ERR_INVALID_ARGUMENT = 1
SAGE_ERR_UNSUPPORTED = 2
SAGE_ERR_CUDA = 3
SAGE_ERR_DEVICE_TIMEOUT = 4
SAGE_ERR_TOO_LARGE = 5
NOALLOC_SCRATCH_BYTES = 8 << 20  # SAGE_NOALLOC_SCRATCH_BYTES

SAGE_FP16, SAGE_BF16, SAGE_FP32 = 0, 1, 2
SAGE_GRAN_BLOCK, SAGE_GRAN_THREAD = 0, 1
SAGE_PV_FP8, SAGE_PV_FP16 = 0, 1

EXPORTS = (
    "sage_buffer_sizes", "sage_quant_qk", "sage_quant_v", "sage_attn_fwd",
    "sage_debug_qk_int32", "sage_poll_device_status", "sage_quant_qk_noalloc",
    "sage_attn_host", "sage_host_workspace_bytes", "sage_debug_watchdog_selftest",
    "sage_quant_qkv",
    "sage_status_string",
)


class SageProblem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int),
        ("heads_q", ctypes.c_int),
        ("heads_kv", ctypes.c_int),
        ("seqlen", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("cu_seqlens_host", ctypes.POINTER(ctypes.c_int32)),
        ("granularity", ctypes.c_int),  # SAGE_GRAN_BLOCK / SAGE_GRAN_THREAD
        ("pv", ctypes.c_int),           # SAGE_PV_FP8 / SAGE_PV_FP16
    ]


class SageSizes(ctypes.Structure):
    _fields_ = [(name, ctypes.c_size_t) for name in (
        "q8", "q_scale", "k8", "k_scale", "k_mean", "v8", "v_scale",
        "workspace_qk", "workspace_v", "t_pad", "workspace_qkv")]


class SageError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsage.so (built in-tree); raise loudly if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"CUDA library {LIB_PATH} is missing; build it with "
            "`python -m quantized_attention_06_b200.build` (there is no CPU fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER
    vp, sz, i64p = ctypes.c_void_p, ctypes.c_size_t, P(ctypes.c_int64)
    L.sage_buffer_sizes.argtypes = [P(SageProblem), P(SageSizes)]
    L.sage_quant_qk.argtypes = [P(SageProblem), vp, i64p, vp, i64p, vp, vp, vp, vp, vp, vp, sz, vp]
    L.sage_quant_v.argtypes = [P(SageProblem), vp, i64p, vp, vp, vp, sz, vp]
    L.sage_quant_qkv.argtypes = [P(SageProblem), vp, i64p, vp, i64p, vp, i64p, vp, vp, vp, vp, vp,
                                 vp, vp, vp, sz, vp]
    L.sage_quant_qk_noalloc.argtypes = [P(SageProblem), vp, i64p, vp, i64p, vp, vp, vp, vp, vp, vp]
    L.sage_attn_fwd.argtypes = [P(SageProblem), vp, vp, vp, vp, vp, vp, ctypes.c_float,
                                ctypes.c_int, vp, ctypes.c_int, i64p, vp, vp]
    L.sage_debug_qk_int32.argtypes = [P(SageProblem), vp, vp, ctypes.c_int, ctypes.c_int, vp, vp]
    L.sage_poll_device_status.argtypes = [vp]
    L.sage_debug_watchdog_selftest.argtypes = [ctypes.c_uint, vp]
    L.sage_attn_host.argtypes = [P(SageProblem), ctypes.c_int, vp, vp, vp, vp, ctypes.c_int,
                                 ctypes.c_float, ctypes.c_int, ctypes.c_int, vp, sz, vp]
    L.sage_host_workspace_bytes.argtypes = [P(SageProblem), ctypes.c_int, ctypes.c_int]
    L.sage_status_string.argtypes = [ctypes.c_int]
    L.sage_status_string.restype = ctypes.c_char_p
    for name in EXPORTS[:-1]:
        getattr(L, name).restype = ctypes.c_int
    L.sage_host_workspace_bytes.restype = ctypes.c_size_t
    _lib = L
    return L


def check(fn: str, status: int) -> None:
    if status != SAGE_OK:
        raise SageError(fn, status, lib().sage_status_string(status).decode())


def strides3(values) -> ctypes.Array:
    return (ctypes.c_int64 * 3)(*[int(v) for v in values])
