"""Python binding of the C ABI in include/sage.h.

PyTorch supplies device memory and the current CUDA stream; every step of the
computation runs in the CUDA kernels of libsage.so.  There is no CPU fallback:
the calls raise when the library or a GPU is missing.

Usage mirrors the tutorial page "SageAttention终极指南" (基础使用示例):

    out = sageattn(q, k, v, tensor_layout="HND", is_causal=False)

with q, k, v of shape (batch, heads, seq_len, head_dim) for "HND",
(batch, seq_len, heads, head_dim) for "NHD", or packed (tokens, heads, head_dim)
together with ``cu_seqlens`` for variable-length batches.
"""

from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib as L

__all__ = ["Problem", "Quantized", "quant_qk", "quant_qk_noalloc", "quant_v", "quant_qkv", "attn_fwd",
           "sageattn", "sageattn_host", "debug_qk_int32", "debug_watchdog_selftest",
           "poll_device_status"]

_IN_DTYPES = {torch.float16: L.SAGE_FP16, torch.bfloat16: L.SAGE_BF16}
# INT8 scale granularity of Q and K: "block" (128-token Q / 64-token K blocks, the
# method as stated) or "thread" (a scale per Q token and per 32-token K block)
_GRANULARITY = {"block": L.SAGE_GRAN_BLOCK, "thread": L.SAGE_GRAN_THREAD}
_OUT_DTYPES = {torch.float16: L.SAGE_FP16, torch.bfloat16: L.SAGE_BF16, torch.float32: L.SAGE_FP32}
# format of the P V product: "fp8" (e4m3 P and V, the method as stated) or "fp16" (P and V
# in the input's 16-bit type, the accuracy fallback)
_PV = {"fp8": L.SAGE_PV_FP8, "fp16": L.SAGE_PV_FP16}


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


class Problem:
    """Shapes of one attention call (sage_problem_t)."""

    def __init__(self, batch, heads_q, heads_kv, seqlen, head_dim, dtype, cu_seqlens=None,
                 granularity="block", pv="fp8"):
        if dtype not in _IN_DTYPES:
            raise TypeError(f"q/k/v must be float16 or bfloat16, got {dtype}")
        if granularity not in _GRANULARITY:
            raise ValueError(f"granularity must be 'block' or 'thread', got {granularity!r}")
        if pv not in _PV:
            raise ValueError(f"pv must be 'fp8' or 'fp16', got {pv!r}")
        self.granularity = granularity
        self.pv = pv
        self.dtype = dtype
        self.varlen = cu_seqlens is not None
        if self.varlen:
            cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
            self.cu_list = cu
            self._cu = (ctypes.c_int32 * len(cu))(*cu)
            cu_ptr = ctypes.cast(self._cu, ctypes.POINTER(ctypes.c_int32))
            batch = len(cu) - 1
            seqlen = max(b - a for a, b in zip(cu[:-1], cu[1:]))
        else:
            self.cu_list = None
            cu_ptr = ctypes.POINTER(ctypes.c_int32)()
        self.c = L.SageProblem(batch, heads_q, heads_kv, seqlen, head_dim, _IN_DTYPES[dtype], cu_ptr,
                               _GRANULARITY[granularity], _PV[pv])
        self.batch, self.heads_q, self.heads_kv = batch, heads_q, heads_kv
        self.seqlen, self.head_dim = seqlen, head_dim
        sz = L.SageSizes()
        L.check("sage_buffer_sizes", L.lib().sage_buffer_sizes(ctypes.byref(self.c), ctypes.byref(sz)))
        self.sizes = sz
        self.t_pad = int(sz.t_pad)

    @property
    def q_block(self) -> int:
        return 1 if self.granularity == "thread" else 128

    @property
    def k_block(self) -> int:
        return 32 if self.granularity == "thread" else 64

    @staticmethod
    def from_tensors(q, k, tensor_layout="HND", cu_seqlens=None, granularity="block",
                     pv="fp8") -> "Problem":
        if cu_seqlens is not None:
            _, hq, d = q.shape
            hkv = k.shape[1]
            return Problem(0, hq, hkv, 0, d, q.dtype, cu_seqlens, granularity, pv)
        if tensor_layout == "HND":
            b, hq, n, d = q.shape
            hkv = k.shape[1]
        elif tensor_layout == "NHD":
            b, n, hq, d = q.shape
            hkv = k.shape[2]
        else:
            raise ValueError(f"tensor_layout must be 'HND' or 'NHD', got {tensor_layout!r}")
        return Problem(b, hq, hkv, n, d, q.dtype, granularity=granularity, pv=pv)


def _strides(t: torch.Tensor, tensor_layout: str, varlen: bool):
    if t.stride(-1) != 1:
        raise ValueError("the head_dim dimension must be contiguous")
    s = t.stride()
    if varlen:
        return L.strides3((0, s[1], s[0]))
    if tensor_layout == "HND":
        return L.strides3((s[0], s[1], s[2]))
    return L.strides3((s[0], s[2], s[1]))


@dataclass
class Quantized:
    """Quantized operands in the padded token space (layouts in include/sage.h)."""
    problem: Problem
    tensor_layout: str
    q8: torch.Tensor = None
    q_scale: torch.Tensor = None
    k8: torch.Tensor = None
    k_scale: torch.Tensor = None
    k_mean: torch.Tensor = None
    v8: torch.Tensor = None
    v_scale: torch.Tensor = None


def _alloc(nbytes: int, dtype, device) -> torch.Tensor:
    esz = torch.empty((), dtype=dtype).element_size()
    return torch.empty(max(1, nbytes // esz), dtype=dtype, device=device)


def _require_cuda(*ts):
    for t in ts:
        if not (isinstance(t, torch.Tensor) and t.is_cuda):
            raise RuntimeError("sage kernels need CUDA tensors on a B200; there is no CPU fallback")
    dev = ts[0].device
    if any(t.device != dev for t in ts):
        raise ValueError("all tensors of one call must be on the same CUDA device")
    return dev


def quant_qk(q, k, tensor_layout="HND", cu_seqlens=None, problem=None, out: Quantized = None,
             workspace=None, granularity="block", pv="fp8") -> Quantized:
    """K smoothing + per-block INT8 quantization of Q and K (sage_quant_qk).
    ``pv`` fixes the PV format of the attention call that follows ("fp8" or "fp16")."""
    with torch.cuda.device(_require_cuda(q, k)):
        return _quant_qk(q, k, tensor_layout, cu_seqlens, problem, out, workspace, granularity, pv)


def _quant_qk(q, k, tensor_layout, cu_seqlens, problem, out, workspace, granularity, pv):
    p = problem or Problem.from_tensors(q, k, tensor_layout, cu_seqlens, granularity, pv)
    z = out or Quantized(p, tensor_layout)
    dev = q.device
    sz = p.sizes
    d, tp = p.head_dim, p.t_pad
    if z.q8 is None:
        z.q8 = torch.empty((p.heads_q, tp, d), dtype=torch.int8, device=dev)
        z.q_scale = torch.empty((p.heads_q, tp // p.q_block), dtype=torch.float32, device=dev)
        z.k8 = torch.empty((p.heads_kv, tp, d), dtype=torch.int8, device=dev)
        z.k_scale = torch.empty((p.heads_kv, tp // p.k_block), dtype=torch.float32, device=dev)
        z.k_mean = torch.empty((p.batch, p.heads_kv, d), dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else _alloc(sz.workspace_qk, torch.float64, dev)
    varlen = p.varlen
    st = L.lib().sage_quant_qk(
        ctypes.byref(p.c), _ptr(q), _strides(q, tensor_layout, varlen),
        _ptr(k), _strides(k, tensor_layout, varlen),
        _ptr(z.q8), _ptr(z.q_scale), _ptr(z.k8), _ptr(z.k_scale), _ptr(z.k_mean),
        _ptr(ws), ws.numel() * ws.element_size(), _stream())
    L.check("sage_quant_qk", st)
    return z


def quant_qk_noalloc(q, k, tensor_layout="HND", cu_seqlens=None, problem=None,
                     out: Quantized = None, granularity="block") -> Quantized:
    """quant_qk without a workspace (sage_quant_qk_noalloc), for callers that cannot
    allocate device memory when they quantize.  The scratch comes from a fixed
    library-owned device array; ``out`` should then hold preallocated outputs.
    Calls that overlap on the GPU race on that shared scratch."""
    with torch.cuda.device(_require_cuda(q, k)):
        return _quant_qk_noalloc(q, k, tensor_layout, cu_seqlens, problem, out, granularity)


def _quant_qk_noalloc(q, k, tensor_layout, cu_seqlens, problem, out, granularity):
    p = problem or Problem.from_tensors(q, k, tensor_layout, cu_seqlens, granularity)
    z = out or Quantized(p, tensor_layout)
    dev = q.device
    d, tp = p.head_dim, p.t_pad
    if z.q8 is None:
        z.q8 = torch.empty((p.heads_q, tp, d), dtype=torch.int8, device=dev)
        z.q_scale = torch.empty((p.heads_q, tp // p.q_block), dtype=torch.float32, device=dev)
        z.k8 = torch.empty((p.heads_kv, tp, d), dtype=torch.int8, device=dev)
        z.k_scale = torch.empty((p.heads_kv, tp // p.k_block), dtype=torch.float32, device=dev)
        z.k_mean = torch.empty((p.batch, p.heads_kv, d), dtype=torch.float32, device=dev)
    st = L.lib().sage_quant_qk_noalloc(
        ctypes.byref(p.c), _ptr(q), _strides(q, tensor_layout, p.varlen),
        _ptr(k), _strides(k, tensor_layout, p.varlen),
        _ptr(z.q8), _ptr(z.q_scale), _ptr(z.k8), _ptr(z.k_scale), _ptr(z.k_mean), _stream())
    L.check("sage_quant_qk_noalloc", st)
    return z


def quant_v(v, z: Quantized, workspace=None) -> Quantized:
    """Per-channel e4m3 quantization of V, written token-contiguous (sage_quant_v).
    With the 16-bit PV format V keeps its values, transposed the same way."""
    with torch.cuda.device(_require_cuda(v)):
        p = z.problem
        dev = v.device
        if z.v8 is None:
            vt = torch.uint8 if p.pv == "fp8" else v.dtype
            z.v8 = torch.empty((p.heads_kv, p.head_dim, p.t_pad), dtype=vt, device=dev)
            z.v_scale = torch.empty((p.batch, p.heads_kv, p.head_dim), dtype=torch.float32, device=dev)
        need = int(p.sizes.workspace_v)
        ws = workspace if workspace is not None else (_alloc(need, torch.float32, dev) if need else None)
        nbytes = 0 if ws is None else ws.numel() * ws.element_size()
        st = L.lib().sage_quant_v(ctypes.byref(p.c), _ptr(v), _strides(v, z.tensor_layout, p.varlen),
                                  _ptr(z.v8), _ptr(z.v_scale), _ptr(ws), nbytes, _stream())
        L.check("sage_quant_v", st)
        return z


def quant_qkv(q, k, v, tensor_layout="HND", cu_seqlens=None, problem=None, out: Quantized = None,
              workspace=None, granularity="block", pv="fp8") -> Quantized:
    """quant_qk and quant_v in one cooperative launch (sage_quant_qkv); the buffers are
    bit-identical to the two separate calls."""
    with torch.cuda.device(_require_cuda(q, k, v)):
        p = problem or Problem.from_tensors(q, k, tensor_layout, cu_seqlens, granularity, pv)
        z = out or Quantized(p, tensor_layout)
        dev = q.device
        d, tp = p.head_dim, p.t_pad
        if z.q8 is None:
            z.q8 = torch.empty((p.heads_q, tp, d), dtype=torch.int8, device=dev)
            z.q_scale = torch.empty((p.heads_q, tp // p.q_block), dtype=torch.float32, device=dev)
            z.k8 = torch.empty((p.heads_kv, tp, d), dtype=torch.int8, device=dev)
            z.k_scale = torch.empty((p.heads_kv, tp // p.k_block), dtype=torch.float32, device=dev)
            z.k_mean = torch.empty((p.batch, p.heads_kv, d), dtype=torch.float32, device=dev)
        if z.v8 is None:
            vt = torch.uint8 if p.pv == "fp8" else v.dtype
            z.v8 = torch.empty((p.heads_kv, d, tp), dtype=vt, device=dev)
            z.v_scale = torch.empty((p.batch, p.heads_kv, d), dtype=torch.float32, device=dev)
        need = int(p.sizes.workspace_qkv)
        ws = workspace if workspace is not None else _alloc(need + 256, torch.uint8, dev)
        base = (ws.data_ptr() + 255) // 256 * 256
        nbytes = ws.numel() * ws.element_size() - (base - ws.data_ptr())
        st = L.lib().sage_quant_qkv(
            ctypes.byref(p.c), _ptr(q), _strides(q, tensor_layout, p.varlen),
            _ptr(k), _strides(k, tensor_layout, p.varlen), _ptr(v), _strides(v, tensor_layout, p.varlen),
            _ptr(z.q8), _ptr(z.q_scale), _ptr(z.k8), _ptr(z.k_scale), _ptr(z.k_mean),
            _ptr(z.v8), _ptr(z.v_scale), ctypes.c_void_p(base), nbytes, _stream())
        L.check("sage_quant_qkv", st)
        return z


def _out_shape(p: Problem, layout: str):
    if p.varlen:
        return (p.cu_list[-1], p.heads_q, p.head_dim)
    if layout == "HND":
        return (p.batch, p.heads_q, p.seqlen, p.head_dim)
    return (p.batch, p.seqlen, p.heads_q, p.head_dim)


def attn_fwd(z: Quantized, is_causal=False, sm_scale=None, out_dtype=None, out=None,
             return_lse=False):
    """The attention kernel on quantized operands (sage_attn_fwd)."""
    with torch.cuda.device(_require_cuda(z.q8, z.k8, z.v8)):
        return _attn_fwd(z, is_causal, sm_scale, out_dtype, out, return_lse)


def _attn_fwd(z, is_causal, sm_scale, out_dtype, out, return_lse):
    p = z.problem
    dev = z.q8.device
    if out is None:
        odt = out_dtype or p.dtype
        if odt not in _OUT_DTYPES:
            raise TypeError(f"unsupported output dtype {odt}")
        out = torch.empty(_out_shape(p, z.tensor_layout), dtype=odt, device=dev)
    lse = torch.empty((p.heads_q, p.t_pad), dtype=torch.float32, device=dev) if return_lse else None
    st = L.lib().sage_attn_fwd(
        ctypes.byref(p.c), _ptr(z.q8), _ptr(z.q_scale), _ptr(z.k8), _ptr(z.k_scale),
        _ptr(z.v8), _ptr(z.v_scale), ctypes.c_float(0.0 if sm_scale is None else float(sm_scale)),
        1 if is_causal else 0, _ptr(out), _OUT_DTYPES[out.dtype],
        _strides(out, z.tensor_layout, p.varlen), _ptr(lse), _stream())
    L.check("sage_attn_fwd", st)
    return (out, lse) if return_lse else out


def sageattn(q, k, v, tensor_layout="HND", is_causal=False, sm_scale=None, cu_seqlens=None,
             out_dtype=None, return_lse=False, granularity="block", pv="fp8"):
    """Quantized attention: smoothing + INT8 Q/K and FP8 V in one launch (quant_qkv),
    then the fused attention kernel.
    granularity="thread" selects a Q scale per token and a K scale per 32 tokens;
    pv="fp16" runs P V in the input's 16-bit type instead of e4m3."""
    z = quant_qkv(q, k, v, tensor_layout, cu_seqlens, granularity=granularity, pv=pv)
    return attn_fwd(z, is_causal=is_causal, sm_scale=sm_scale, out_dtype=out_dtype,
                    return_lse=return_lse)


_HOST_WS = {}


def sageattn_host(q, k, v, tensor_layout="HND", is_causal=False, sm_scale=None, out=None,
                  out_dtype=None, kv_heads_per_chunk=0, device=None, synchronize=True,
                  granularity="block", pv="fp8"):
    """sageattn on host tensors (sage_attn_host): chunks of heads are copied in,
    computed and copied out with the copies overlapping the kernels.

    q, k, v: contiguous CPU tensors, (B, H, N, d) for "HND" or (B, N, H, d) for
    "NHD", pinned for overlap.  Returns the output as a CPU tensor (pinned when
    allocated here) of the same layout; with synchronize=False the call returns once
    the work is enqueued on the current stream, and `out` must not be read before
    that stream has been synchronized.
    """
    for t in (q, k, v):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("sageattn_host takes contiguous host tensors")
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if not torch.cuda.is_available():
        raise RuntimeError("sageattn_host needs a CUDA device: there is no CPU fallback")
    if tensor_layout == "HND":
        b, hq, n, d = q.shape
        hkv = k.shape[1]
        code = 0
    elif tensor_layout == "NHD":
        b, n, hq, d = q.shape
        hkv = k.shape[2]
        code = 1
    else:
        raise ValueError(f"tensor_layout must be HND or NHD, got {tensor_layout}")
    p = Problem(b, hq, hkv, n, d, q.dtype, granularity=granularity, pv=pv)
    odt = out_dtype or q.dtype
    if odt not in _OUT_DTYPES:
        raise TypeError(f"unsupported output dtype {odt}")
    if out is None:
        out = torch.empty(q.shape, dtype=odt, pin_memory=True)
    lib = L.lib()
    need = int(lib.sage_host_workspace_bytes(ctypes.byref(p.c), int(kv_heads_per_chunk), _OUT_DTYPES[odt]))
    if need == 0:
        raise ValueError("sage_host_workspace_bytes rejected the problem")
    key = (dev.index, need)
    ws = _HOST_WS.get(key)
    if ws is None:
        _HOST_WS.clear()
        ws = _HOST_WS[key] = torch.empty(need + 256, dtype=torch.uint8, device=dev)
    base = (ws.data_ptr() + 255) // 256 * 256
    with torch.cuda.device(dev):
        st = lib.sage_attn_host(
            ctypes.byref(p.c), code, _ptr(q), _ptr(k), _ptr(v), _ptr(out), _OUT_DTYPES[odt],
            ctypes.c_float(0.0 if sm_scale is None else float(sm_scale)), 1 if is_causal else 0,
            int(kv_heads_per_chunk), ctypes.c_void_p(base), need, _stream())
        L.check("sage_attn_host", st)
        if synchronize:
            torch.cuda.current_stream().synchronize()
    return out


def debug_qk_int32(z: Quantized, seq: int, head_q: int) -> torch.Tensor:
    """Exact int32 scores of one (sequence, query head) over its padded rows (test hook)."""
    with torch.cuda.device(_require_cuda(z.q8, z.k8)):
        return _debug_qk_int32(z, seq, head_q)


def _debug_qk_int32(z, seq, head_q):
    p = z.problem
    n = (p.cu_list[seq + 1] - p.cu_list[seq]) if p.varlen else p.seqlen
    plen = -(-n // 128) * 128
    s = torch.empty((plen, plen), dtype=torch.int32, device=z.q8.device)
    st = L.lib().sage_debug_qk_int32(ctypes.byref(p.c), _ptr(z.q8), _ptr(z.k8), seq, head_q,
                                     _ptr(s), _stream())
    L.check("sage_debug_qk_int32", st)
    return s


def debug_watchdog_selftest(limit_us: int = 2000) -> None:
    """Test hook: enqueue a kernel whose bounded wait runs out after limit_us and
    records a timeout in the device watchdog word (read with poll_device_status)."""
    L.check("sage_debug_watchdog_selftest",
            L.lib().sage_debug_watchdog_selftest(int(limit_us), _stream()))


def poll_device_status() -> int:
    """Synchronize the current stream and read/clear the device watchdog word."""
    return L.lib().sage_poll_device_status(_stream())
