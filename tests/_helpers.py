"""Shared helpers for the parity tests: run the CUDA path and the oracle on the
same seeded inputs and map the GPU's padded buffers back to per-head arrays."""

from __future__ import annotations

import numpy as np
import torch

import oracle as orc
from quantized_attention_06_b200 import api

TORCH_DT = {"fp16": torch.float16, "bf16": torch.bfloat16}

# GPU vs oracle bars for the attention output (both carry the same quantization)
MAX_ABS = 2e-3
MIN_COS = 0.9999

# (case, max-abs, cos) of every comparison; written out by conftest when
# SAGE_PARITY_REPORT names a file
REPORT = []


def to_device(x: np.ndarray, dtype: str, layout: str, varlen: bool) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x)).to(TORCH_DT[dtype])
    if not varlen and layout == "NHD":
        t = t.permute(0, 2, 1, 3).contiguous()
    return t.cuda()


def from_device_out(out: torch.Tensor, layout: str, varlen: bool) -> np.ndarray:
    o = out.float().cpu().numpy().astype(np.float64)
    if not varlen and layout == "NHD":
        o = o.transpose(0, 2, 1, 3)
    return o


def seq_views(x: dict, varlen: bool):
    """Yield (seq index, q (Hq,n,d), k, v (Hkv,n,d), token offset) per sequence."""
    if varlen:
        cu = x["cu_seqlens"]
        for b in range(len(cu) - 1):
            s0, s1 = cu[b], cu[b + 1]
            yield b, x["q"][s0:s1].transpose(1, 0, 2), x["k"][s0:s1].transpose(1, 0, 2), \
                x["v"][s0:s1].transpose(1, 0, 2), s0
    else:
        for b in range(x["q"].shape[0]):
            yield b, x["q"][b], x["k"][b], x["v"][b], None


def padded_offsets(lens):
    offs, o = [], 0
    for n in lens:
        offs.append(o)
        o += -(-n // 128) * 128
    return offs, o


def oracle_pv(pv: str, dtype: str) -> str:
    """The oracle's PV format for the library's: e4m3, or the input's 16-bit type."""
    return "e4m3" if pv == "fp8" else dtype


def run_gpu(x: dict, dtype: str, layout: str, varlen: bool, causal: bool, out_dtype=torch.float32,
            return_lse=True, pv="fp8", granularity="block"):
    q = to_device(x["q"], dtype, layout, varlen)
    k = to_device(x["k"], dtype, layout, varlen)
    v = to_device(x["v"], dtype, layout, varlen)
    cu = x["cu_seqlens"] if varlen else None
    z = api.quant_qk(q, k, layout, cu, granularity=granularity, pv=pv)
    api.quant_v(v, z)
    out, lse = api.attn_fwd(z, is_causal=causal, out_dtype=out_dtype, return_lse=True)
    torch.cuda.synchronize()
    assert api.poll_device_status() == 0
    return z, out, lse


def reference_rows(q, k, v, rows, causal):
    """Full-precision softmax attention (fp64, no quantization) for the given query rows."""
    x = (q[rows].astype(np.float64) @ k.astype(np.float64).T) / np.sqrt(q.shape[1])
    if causal:
        x = np.where(np.arange(k.shape[0])[None, :] > np.asarray(rows)[:, None], -np.inf, x)
    x = x - x.max(axis=1, keepdims=True)
    p = np.exp(x)
    return (p @ v.astype(np.float64)) / p.sum(axis=1, keepdims=True)


def metrics(a: np.ndarray, b: np.ndarray):
    a, b = a.ravel().astype(np.float64), b.ravel().astype(np.float64)
    cos = float(a @ b / (np.linalg.norm(a) * np.linalg.norm(b) + 1e-300))
    rel_l1 = float(np.sum(np.abs(a - b)) / (np.sum(np.abs(b)) + 1e-300))
    return float(np.max(np.abs(a - b))), cos, rel_l1
