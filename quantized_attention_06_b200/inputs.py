"""Seeded synthetic attention inputs.

This module is shared by the CUDA path's tests, the oracle's tests and the
benchmark.  It holds none of the attention method's arithmetic: it only draws
Q, K, V with the shapes and value distributions of the five workloads below and
rounds them to the input dtype, so that both sides of a parity check receive
exactly the same numbers.

Distributions (all iid, NumPy PCG64 via ``default_rng(seed)``):

* Q, K, V base draws ~ N(0, 1) in float32.
* Optional heavy tails: an independent Bernoulli(``tail_frac``) mask on Q and on
  K multiplies those entries by ``tail_scale`` (video-DiT workload).
* K gets a per-(sequence, kv-head, channel) offset ~ N(0, sigma^2), drawn once
  and added to every token: the channel-wise outlier structure that K smoothing
  targets (glossary page "SageAttention(セージアテンション)", 概要).
* Values are then rounded to fp16 or bf16 with round-to-nearest-even and kept
  as float32 arrays holding exactly representable values.

Draw order is fixed: sequence lengths (varlen only), Q, K, V, Q tail mask,
K tail mask, K offset.
"""

from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

__all__ = ["Workload", "WORKLOADS", "sweep_workload", "generate", "round_to_dtype"]


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    heads_q: int
    heads_kv: int
    seqlen: int                     # dense length; for varlen the maximum length
    head_dim: int
    dtype: str                      # "fp16" | "bf16"
    layout: str                     # "HND" (B,H,N,d) | "NHD" (B,N,H,d); varlen is packed (T,H,d)
    causal: tuple = (False,)
    seed: int = 0
    k_offset_sigma: float = 3.0
    tail_frac: float = 0.0
    tail_scale: float = 1.0
    varlen: bool = False
    varlen_range: tuple = (512, 8192)
    varlen_count: int = 8

    def ops(self, causal: bool, seqlens=None) -> float:
        """Tensor-core work in the convention 4*B*H*N^2*d, halved when causal."""
        lens = list(seqlens) if seqlens is not None else [self.seqlen] * self.batch
        tot = sum(4.0 * self.heads_q * n * n * self.head_dim for n in lens)
        return tot / 2 if causal else tot


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 2, 256, 64, "fp16", "HND", (False,), seed=0,
                     k_offset_sigma=2.0),
    "prefill": Workload("prefill", 4, 32, 32, 1024, 128, "bf16", "HND", (False, True),
                        seed=1, k_offset_sigma=3.0),
    "sweep": Workload("sweep", 1, 32, 32, 32768, 128, "fp16", "HND", (False, True),
                      seed=2, k_offset_sigma=3.0),
    "dit": Workload("dit", 2, 48, 48, 17550, 64, "bf16", "NHD", (False,), seed=3,
                    k_offset_sigma=4.0, tail_frac=0.02, tail_scale=20.0),
    "gqa_varlen": Workload("gqa_varlen", 8, 32, 8, 8192, 128, "bf16", "NHD", (True,),
                           seed=4, k_offset_sigma=3.0, varlen=True),
}

SWEEP_LENGTHS = (1024, 2048, 4096, 8192, 16384, 32768)


def sweep_workload(n: int) -> Workload:
    """The kernel-sweep workload (B=1, H=32, d=128, fp16) at sequence length n."""
    return replace(WORKLOADS["sweep"], name=f"sweep_{n}", seqlen=n)


def round_to_dtype(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to fp16 or bf16 (round-to-nearest-even), returned as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "fp16":
        return x.astype(np.float16).astype(np.float32)
    if dtype == "bf16":
        b = x.view(np.uint32)
        bias = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
        return ((b + bias) & np.uint32(0xFFFF0000)).view(np.float32)
    raise ValueError(f"unknown dtype {dtype}")


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def generate(w: Workload, seqlens=None) -> dict:
    """Draw the inputs of workload ``w``.

    Dense workloads return q (B,Hq,N,d), k, v (B,Hkv,N,d) in logical HND order
    (an NHD caller permutes them).  Varlen workloads return packed arrays
    q (T,Hq,d), k, v (T,Hkv,d) plus ``seqlens`` and ``cu_seqlens``; pass
    ``seqlens`` to override the seeded length draw.
    """
    rng = np.random.default_rng(w.seed)
    out = {}
    if w.varlen:
        lo, hi = w.varlen_range
        drawn = rng.integers(lo, hi + 1, size=w.varlen_count)
        lens = np.asarray(seqlens if seqlens is not None else drawn, dtype=np.int64)
        total = int(lens.sum())
        qshape = (total, w.heads_q, w.head_dim)
        kshape = (total, w.heads_kv, w.head_dim)
        out["seqlens"] = lens.astype(np.int32)
        out["cu_seqlens"] = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    else:
        qshape = (w.batch, w.heads_q, w.seqlen, w.head_dim)
        kshape = (w.batch, w.heads_kv, w.seqlen, w.head_dim)
    q = _normal(rng, qshape)
    k = _normal(rng, kshape)
    v = _normal(rng, kshape)
    if w.tail_frac > 0:
        mq = rng.random(size=qshape, dtype=np.float32) < w.tail_frac
        mk = rng.random(size=kshape, dtype=np.float32) < w.tail_frac
        q[mq] *= np.float32(w.tail_scale)
        k[mk] *= np.float32(w.tail_scale)
    if w.varlen:
        nseq = len(out["seqlens"])
        off = _normal(rng, (nseq, w.heads_kv, w.head_dim)) * np.float32(w.k_offset_sigma)
        seq_of_token = np.repeat(np.arange(nseq), out["seqlens"])
        k += off[seq_of_token]
    else:
        off = _normal(rng, (w.batch, w.heads_kv, 1, w.head_dim)) * np.float32(w.k_offset_sigma)
        k += off
    out["q"] = round_to_dtype(q, w.dtype)
    out["k"] = round_to_dtype(k, w.dtype)
    out["v"] = round_to_dtype(v, w.dtype)
    return out
