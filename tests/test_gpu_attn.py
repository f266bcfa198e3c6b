"""GPU parity of sage_attn_fwd against the oracle.

The reference is ``oracle.attention_head``: the same smoothing, block quantization
and integer QK^T as the kernel, then everything after it in fp64 (the definition).
Bars, on fp32 output: max-abs error <= 2e-3 and cosine similarity >= 0.9999; lse
within 1e-3.  The kernel forms p in fp32 but decides every e4m3 P code that lies near
a rounding midpoint from the fp64 definition, so its codes are the definition's.  The
report also records the distance to ``attention_head_fp32_logits`` (fp32 logits, exact
exponential), which differs from the definition exactly where fp32 logits would flip
a code.  Small cases are compared element by element on every row; full-size
workloads on sampled rows (first and last tiles included) of several (sequence,
head) pairs.  fp16 / bf16 outputs are compared against the reference rounded to that
dtype, with one extra unit in the last place allowed.

Both PV formats are covered: e4m3 P and V (the method) and the 16-bit option
(P and V in the input's type), each against the references with the same format.
"""

from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle as orc
from quantized_attention_06_b200.inputs import (SWEEP_LENGTHS, WORKLOADS, Workload, generate,
                                                sweep_workload)

from _helpers import (MAX_ABS, MIN_COS, REPORT, from_device_out, metrics, oracle_pv, padded_offsets,
                      run_gpu, seq_views)

pytestmark = pytest.mark.gpu


def _oracle_rows(x, w, causal, pairs, pv="fp8", granularity="block"):
    """{(b, h): (rows, out64, lse64, out32)}: the fp64 definition and the fp32-logit
    reference for the requested (b, h, rows)."""
    g = w.heads_q // w.heads_kv
    qb, kb = (1, 32) if granularity == "thread" else (orc.BLKQ, orc.BLKK)
    views = {b: (q, k, v) for b, q, k, v, _ in seq_views(x, w.varlen)}
    res = {}
    for b, h, rows in pairs:
        q, k, v = views[b]
        kw = dict(causal=causal, rows=rows, pv=oracle_pv(pv, w.dtype), qblk=qb, kblk=kb)
        r64 = orc.attention_head(q[h], k[h // g], v[h // g], **kw)
        r32 = orc.attention_head_fp32_logits(q[h], k[h // g], v[h // g], **kw)
        res[(b, h)] = (r64["rows"], r64["out"], r64["lse"], r32["out"])
    return res


def _gpu_rows(out_np, lse_np, x, w, b, h, rows):
    lens = [int(n) for n in x["seqlens"]] if w.varlen else [w.seqlen] * w.batch
    offs, _ = padded_offsets(lens)
    if w.varlen:
        s0 = int(x["cu_seqlens"][b])
        o = out_np[s0 + rows, h]
    else:
        o = out_np[b, h, rows]
    return o, lse_np[h, offs[b] + rows]


def check_parity(x, w, causal, pairs, out_dtype=torch.float32, pv="fp8", granularity="block",
                 tag=""):
    """Run the CUDA path once and compare the requested rows with both references."""
    z, out, lse = run_gpu(x, w.dtype, w.layout, w.varlen, causal, out_dtype=out_dtype, pv=pv,
                          granularity=granularity)
    out_np = from_device_out(out, w.layout, w.varlen)
    lse_np = lse.cpu().numpy()
    ref = _oracle_rows(x, w, causal, pairs, pv, granularity)
    for (b, h), (rows, o64, lse_ref, o32) in ref.items():
        o_gpu, l_gpu = _gpu_rows(out_np, lse_np, x, w, b, h, rows)
        if out_dtype == torch.float32:
            mx, cos, _ = metrics(o_gpu, o64)
            assert mx <= MAX_ABS, (b, h, mx)
        else:
            o_ref_r = torch.from_numpy(o64).to(out_dtype).double().numpy()
            mant = 7 if out_dtype == torch.bfloat16 else 10        # explicit mantissa bits
            _, ex = np.frexp(np.maximum(np.abs(o_ref_r), 2.0 ** -14))
            ulp = np.ldexp(1.0, ex - 1 - mant)                      # one unit in the last place
            assert np.all(np.abs(o_gpu - o_ref_r) <= MAX_ABS + ulp), (b, h)
            _, cos, _ = metrics(o_gpu, o64)
        REPORT.append({"case": f"{tag}{w.name} causal={causal} pv={pv} gran={granularity} "
                               f"out={str(out_dtype).split('.')[-1]} b={b} h={h}",
                       "rows": int(len(rows)), "max_abs_vs_fp64": float(np.max(np.abs(o_gpu - o64))),
                       "cos_vs_fp64": cos,
                       "max_abs_vs_fp32_logits": float(np.max(np.abs(o_gpu - o32))),
                       "fp32_logits_vs_fp64_max_abs": float(np.max(np.abs(o32 - o64))),
                       "lse_max_abs": float(np.max(np.abs(l_gpu - lse_ref)))})
        assert cos >= MIN_COS, (b, h, cos)
        assert np.max(np.abs(l_gpu - lse_ref)) <= 1e-3, (b, h)
    return out_np


SMALL = [
    WORKLOADS["tiny"],
    Workload("r1", 1, 2, 1, 1, 64, "fp16", "HND", seed=6),
    Workload("r63", 2, 4, 2, 63, 128, "bf16", "NHD", seed=5),
    Workload("r129", 1, 2, 2, 129, 128, "fp16", "HND", seed=10),
    Workload("r200", 1, 3, 3, 200, 64, "bf16", "HND", seed=7, tail_frac=0.02, tail_scale=20.0),
    Workload("r383", 2, 2, 2, 383, 128, "fp16", "NHD", seed=8, k_offset_sigma=4.0),
    Workload("r640", 1, 4, 1, 640, 128, "bf16", "HND", seed=11),
    Workload("vl", 5, 4, 2, 700, 128, "bf16", "NHD", seed=9, varlen=True, varlen_range=(1, 700),
             varlen_count=5),
    Workload("vl64", 4, 6, 3, 600, 64, "fp16", "NHD", seed=12, varlen=True, varlen_range=(100, 600),
             varlen_count=4),
]


def _all_rows(x, w):
    return [(b, h, np.arange(q.shape[1])) for b, q, _, _, _ in seq_views(x, w.varlen)
            if q.shape[1] > 0 for h in range(w.heads_q)]


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_attention_small_all_rows(w, causal, pv):
    x = generate(w)
    check_parity(x, w, causal, _all_rows(x, w), pv=pv)


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
def test_attention_half_outputs(out_dtype):
    w = SMALL[5]
    x = generate(w)
    pairs = [(b, h, np.arange(w.seqlen)) for b in range(w.batch) for h in range(w.heads_q)]
    check_parity(x, w, True, pairs, out_dtype=out_dtype)


def test_attention_varlen_with_empty_sequence():
    w = replace(WORKLOADS["gqa_varlen"], name="vl_empty")
    x = generate(w, seqlens=[300, 0, 129, 1])
    pairs = [(b, h, np.arange(n)) for b, n in enumerate([300, 0, 129, 1]) if n > 0
             for h in (0, 7, 31)]
    check_parity(x, w, True, pairs)


def sample_rows(n, k=1024):
    head = np.arange(min(n, 256))
    tail = np.arange(max(0, n - 256), n)
    mid = np.linspace(0, n - 1, k).astype(np.int64)
    return np.unique(np.concatenate([head, mid, tail]))


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
@pytest.mark.parametrize("causal", [False, True])
def test_attention_prefill(causal, pv):
    w = WORKLOADS["prefill"]
    x = generate(w)
    pairs = [(b, h, np.arange(w.seqlen)) for b, h in ((0, 0), (1, 13), (2, 31), (3, 7))]
    check_parity(x, w, causal, pairs, pv=pv)


@pytest.mark.parametrize("n", SWEEP_LENGTHS)
@pytest.mark.parametrize("causal", [False, True])
def test_attention_sweep_sampled(n, causal):
    w = sweep_workload(n)
    x = generate(w)
    pairs = [(0, h, sample_rows(n)) for h in (0, 9, 22, 31)]
    check_parity(x, w, causal, pairs)


@pytest.mark.parametrize("n", [4096, 32768])
def test_attention_sweep_sampled_pv16(n):
    w = sweep_workload(n)
    x = generate(w)
    pairs = [(0, h, sample_rows(n, 512)) for h in (0, 31)]
    check_parity(x, w, False, pairs, pv="fp16")


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
def test_attention_dit_sampled(pv):
    w = WORKLOADS["dit"]
    x = generate(w)
    pairs = [(b, h, sample_rows(w.seqlen)) for b, h in ((0, 0), (0, 47), (1, 20), (1, 33))]
    check_parity(x, w, False, pairs, pv=pv)


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
def test_attention_gqa_varlen_sampled(pv):
    w = WORKLOADS["gqa_varlen"]
    x = generate(w)
    lens = [int(n) for n in x["seqlens"]]
    pairs = [(b, h, sample_rows(lens[b], 512)) for b in (0, 3, 7) for h in (0, 5, 31)]
    check_parity(x, w, True, pairs, pv=pv)


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
def test_gqa_equals_repeated_kv_on_gpu(pv):
    w = Workload("gqa", 1, 8, 2, 300, 128, "bf16", "HND", seed=13)
    x = generate(w)
    _, out_a, _ = run_gpu(x, w.dtype, w.layout, False, True, pv=pv)
    x2 = dict(x, k=np.repeat(x["k"], 4, axis=1), v=np.repeat(x["v"], 4, axis=1))
    _, out_b, _ = run_gpu(x2, w.dtype, w.layout, False, True, pv=pv)
    assert torch.equal(out_a, out_b)


def test_layouts_agree_on_gpu():
    w = Workload("lay", 2, 4, 4, 333, 64, "fp16", "HND", seed=14)
    x = generate(w)
    _, out_h, _ = run_gpu(x, w.dtype, "HND", False, False)
    _, out_n, _ = run_gpu(x, w.dtype, "NHD", False, False)
    assert torch.equal(out_h, out_n.permute(0, 2, 1, 3))
