"""sage_quant_qkv: Q, K and V quantized in one cooperative launch.  Its buffers must be
bit-identical to the separate calls sage_quant_qk + sage_quant_v (which are themselves
bit-exact against the oracle in test_gpu_quant.py), for dense and packed inputs, both
layouts, both granularities and both PV formats; one case is also checked against the
oracle directly."""

import numpy as np
import pytest
import torch

import oracle as orc
from quantized_attention_06_b200 import api
from quantized_attention_06_b200.inputs import WORKLOADS, Workload, generate

from _helpers import padded_offsets, seq_views, to_device

pytestmark = pytest.mark.gpu

CASES = [
    WORKLOADS["tiny"],
    Workload("r63", 2, 4, 2, 63, 128, "bf16", "NHD", seed=5),
    Workload("r200", 1, 3, 3, 200, 64, "bf16", "HND", seed=7, tail_frac=0.02, tail_scale=20.0),
    Workload("r1000", 2, 4, 4, 1000, 128, "fp16", "NHD", seed=21, k_offset_sigma=4.0),
    Workload("vl", 5, 4, 2, 700, 128, "bf16", "NHD", seed=9, varlen=True, varlen_range=(1, 700),
             varlen_count=5),
    Workload("vl64", 4, 6, 3, 600, 64, "fp16", "NHD", seed=12, varlen=True, varlen_range=(100, 600),
             varlen_count=4),
    WORKLOADS["prefill"],
]

NAMES = ("q8", "q_scale", "k8", "k_scale", "k_mean", "v8", "v_scale")


def _both(w, x, granularity, pv):
    q, k, v = (to_device(x[n], w.dtype, w.layout, w.varlen) for n in ("q", "k", "v"))
    cu = x["cu_seqlens"] if w.varlen else None
    ref = api.quant_qk(q, k, w.layout, cu, granularity=granularity, pv=pv)
    api.quant_v(v, ref)
    p = ref.problem
    # poison the fused call's outputs so stale values cannot pass for fresh ones
    new = api.Quantized(p, w.layout, **{n: torch.full_like(getattr(ref, n), 77 if getattr(ref, n).dtype
                                                           in (torch.int8, torch.uint8) else -1)
                                         for n in NAMES})
    api.quant_qkv(q, k, v, w.layout, cu, problem=p, out=new)
    torch.cuda.synchronize()
    assert api.poll_device_status() == 0
    return ref, new


@pytest.mark.parametrize("pv", ["fp8", "fp16"])
@pytest.mark.parametrize("granularity", ["block", "thread"])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fused_equals_separate_calls(w, granularity, pv):
    ref, new = _both(w, generate(w), granularity, pv)
    for n in NAMES:
        a, b = getattr(ref, n), getattr(new, n)
        assert torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a,
                           b.view(torch.uint8) if b.dtype == torch.bfloat16 else b), (w.name, n)


def test_fused_with_empty_sequence_matches_oracle():
    w = WORKLOADS["gqa_varlen"]
    x = generate(w, seqlens=[300, 0, 129, 1])
    ref, new = _both(w, x, "block", "fp8")
    for n in NAMES:
        assert torch.equal(getattr(ref, n), getattr(new, n)), n
    lens = [300, 0, 129, 1]
    offs, _ = padded_offsets(lens)
    k8 = new.k8.cpu().numpy(); ks = new.k_scale.cpu().numpy(); km = new.k_mean.cpu().numpy()
    v8 = new.v8.cpu().numpy(); vs = new.v_scale.cpu().numpy()
    for b, qb, kb, vb, _ in seq_views(x, True):
        n, o = lens[b], offs[b]
        if n == 0:
            continue
        for hk in (0, 5):
            mu = orc.k_channel_mean(kb[hk])
            assert np.array_equal(km[b, hk], mu)
            c8, sc = orc.quantize_int8_blocks(orc.smooth_k(kb[hk], mu), orc.BLKK)
            assert np.array_equal(k8[hk, o:o + n], c8[:n]) and np.array_equal(ks[hk, o // 64:o // 64 + len(sc)], sc)
            e, sv = orc.quantize_v_e4m3(vb[hk])
            assert np.array_equal(v8[hk, :, o:o + n], e.T) and np.array_equal(vs[b, hk], sv)


def test_fused_full_size_sweep_equals_separate_calls():
    # the 32K sweep shape: enough tiles that every CTA runs several per phase
    g = torch.Generator(device="cuda").manual_seed(5)
    q, k, v = (torch.randn(1, 32, 32768, 128, generator=g, device="cuda").half() for _ in range(3))
    ref = api.quant_qk(q, k)
    api.quant_v(v, ref)
    new = api.quant_qkv(q, k, v)
    torch.cuda.synchronize()
    for n in NAMES:
        assert torch.equal(getattr(ref, n), getattr(new, n)), n
