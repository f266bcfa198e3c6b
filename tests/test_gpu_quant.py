"""GPU parity of the quantization kernels and the int32 scores against the oracle.

Every quantized buffer (q8, q_scale, k8, k_scale, k_mean, v8, v_scale) and the
int32 S = Q8 K8^T must be bit-exact, padding included."""

from dataclasses import replace

import numpy as np
import pytest
import torch

import oracle as orc
from quantized_attention_06_b200 import api
from quantized_attention_06_b200.inputs import WORKLOADS, Workload, generate

from _helpers import padded_offsets, seq_views, to_device

pytestmark = pytest.mark.gpu


def _quantize(x, w: Workload):
    q = to_device(x["q"], w.dtype, w.layout, w.varlen)
    k = to_device(x["k"], w.dtype, w.layout, w.varlen)
    v = to_device(x["v"], w.dtype, w.layout, w.varlen)
    z = api.quant_qk(q, k, w.layout, x.get("cu_seqlens") if w.varlen else None)
    api.quant_v(v, z)
    torch.cuda.synchronize()
    assert api.poll_device_status() == 0
    return z


def _check_quant(x, w: Workload, z, heads=None):
    q8 = z.q8.cpu().numpy(); qs = z.q_scale.cpu().numpy()
    k8 = z.k8.cpu().numpy(); ks = z.k_scale.cpu().numpy(); km = z.k_mean.cpu().numpy()
    v8 = z.v8.cpu().numpy(); vs = z.v_scale.cpu().numpy()
    lens = [int(n) for n in x["seqlens"]] if w.varlen else [w.seqlen] * w.batch
    offs, tpad = padded_offsets(lens)
    assert z.problem.t_pad == tpad
    g = w.heads_q // w.heads_kv
    for b, qb, kb, vb, _ in seq_views(x, w.varlen):
        n, o, P = lens[b], offs[b], -(-lens[b] // 128) * 128
        if n == 0:
            assert np.all(km[b] == 0) and np.all(vs[b] == 0)
            continue
        for hk in range(w.heads_kv) if heads is None else sorted({h // g for h in heads}):
            mu = orc.k_channel_mean(kb[hk])
            assert np.array_equal(km[b, hk], mu), (b, hk)
            k8o, kso = orc.quantize_int8_blocks(orc.smooth_k(kb[hk], mu), orc.BLKK)
            nk = k8o.shape[0]
            assert np.array_equal(k8[hk, o:o + nk], k8o), (b, hk)
            assert np.all(k8[hk, o + nk:o + P] == 0)
            assert np.array_equal(ks[hk, o // 64:o // 64 + len(kso)], kso)
            assert np.all(ks[hk, o // 64 + len(kso):(o + P) // 64] == 0)
            v8o, svo = orc.quantize_v_e4m3(vb[hk])
            assert np.array_equal(vs[b, hk], svo), (b, hk)
            assert np.array_equal(v8[hk, :, o:o + n], v8o.T), (b, hk)
            assert np.all(v8[hk, :, o + n:o + P] == 0)
        for h in range(w.heads_q) if heads is None else heads:
            q8o, qso = orc.quantize_int8_blocks(qb[h], orc.BLKQ)
            assert np.array_equal(q8[h, o:o + P], q8o), (b, h)
            assert np.array_equal(qs[h, o // 128:(o + P) // 128], qso), (b, h)


SMALL = [
    WORKLOADS["tiny"],
    Workload("r63", 2, 4, 2, 63, 128, "bf16", "NHD", seed=5),
    Workload("r1", 1, 2, 1, 1, 64, "fp16", "HND", seed=6),
    Workload("r200", 1, 3, 3, 200, 64, "bf16", "HND", seed=7, tail_frac=0.02, tail_scale=20.0),
    Workload("r383", 2, 2, 2, 383, 128, "fp16", "NHD", seed=8, k_offset_sigma=4.0),
    Workload("vl", 5, 4, 2, 700, 128, "bf16", "NHD", seed=9, varlen=True, varlen_range=(1, 700),
             varlen_count=5),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_quant_bit_exact_small(w):
    x = generate(w)
    z = _quantize(x, w)
    _check_quant(x, w, z)


def test_quant_bit_exact_varlen_with_empty_sequence():
    w = replace(WORKLOADS["gqa_varlen"], name="vl_empty")
    x = generate(w, seqlens=[300, 0, 129, 1])
    z = _quantize(x, w)
    _check_quant(x, w, z)


@pytest.mark.parametrize("name", ["prefill", "dit", "gqa_varlen"])
def test_quant_bit_exact_full_size(name):
    w = WORKLOADS[name]
    x = generate(w)
    z = _quantize(x, w)
    heads = [0, w.heads_q // 2, w.heads_q - 1]
    _check_quant(x, w, z, heads=heads)


def test_quant_bit_exact_sweep_32k():
    from quantized_attention_06_b200.inputs import sweep_workload
    w = sweep_workload(32768)
    x = generate(w)
    z = _quantize(x, w)
    _check_quant(x, w, z, heads=[0, 17, 31])


@pytest.mark.parametrize("w", [WORKLOADS["tiny"], SMALL[4], SMALL[5],
                               replace(WORKLOADS["prefill"], batch=1, heads_q=2, heads_kv=2)],
                         ids=lambda w: w.name)
def test_int32_scores_bit_exact(w):
    x = generate(w)
    z = _quantize(x, w)
    g = w.heads_q // w.heads_kv
    for b, qb, kb, _, _ in seq_views(x, w.varlen):
        n = qb.shape[1]
        if n == 0:
            continue
        for h in (0, w.heads_q - 1):
            q8o, _ = orc.quantize_int8_blocks(qb[h], orc.BLKQ)
            k8o, _ = orc.quantize_int8_blocks(orc.smooth_k(kb[h // g], orc.k_channel_mean(kb[h // g])),
                                             orc.BLKK)
            P = q8o.shape[0]
            k8p = np.zeros((P, k8o.shape[1]), dtype=np.int8)
            k8p[:k8o.shape[0]] = k8o[:P]
            s = api.debug_qk_int32(z, b, h).cpu().numpy()
            assert np.array_equal(s, orc.integer_scores(q8o, k8p)), (b, h)
