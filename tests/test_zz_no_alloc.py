"""sage_quant_qk_noalloc: the quantization entry point for callers that cannot
allocate device memory when they quantize (a framework hook whose allocator is
locked, a plugin limited to the tensors it is handed, a pipeline with every
buffer reserved up front).  It takes its scratch from a fixed library-owned
device array instead of a caller workspace.

This file is named so that pytest collects it last: a failure here leaves every
other test already run.  It passes on its own in a fresh process and after the
rest of the suite (the shared scratch keeps whatever the previous call left).
"""

import ctypes

import pytest
import torch

from quantized_attention_06_b200 import _lib as L
from quantized_attention_06_b200 import api
from quantized_attention_06_b200.inputs import WORKLOADS, Workload, generate

CASES = [
    Workload("noalloc_nhd", 2, 8, 2, 700, 128, "bf16", "NHD", seed=31, k_offset_sigma=3.0),
    Workload("noalloc_hnd", 1, 4, 4, 333, 64, "fp16", "HND", seed=32, tail_frac=0.02,
             tail_scale=20.0),
    WORKLOADS["prefill"],
]


def _device(x, w):
    t = torch.from_numpy(x).to(torch.float16 if w.dtype == "fp16" else torch.bfloat16)
    if w.layout == "NHD":
        t = t.permute(0, 2, 1, 3).contiguous()
    return t.cuda()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    # several calls in a row, of different shapes, each against sage_quant_qk
    for rep in range(2):
        for w in CASES:
            x = generate(w)
            q, k = _device(x["q"], w), _device(x["k"], w)
            ref = api.quant_qk(q, k, w.layout)
            # poison the outputs so stale values cannot pass for fresh ones
            new = api.Quantized(ref.problem, w.layout,
                                q8=torch.full_like(ref.q8, 77), q_scale=torch.full_like(ref.q_scale, -1),
                                k8=torch.full_like(ref.k8, 77), k_scale=torch.full_like(ref.k_scale, -1),
                                k_mean=torch.full_like(ref.k_mean, -1))
            api.quant_qk_noalloc(q, k, w.layout, problem=ref.problem, out=new)
            torch.cuda.synchronize()
            assert api.poll_device_status() == 0
            for name in ("q8", "q_scale", "k8", "k_scale", "k_mean"):
                assert torch.equal(getattr(ref, name), getattr(new, name)), (rep, w.name, name)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # K-mean scratch = Hkv * (T_pad / 128) * d * 8 bytes; this one needs 32 MiB
    p = L.SageProblem(1, 64, 64, 65536, 128, L.SAGE_FP16, ctypes.POINTER(ctypes.c_int32)())
    sz = L.SageSizes()
    assert L.lib().sage_buffer_sizes(ctypes.byref(p), ctypes.byref(sz)) == 0
    assert sz.workspace_qk > L.NOALLOC_SCRATCH_BYTES
    fake = 1 << 32  # never dereferenced: the size check comes first
    s3 = L.strides3((65536 * 64 * 128, 65536 * 128, 128))
    st = L.lib().sage_quant_qk_noalloc(ctypes.byref(p), fake, s3, fake, s3, fake, fake, fake,
                                       fake, fake, None)
    assert st == L.SAGE_ERR_TOO_LARGE
    assert L.lib().sage_status_string(st) == b"SAGE_ERR_TOO_LARGE"
