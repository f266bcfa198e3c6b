"""Host-side checks of the C ABI: the library loads without a GPU, exports every
symbol include/sage.h declares, computes buffer sizes, rejects bad arguments
before touching the device, and fails loudly (no CPU fallback) without a GPU."""

import ctypes
import os
import re

import pytest
import torch

from quantized_attention_06_b200 import _lib as L
from quantized_attention_06_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return L.lib()


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "sage.h")).read()
    return sorted(set(re.findall(r"^\s*(?:sage_status_t|const char\*|size_t)\s+(sage_\w+)\(", src, re.M)))


def test_exports_every_declared_symbol(lib):
    names = _declared_symbols()
    assert len(names) == len(L.EXPORTS)
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(L.EXPORTS)


def test_status_strings(lib):
    assert lib.sage_status_string(0) == b"SAGE_OK"
    assert lib.sage_status_string(4) == b"SAGE_ERR_DEVICE_TIMEOUT"


def _problem(b=2, hq=4, hkv=2, n=300, d=128, dtype=L.SAGE_FP16, cu=None):
    if cu is not None:
        arr = (ctypes.c_int32 * len(cu))(*cu)
        p = L.SageProblem(len(cu) - 1, hq, hkv, 0, d, dtype, ctypes.cast(arr, ctypes.POINTER(ctypes.c_int32)))
        p._keep = arr
        return p
    return L.SageProblem(b, hq, hkv, n, d, dtype, ctypes.POINTER(ctypes.c_int32)())


def _sizes(lib, p):
    s = L.SageSizes()
    return lib.sage_buffer_sizes(ctypes.byref(p), ctypes.byref(s)), s


def test_buffer_sizes_dense(lib):
    st, s = _sizes(lib, _problem())
    assert st == 0
    tp = 2 * 384
    assert s.t_pad == tp
    assert s.q8 == 4 * tp * 128 and s.k8 == 2 * tp * 128 and s.v8 == 2 * 128 * tp
    assert s.q_scale == 4 * (tp // 128) * 4 and s.k_scale == 2 * (tp // 64) * 4
    assert s.k_mean == s.v_scale == 2 * 2 * 128 * 4
    assert s.workspace_qk == 2 * (tp // 128) * 128 * 8


def test_buffer_sizes_varlen(lib):
    st, s = _sizes(lib, _problem(cu=[0, 1, 129, 129, 500], d=64))
    assert st == 0
    assert s.t_pad == 128 + 128 + 0 + 384


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), L.SAGE_ERR_UNSUPPORTED),
    (dict(dtype=7), L.SAGE_ERR_UNSUPPORTED),
    (dict(hq=6, hkv=4), L.SAGE_ERR_INVALID_ARGUMENT),
    (dict(n=0), L.SAGE_ERR_INVALID_ARGUMENT),
    (dict(b=0), L.SAGE_ERR_INVALID_ARGUMENT),
    (dict(cu=[1, 5]), L.SAGE_ERR_INVALID_ARGUMENT),
    (dict(cu=[0, 5, 3]), L.SAGE_ERR_INVALID_ARGUMENT),
    (dict(cu=[0, 0]), L.SAGE_ERR_INVALID_ARGUMENT),
])
def test_invalid_problems_rejected(lib, kw, code):
    st, _ = _sizes(lib, _problem(**kw))
    assert st == code


FAKE = 1 << 32  # 16-byte aligned, never dereferenced: validation fails first


def _quant_qk(lib, p, q=FAKE, strides=(300 * 512, 300 * 128, 128), ws_bytes=1 << 30, stream=None):
    s = L.strides3(strides)
    return lib.sage_quant_qk(ctypes.byref(p), q, s, FAKE, s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                             ws_bytes, stream)


def test_bad_pointers_strides_and_workspace_rejected(lib):
    p = _problem()
    assert _quant_qk(lib, p, q=None) == L.SAGE_ERR_INVALID_ARGUMENT
    assert _quant_qk(lib, p, q=FAKE + 8) == L.SAGE_ERR_INVALID_ARGUMENT         # misaligned
    assert _quant_qk(lib, p, strides=(1, 300 * 128, 128)) == L.SAGE_ERR_INVALID_ARGUMENT
    assert _quant_qk(lib, p, strides=(300 * 512, 300 * 128, 100)) == L.SAGE_ERR_INVALID_ARGUMENT
    assert _quant_qk(lib, p, ws_bytes=16) == L.SAGE_ERR_INVALID_ARGUMENT
    s3 = L.strides3((300 * 512, 300 * 128, 128))
    assert lib.sage_attn_fwd(ctypes.byref(p), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ctypes.c_float(0.0),
                             0, FAKE, 9, s3, None, None) == L.SAGE_ERR_UNSUPPORTED
    assert lib.sage_debug_qk_int32(ctypes.byref(p), FAKE, FAKE, 5, 0, FAKE, None) == \
        L.SAGE_ERR_INVALID_ARGUMENT


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the GPU-less host")
def test_valid_call_without_gpu_fails_loudly(lib):
    # arguments pass validation; with no device the library reports a CUDA error
    assert _quant_qk(lib, _problem()) == L.SAGE_ERR_CUDA
    with pytest.raises(RuntimeError):
        from quantized_attention_06_b200 import api
        api.Problem(1, 2, 2, 256, 64, torch.float16)  # sizes work on the host ...
        api.sageattn(torch.zeros(1, 2, 256, 64, dtype=torch.float16),
                     torch.zeros(1, 2, 256, 64, dtype=torch.float16),
                     torch.zeros(1, 2, 256, 64, dtype=torch.float16))  # ... compute does not


def _attn_host(lib, p, layout=0, ptr=FAKE, ws=FAKE, ws_bytes=1 << 40, chunk=0, odt=L.SAGE_FP16):
    return lib.sage_attn_host(ctypes.byref(p), layout, ptr, FAKE, FAKE, FAKE, odt, ctypes.c_float(0.0),
                              0, chunk, ws, ws_bytes, None)


def test_host_pipeline_workspace_and_validation(lib):
    p = _problem(b=2, hq=4, hkv=2, n=300, d=128)
    # default chunking: at least 8 chunks where possible -> one KV head per chunk here
    one = lib.sage_host_workspace_bytes(ctypes.byref(p), 1, L.SAGE_FP16)
    assert one > 0 and lib.sage_host_workspace_bytes(ctypes.byref(p), 0, L.SAGE_FP16) == one
    two = lib.sage_host_workspace_bytes(ctypes.byref(p), 2, L.SAGE_FP16)
    assert two > one
    # a slot holds q, k, v and the output of its heads plus the quantized buffers
    st, s = _sizes(lib, _problem(b=1, hq=2, hkv=1, n=300, d=128))
    assert st == 0
    q_in, kv_in, o = 2 * 300 * 128 * 2, 300 * 128 * 2, 2 * 300 * 128 * 2
    parts = [q_in, kv_in, kv_in, o, s.q8, s.q_scale, s.k8, s.k_scale, s.k_mean, s.v8, s.v_scale,
             s.workspace_qk, s.workspace_v]
    assert one == 2 * sum((x + 255) // 256 * 256 for x in parts)
    assert lib.sage_host_workspace_bytes(ctypes.byref(p), 1, L.SAGE_FP32) > one
    # rejected before anything is enqueued
    assert _attn_host(lib, p, layout=2) == L.SAGE_ERR_INVALID_ARGUMENT
    assert _attn_host(lib, p, ptr=None) == L.SAGE_ERR_INVALID_ARGUMENT
    assert _attn_host(lib, p, ptr=FAKE + 8) == L.SAGE_ERR_INVALID_ARGUMENT
    assert _attn_host(lib, p, ws=FAKE + 16) == L.SAGE_ERR_INVALID_ARGUMENT      # slots are 256-aligned
    assert _attn_host(lib, p, chunk=1, ws_bytes=one - 1) == L.SAGE_ERR_INVALID_ARGUMENT
    assert _attn_host(lib, p, odt=7) == L.SAGE_ERR_INVALID_ARGUMENT
    vl = _problem(hq=4, hkv=2, d=128, cu=[0, 100, 300])
    assert lib.sage_host_workspace_bytes(ctypes.byref(vl), 0, L.SAGE_FP16) == 0
    assert _attn_host(lib, vl) == L.SAGE_ERR_INVALID_ARGUMENT


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the GPU-less host")
def test_host_pipeline_without_gpu_fails_loudly(lib):
    p = _problem(b=1, hq=2, hkv=2, n=256, d=64)
    assert _attn_host(lib, p) == L.SAGE_ERR_CUDA


def test_granularity_sizes_and_validation(lib):
    p = _problem(b=2, hq=4, hkv=2, n=300, d=128)
    p.granularity = L.SAGE_GRAN_THREAD
    st, s = _sizes(lib, p)
    assert st == 0
    tp = 2 * 384
    assert s.q_scale == 4 * tp * 4 and s.k_scale == 2 * (tp // 32) * 4   # per token / per 32
    assert s.q8 == 4 * tp * 128 and s.k8 == 2 * tp * 128                   # codes unchanged
    for bad in (2, -1, 7):
        p.granularity = bad
        assert _sizes(lib, p)[0] == L.SAGE_ERR_INVALID_ARGUMENT
        assert _quant_qk(lib, p) == L.SAGE_ERR_INVALID_ARGUMENT


def test_python_problem_granularity():
    from quantized_attention_06_b200 import api
    p = api.Problem(1, 2, 2, 300, 64, torch.float16, granularity="thread")
    assert p.q_block == 1 and p.k_block == 32 and p.c.granularity == L.SAGE_GRAN_THREAD
    assert p.sizes.q_scale == 2 * p.t_pad * 4
    assert api.Problem(1, 2, 2, 300, 64, torch.float16).k_block == 64
    with pytest.raises(ValueError):
        api.Problem(1, 2, 2, 300, 64, torch.float16, granularity="warp")


def test_watchdog_selftest_argument_range(lib):
    assert lib.sage_debug_watchdog_selftest(0, None) == L.SAGE_ERR_INVALID_ARGUMENT
    assert lib.sage_debug_watchdog_selftest(1000001, None) == L.SAGE_ERR_INVALID_ARGUMENT
