"""sage_attn_host (sageattn_host): the path on host buffers, pipelined over chunks
of heads, gives bit-identical outputs to the device path (every head's quantization
and attention are independent of the other heads)."""

import pytest
import torch

from quantized_attention_06_b200 import api

pytestmark = pytest.mark.gpu


def _inputs(b, hq, hkv, n, d, dtype, layout, seed):
    g = torch.Generator().manual_seed(seed)
    shape = (lambda h: (b, h, n, d)) if layout == "HND" else (lambda h: (b, n, h, d))
    q = torch.randn(shape(hq), generator=g).to(dtype)
    k = (torch.randn(shape(hkv), generator=g) + 3 * torch.randn(d, generator=g)).to(dtype)
    v = torch.randn(shape(hkv), generator=g).to(dtype)
    return [t.contiguous().pin_memory() for t in (q, k, v)]


@pytest.mark.parametrize("layout", ["HND", "NHD"])
@pytest.mark.parametrize("chunk", [0, 1, 2, 3])
def test_host_path_equals_device_path(layout, chunk):
    q, k, v = _inputs(2, 8, 4, 300, 128, torch.float16, layout, 1 + chunk)
    ref = api.sageattn(q.cuda(), k.cuda(), v.cuda(), tensor_layout=layout).cpu()
    out = api.sageattn_host(q, k, v, tensor_layout=layout, kv_heads_per_chunk=chunk)
    assert out.shape == ref.shape and out.dtype == ref.dtype
    assert torch.equal(out, ref)


@pytest.mark.parametrize("causal", [False, True])
def test_host_path_causal_bf16_fp32_out(causal):
    q, k, v = _inputs(1, 6, 2, 1000, 64, torch.bfloat16, "HND", 7)
    ref = api.sageattn(q.cuda(), k.cuda(), v.cuda(), is_causal=causal, out_dtype=torch.float32).cpu()
    out = api.sageattn_host(q, k, v, is_causal=causal, out_dtype=torch.float32, kv_heads_per_chunk=1)
    assert out.dtype == torch.float32
    assert torch.equal(out, ref)


def test_host_path_back_to_back_and_stream_order():
    # two calls enqueued without synchronizing share the internal copy streams; the
    # second must not overwrite slots the first still uses
    q1, k1, v1 = _inputs(1, 4, 4, 2048, 128, torch.float16, "HND", 11)
    q2, k2, v2 = _inputs(1, 4, 4, 2048, 128, torch.float16, "HND", 12)
    r1 = api.sageattn(q1.cuda(), k1.cuda(), v1.cuda()).cpu()
    r2 = api.sageattn(q2.cuda(), k2.cuda(), v2.cuda()).cpu()
    o1 = api.sageattn_host(q1, k1, v1, kv_heads_per_chunk=1, synchronize=False)
    o2 = api.sageattn_host(q2, k2, v2, kv_heads_per_chunk=1, synchronize=False)
    torch.cuda.current_stream().synchronize()
    assert torch.equal(o1, r1) and torch.equal(o2, r2)
    assert api.poll_device_status() == 0


@pytest.mark.parametrize("chunk", [3, 0])
def test_host_path_short_chunk_in_slot_zero(chunk):
    # Hkv = 8 in chunks of 3 gives chunks of 3, 3, 2 per batch entry; with B = 3 the
    # short chunk lands in slot 0 as well as slot 1.  Every slot must keep the full
    # chunk's size as its stride, or a later chunk's buffers overlap one still in flight.
    q, k, v = _inputs(3, 16, 8, 257, 128, torch.bfloat16, "NHD", 31)
    ref = api.sageattn(q.cuda(), k.cuda(), v.cuda(), tensor_layout="NHD").cpu()
    out = api.sageattn_host(q, k, v, tensor_layout="NHD", kv_heads_per_chunk=chunk)
    assert torch.equal(out, ref)
    assert api.poll_device_status() == 0
