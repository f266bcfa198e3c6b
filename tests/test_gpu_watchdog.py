"""The failure path of the bounded waits, without a GPU fault: a kernel waits on an
mbarrier phase that nothing completes, gives up after its limit and records a
timeout in the device watchdog word; the host reads SAGE_ERR_DEVICE_TIMEOUT, the
word is cleared, and the context keeps running the real kernels correctly."""

import numpy as np
import pytest

import oracle as orc
from quantized_attention_06_b200 import _lib as L
from quantized_attention_06_b200 import api
from quantized_attention_06_b200.inputs import WORKLOADS, generate

from _helpers import from_device_out, metrics, run_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_reports_and_context_survives():
    try:
        api.debug_watchdog_selftest(2000)
        assert api.poll_device_status() == L.SAGE_ERR_DEVICE_TIMEOUT
    finally:
        api.poll_device_status()            # cleared whatever happened above
    assert api.poll_device_status() == L.SAGE_OK
    w = WORKLOADS["tiny"]
    x = generate(w)
    _, out, _ = run_gpu(x, w.dtype, w.layout, w.varlen, False)
    o = from_device_out(out, w.layout, w.varlen)
    for h in range(w.heads_q):
        ref = orc.attention_head(x["q"][0, h], x["k"][0, h], x["v"][0, h])["out"]
        mx, cos, _ = metrics(o[0, h], ref)
        assert mx <= 2e-3 and cos >= 0.9999
