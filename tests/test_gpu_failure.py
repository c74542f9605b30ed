"""Failure detection on the GPU without a fault (GPU).

Every wait inside the library's kernels is bounded: when its limit passes the
kernel records a code in the device error word, stops and returns, and the
context stays usable.  Here a wait that nothing completes runs out on
purpose; the host reads the code, and the next call works.
"""
import numpy as np
import pytest
import torch

import gqe_inputs as gi
import oracle as orc
from helpers import assert_close_attn, bf16_dev, to_f64

pytestmark = pytest.mark.gpu

gq = pytest.importorskip("moe_gqa_query_b200")

TIMEOUT_CODE = 0x7F1


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield


def test_bounded_wait_reports_and_the_context_stays_usable():
    torch.cuda.synchronize()
    assert gq.gqe_device_error() == 0
    gq.gqe_debug_wait_timeout()
    torch.cuda.synchronize()             # returns: the wait gave up on its own
    assert gq.gqe_device_error() == TIMEOUT_CODE
    assert gq.gqe_device_error() == 0    # read and cleared
    # the next call on the same context is correct
    dims = gi.GQEDims(B=1, T=128, D=256, G=2, E=2, k=1, d=64)
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    q = gi.normal_bf16(1, "q", (B, G, T, k, d))
    qs = gi.normal_bf16(1, "qsh", (B, T, d))
    K = gi.normal_bf16(1, "K", (B, G, T, d))
    V = gi.normal_bf16(1, "V", (B, G, T, d))
    o = torch.empty((B, G, T, k, d), dtype=torch.bfloat16, device="cuda")
    os_ = torch.empty((B, T, d), dtype=torch.bfloat16, device="cuda")
    gq.gqe_attn_prefill(gq.make_dims(dims), bf16_dev(q), bf16_dev(qs), bf16_dev(K), bf16_dev(V), o, os_, None)
    torch.cuda.synchronize()
    o_ref, os_ref, _, _ = orc.attn_prefill(q, qs, K, V, dims)
    assert_close_attn(to_f64(o), o_ref, "o after a timeout")
    assert gq.gqe_device_error() == 0
