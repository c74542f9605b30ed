"""Decode attention for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they decode: a serving engine that
reserved all device memory for its own pool at start-up, or a decode loop
that cannot pay cudaMalloc's implicit device synchronisation.  For them the
library offers gqe_attn_decode_noalloc, which keeps the split-L partial states
in one fixed device array inside the library instead of a caller workspace.

These tests call it through the C ABI and compare it with gqe_attn_decode
(caller workspace) within the attention tolerance, on two calls in a row: the
second call has other inputs and shorter caches, so state left in the shared
array by the first call would show.  Shapes whose partial states exceed the
array are refused before anything is launched.  The file sorts last so that a
run stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

import gqe_inputs as gi
from helpers import assert_close_attn, to_f64

pytestmark = pytest.mark.gpu

gq = pytest.importorskip("moe_gqa_query_b200")


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    assert gq.gqe_device_error() == 0


def _decode_both(dims, L_max, lens, seed):
    B, G, k, d = dims.B, dims.G, dims.k, dims.d
    gen = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, G, k, d), device="cuda", generator=gen).to(torch.bfloat16)
    qs = torch.randn((B, d), device="cuda", generator=gen).to(torch.bfloat16)
    Kc = torch.randn((B, G, L_max, d), device="cuda", generator=gen).to(torch.bfloat16)
    Vc = torch.randn((B, G, L_max, d), device="cuda", generator=gen).to(torch.bfloat16)
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    dc = gq.make_dims(dims, T=1)
    # existing entry point, caller workspace
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_DECODE, L_max),), dtype=torch.uint8, device="cuda")
    o_ref = torch.empty_like(q)
    os_ref = torch.empty_like(qs)
    gq.gqe_attn_decode(dc, q, qs, Kc, Vc, L_max, cl, o_ref, os_ref, ws)
    # no-allocation entry point
    o = torch.full_like(q, float("nan"))
    os_ = torch.full_like(qs, float("nan"))
    gq.gqe_attn_decode_noalloc(dc, q, qs, Kc, Vc, L_max, cl, o, os_)
    torch.cuda.synchronize()
    return to_f64(o), to_f64(o_ref), to_f64(os_), to_f64(os_ref)


@pytest.mark.parametrize("d", [64, 128])
def test_noalloc_decode_matches_workspace_decode_two_calls(d):
    dims = gi.GQEDims(B=4, T=1, D=256, G=3, E=4, k=2, d=d, sg=1)
    calls = [(5000, [5000, 4000, 2500, 17], 1),     # first call: long caches
             (5000, [100, 3000, 1, 64], 2)]         # second call: other inputs, shorter caches
    for L_max, lens, seed in calls:
        o, o_ref, os_, os_ref = _decode_both(dims, L_max, lens, seed)
        assert np.isfinite(o).all() and np.isfinite(os_).all()
        assert_close_attn(o, o_ref, f"noalloc routed rows (seed {seed})")
        assert_close_attn(os_, os_ref, f"noalloc shared row (seed {seed})")


def test_noalloc_decode_main_layer_shape_fits():
    """The main-layer decode (64 sequences, 8 groups, 32768 keys) fits the array."""
    w = gi.WORKLOADS["decode"]
    dc = gq.make_dims(w.dims, T=1)
    assert gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_DECODE, w.L) <= gq.DECODE_NOALLOC_MAX_BYTES


def test_noalloc_decode_rejects_oversize_before_launch():
    dims = gi.GQEDims(B=64, T=1, D=1024, G=8, E=2, k=1, d=64)
    dc = gq.make_dims(dims, T=1)
    L_max = 1 << 17
    assert gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_DECODE, L_max) > gq.DECODE_NOALLOC_MAX_BYTES
    buf = torch.empty((64,), dtype=torch.bfloat16, device="cuda")   # never read: refused first
    cl = torch.ones((64,), dtype=torch.int32, device="cuda")
    with pytest.raises(gq.GQEError) as ei:
        gq.gqe_attn_decode_noalloc(dc, buf, buf, buf, buf, L_max, cl, buf, buf)
    assert ei.value.status == 3     # GQE_ERR_WORKSPACE
