"""The whole prefill forward behind one C-ABI call.

gqe_layer_forward (device x and y) and gqe_layer_forward_host (x and y in
pinned host memory, the batch cut into chunks of sequences whose copies in,
forwards and copies back overlap on three streams) chain the same entry
points as GQELayer.forward.  Checks:
  - tiny workload: the one-call result equals GQELayer.forward's and matches
    the fp64 oracle on every row (max-abs 2e-2, mean-abs 2e-3);
  - main-layer and wide/skewed workloads through host buffers, chunks of one
    sequence, of a ragged size and of the whole batch: every sequence against
    GQELayer.forward on the device (the same kernels on the same rows), within
    max-abs 2e-2 and a per-sequence mean-abs of 2e-4, ten times below the
    error a sequence written to the wrong place would leave (about 1.7e-2);
  - two calls in a row on other inputs with no synchronisation between them
    (the second call's copies and forwards are ordered behind the first's
    only by what the first call leaves on the streams);
  - the three streams given as one stream.
"""
import numpy as np
import pytest
import torch

import gqe_inputs as gi
import oracle as orc
from helpers import assert_close_attn, bf16_dev, to_f64

pytestmark = pytest.mark.gpu

gq = pytest.importorskip("moe_gqa_query_b200")

SEQ_MEAN_ABS = 2e-4


@pytest.fixture(autouse=True)
def _cuda_and_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    assert gq.gqe_device_error() == 0
    torch.cuda.empty_cache()


def _layer(w, seed=0):
    dims = w.dims
    Wt = gi.layer_weights(dims, seed)
    bias = gi.router_bias(w, seed)
    layer = gq.GQELayer(dims, {k_: torch.from_numpy(v.view(np.int16)) for k_, v in Wt.items()}, bias)
    return Wt, bias, layer


def _pinned(x_u16):
    return torch.from_numpy(np.ascontiguousarray(x_u16).view(np.int16)).view(torch.bfloat16).pin_memory()


def _host_out(dims):
    return torch.full((dims.B, dims.T, dims.D), float("nan"), dtype=torch.bfloat16).pin_memory()


def _assert_per_sequence(got, ref, what):
    """got, ref [B, T, D] float64: every sequence within max-abs 2e-2 and
    mean-abs SEQ_MEAN_ABS of the reference."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    for b in range(got.shape[0]):
        err = np.abs(got[b] - ref[b])
        mx, mean = float(err.max()), float(err.mean())
        assert mx <= 2e-2 and mean <= SEQ_MEAN_ABS, f"{what} sequence {b}: max-abs {mx:.3e} mean-abs {mean:.3e}"


def test_layer_forward_one_call_tiny_against_oracle():
    w = gi.WORKLOADS["tiny_prefill"]
    dims = w.dims
    Wt, bias, layer = _layer(w)
    x = gi.layer_input(dims, 0)
    xd = bf16_dev(x)
    dc = gq.make_dims(dims)
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_LAYER_FORWARD),), dtype=torch.uint8, device="cuda")
    y = torch.full((dims.B, dims.T, dims.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    gq.gqe_layer_forward(dc, gq.layer_weights(layer), xd, y, ws)
    y_layer = layer.forward(xd).clone()
    torch.cuda.synchronize()
    assert torch.equal(y, y_layer), "one-call forward differs from the chained calls"
    ref = orc.gqe_forward(x, Wt, dims, bias)
    assert_close_attn(to_f64(y).reshape(dims.N, -1), ref["y"], "gqe_layer_forward y vs oracle")
    # the host form on the same workload, one chunk per sequence, and with a
    # chunk size above the batch (the batch runs as one chunk)
    for chunk in (1, 4):
        yh = _host_out(dims)
        layer.forward_host_c(_pinned(x), yh, chunk_seqs=chunk)
        torch.cuda.synchronize()
        assert torch.equal(yh, y.cpu()), f"host-buffer forward (chunk {chunk}) differs from the device one"


@pytest.mark.parametrize("wname,chunks", [("main_prefill", (1, 2, 3, 8)), ("wide_skewed_prefill", (1,))])
def test_layer_forward_host_chunks(wname, chunks):
    w = gi.WORKLOADS[wname]
    dims = w.dims
    _, _, layer = _layer(w)
    x = gi.layer_input(dims, 0)
    ref = to_f64(layer.forward(bf16_dev(x)))
    xh = _pinned(x)
    for c in chunks:
        yh = _host_out(dims)
        layer.forward_host_c(xh, yh, chunk_seqs=c)
        torch.cuda.synchronize()
        _assert_per_sequence(to_f64(yh), ref, f"{wname} chunk {c}")


def test_layer_forward_host_two_calls_in_a_row():
    w = gi.WORKLOADS["main_prefill"]
    dims = w.dims
    _, _, layer = _layer(w)
    xs = [gi.layer_input(dims, s) for s in (3, 4)]
    refs = [to_f64(layer.forward(bf16_dev(x))) for x in xs]
    xh = [_pinned(x) for x in xs]
    yh = [_host_out(dims) for _ in xs]
    torch.cuda.synchronize()
    for i in range(2):     # chained on the layer's streams, no synchronisation or join between the calls
        layer.forward_host_c(xh[i], yh[i], chunk_seqs=1, join=False)
    torch.cuda.synchronize()
    for i in range(2):
        _assert_per_sequence(to_f64(yh[i]), refs[i], f"call {i}")


def test_layer_forward_host_single_stream():
    w = gi.WORKLOADS["main_prefill"]
    dims = w.dims
    _, _, layer = _layer(w)
    x = gi.layer_input(dims, 5)
    ref = to_f64(layer.forward(bf16_dev(x)))
    cd = gq.make_dims(dims, B=2)
    ws = torch.empty((gq.gqe_workspace_size(cd, gq.GQE_OP_LAYER_FORWARD_HOST),), dtype=torch.uint8, device="cuda")
    yh = _host_out(dims)
    s = torch.cuda.current_stream()
    gq.gqe_layer_forward_host(gq.make_dims(dims), gq.layer_weights(layer), _pinned(x), yh, 2, ws, s, s, s)
    torch.cuda.synchronize()
    _assert_per_sequence(to_f64(yh), ref, "single stream")
