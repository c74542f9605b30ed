"""Decode attention for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc when they decode: a serving engine that
reserved all device memory for its own pool at start-up, or a decode loop
that cannot pay cudaMalloc's implicit device synchronisation.  For them the
library offers gqe_attn_decode_noalloc, which keeps the split-L partial states
in one fixed device array inside the library instead of a caller workspace.

These tests call it through the C ABI and compare it with gqe_attn_decode
(caller workspace) and with the fp64 oracle, within the attention tolerance,
on two calls in a row: the second call has other inputs and shorter caches,
so state left in the shared array by the first call would show.  One call
runs the main-layer decode shape (64 sequences, 8 groups, 32768 keys) and is
checked on sampled sequences.  Shapes whose partial states exceed the
array are refused before anything is launched.  The file sorts last so that a
run stopping at the first failure has run every other test first.
"""
import numpy as np
import pytest
import torch

import gqe_inputs as gi
import oracle as orc
from helpers import assert_close_attn, bf16_dev, to_f64

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


def _noalloc(dims, q, qs, Kc, Vc, L_max, lens):
    dc = gq.make_dims(dims, T=1)
    o = torch.full((dims.B, dims.G, dims.k, dims.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    os_ = torch.full((dims.B, dims.d), float("nan"), dtype=torch.bfloat16, device="cuda")
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    gq.gqe_attn_decode_noalloc(dc, q, qs, Kc, Vc, L_max, cl, o, os_)
    torch.cuda.synchronize()
    return to_f64(o), to_f64(os_)


@pytest.mark.parametrize("d", [64, 128])
def test_noalloc_decode_against_oracle_two_calls(d):
    """Seeded inputs, both calls checked against the oracle's decode attention."""
    dims = gi.GQEDims(B=3, T=1, D=256, G=2, E=4, k=2, d=d, sg=1)
    L_max = 3000
    for seed, lens in ((41, [3000, 1, 1234]), (42, [77, 2999, 640])):
        q = gi.normal_bf16(seed, "q", (dims.B, dims.G, dims.k, d))
        qs = gi.normal_bf16(seed, "qsh", (dims.B, d))
        Kc = gi.normal_bf16(seed, "Kc", (dims.B, dims.G, L_max, d))
        Vc = gi.normal_bf16(seed, "Vc", (dims.B, dims.G, L_max, d))
        o, os_ = _noalloc(dims, bf16_dev(q), bf16_dev(qs), bf16_dev(Kc), bf16_dev(Vc), L_max, lens)
        o_ref, os_ref = orc.attn_decode(q, qs, Kc, Vc, np.array(lens), dims)
        assert_close_attn(o, o_ref, f"noalloc routed rows vs oracle (seed {seed})")
        assert_close_attn(os_, os_ref, f"noalloc shared row vs oracle (seed {seed})")


def test_noalloc_decode_main_layer_sampled():
    """The main-layer decode (64 x 8 x 32768 x 64 cache, 4.3 MB of partial
    states in the array): three sequences regenerated on the host and checked
    against the oracle, the whole output against gqe_attn_decode."""
    w = gi.WORKLOADS["decode"]
    dims, L_max = w.dims, w.L
    B, G, k, d = dims.B, dims.G, dims.k, dims.d
    seed, rows = 51, [0, 29, 63]
    q = gi.normal_bf16(seed, "q", (B, G, k, d))
    qs = gi.normal_bf16(seed, "qsh", (B, d))
    gen = torch.Generator(device="cuda").manual_seed(seed)
    Kc = torch.empty((B, G, L_max, d), dtype=torch.bfloat16, device="cuda").normal_(generator=gen)
    Vc = torch.empty_like(Kc).normal_(generator=gen)
    host = {}
    for b in rows:
        Kb = gi.normal_bf16(seed, "Kc", (B, G, L_max, d), rows=[b])
        Vb = gi.normal_bf16(seed, "Vc", (B, G, L_max, d), rows=[b])
        Kc[b] = bf16_dev(Kb[0])
        Vc[b] = bf16_dev(Vb[0])
        host[b] = (Kb, Vb)
    lens = [L_max] * B
    o, os_ = _noalloc(dims, bf16_dev(q), bf16_dev(qs), Kc, Vc, L_max, lens)
    sub = dims.replace(B=1)
    for b in rows:
        Kb, Vb = host[b]
        o_ref, os_ref = orc.attn_decode(q[b:b + 1], qs[b:b + 1], Kb, Vb, np.array([L_max]), sub)
        assert_close_attn(o[b], o_ref[0], f"noalloc main-layer decode b{b}")
        assert_close_attn(os_[b], os_ref[0], f"noalloc main-layer decode shared b{b}")
    dc = gq.make_dims(dims, T=1)
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_DECODE, L_max),), dtype=torch.uint8, device="cuda")
    o2 = torch.empty((B, G, k, d), dtype=torch.bfloat16, device="cuda")
    os2 = torch.empty((B, d), dtype=torch.bfloat16, device="cuda")
    gq.gqe_attn_decode(dc, bf16_dev(q), bf16_dev(qs), Kc, Vc, L_max, torch.tensor(lens, dtype=torch.int32,
                       device="cuda"), o2, os2, ws)
    torch.cuda.synchronize()
    assert_close_attn(o, to_f64(o2), "noalloc vs workspace decode, all sequences")
    assert_close_attn(os_, to_f64(os2), "noalloc vs workspace decode shared, all sequences")
