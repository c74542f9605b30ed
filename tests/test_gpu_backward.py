"""Parity of the backward calls with the fp64 backward oracle (GPU).

The backward oracle is pinned by finite differences of the forward oracle
(tests/test_oracle_backward_pins.py).  Each call gets the same bf16 inputs as
the oracle (the forward output O and log-sum-exp included: per-call parity).
Gradients are held to the worst-case error of their arithmetic
(helpers.assert_close_grad, oracle attn_prefill_bwd_error_bound): bf16
rounding of every MMA operand and of the result, fp32 accumulation; plus a
mean-abs check of 2e-3 of the reference's rms.
"""
import numpy as np
import pytest
import torch

import gqe_inputs as gi
import oracle as orc
from oracle import gqe_backward as ob
from helpers import assert_close_grad, bf16_dev, to_f64

pytestmark = pytest.mark.gpu

gq = pytest.importorskip("moe_gqa_query_b200")


@pytest.fixture(autouse=True)
def _cuda_and_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    assert gq.gqe_device_error() == 0


def D(**kw):
    base = dict(B=1, T=128, D=256, G=2, E=2, k=1, d=64)
    base.update(kw)
    return gi.GQEDims(**base)


# ----------------------------------------------------------------------------
# attention backward

def _attn_bwd_inputs(dims, seed):
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    q = gi.normal_bf16(seed, "q", (B, G, T, k, d))
    qs = gi.normal_bf16(seed, "qsh", (B, T, d))
    K = gi.normal_bf16(seed, "K", (B, G, T, d))
    V = gi.normal_bf16(seed, "V", (B, G, T, d))
    dO = gi.normal_bf16(seed, "do", (B, G, T, k, d))
    dOs = gi.normal_bf16(seed, "dosh", (B, T, d))
    return q, qs, K, V, dO, dOs


def _run_attn_bwd(dims, q, qs, K, V, dO, dOs):
    """Forward on the GPU (o, LSE), then the backward call on the same inputs."""
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    sh = bool(dims.n_shared)
    dc = gq.make_dims(dims)
    tq, tqs, tK, tV = bf16_dev(q), bf16_dev(qs) if sh else None, bf16_dev(K), bf16_dev(V)
    o = torch.empty((B, G, T, k, d), dtype=torch.bfloat16, device="cuda")
    os_ = torch.empty((B, T, d), dtype=torch.bfloat16, device="cuda") if sh else None
    lse = torch.empty((B * G * T * k + B * T * dims.n_shared,), dtype=torch.float32, device="cuda")
    gq.gqe_attn_prefill(dc, tq, tqs, tK, tV, o, os_, lse)
    nan = float("nan")
    dq = torch.full_like(o, nan)
    dqs = torch.full_like(os_, nan) if sh else None
    dK = torch.full_like(tK, nan)
    dV = torch.full_like(tV, nan)
    ws = torch.full((gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_BWD) // 4 + 64,), nan, dtype=torch.float32,
                    device="cuda")
    gq.gqe_attn_prefill_bwd(dc, tq, tqs, tK, tV, o, os_, lse, bf16_dev(dO), bf16_dev(dOs) if sh else None,
                            dq, dqs, dK, dV, ws)
    torch.cuda.synchronize()
    return dq, dqs, dK, dV, to_f64(o), to_f64(os_) if sh else None, lse.cpu().numpy().astype(np.float64)


ATTN_BWD_SMALL = {
    "tiny": D(),
    "ragged_k2_sg1": D(B=2, T=200, G=3, E=3, k=2, sg=1),
    "k1_multi_tile": D(B=1, T=520, G=2, E=2, k=1, sg=1),
    "k3_no_shared": D(B=2, T=50, G=1, E=3, k=3, n_shared=0),
    "single_token": D(B=2, T=1, G=2, E=2, k=2),
    "k8_E8": D(B=1, T=70, G=1, E=8, k=8),
    "k4_E8_ragged": D(B=1, T=300, G=2, E=8, k=4),
    "d128_k4_ragged": D(B=1, T=257, G=2, E=4, k=4, d=128),
    "d128_k1_multi_tile_sg1": D(B=2, T=400, G=2, E=2, k=1, d=128, sg=1),
    "d128_no_shared": D(B=1, T=64, G=1, E=3, k=2, d=128, n_shared=0),
}


@pytest.mark.parametrize("case", list(ATTN_BWD_SMALL))
def test_attn_bwd_small(case):
    dims = ATTN_BWD_SMALL[case]
    q, qs, K, V, dO, dOs = _attn_bwd_inputs(dims, 21)
    dq, dqs, dK, dV, o, os_, lse = _run_attn_bwd(dims, q, qs, K, V, dO, dOs)
    # per-call parity: Delta and P from the forward output and LSE the call received
    args = (q, qs if dims.n_shared else None, K, V, dO, dOs if dims.n_shared else None, dims, o, os_, lse)
    r_dq, r_dqs, r_dK, r_dV = ob.attn_prefill_bwd(*args)
    m_dq, m_dqs, m_dK, m_dV = ob.attn_prefill_bwd_error_bound(*args)
    errs = [assert_close_grad(to_f64(dq), r_dq, m_dq, "dq_routed"), assert_close_grad(to_f64(dK), r_dK, m_dK, "dK"),
            assert_close_grad(to_f64(dV), r_dV, m_dV, "dV")]
    if dims.n_shared:
        errs.append(assert_close_grad(to_f64(dqs), r_dqs, m_dqs, "dq_sh"))
    print(f"[attn bwd {case}] err/bound, mean/rms:", [(f"{a:.2f}", f"{b:.2e}") for a, b in errs])


@pytest.mark.parametrize("wname", ["main_prefill", "wide_skewed_prefill"])
def test_attn_bwd_full_size_sampled(wname):
    """Full workload size in the bench's launch configuration; dK, dV and dq of
    two whole KV sequences (one of them the shared head's group) against the
    oracle computed per sequence."""
    dims = gi.WORKLOADS[wname].dims
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    q, qs, K, V, dO, dOs = _attn_bwd_inputs(dims, 22)
    dq, dqs, dK, dV, o, os_, lse = _run_attn_bwd(dims, q, qs, K, V, dO, dOs)
    g_dq, g_dqs, g_dK, g_dV = to_f64(dq), to_f64(dqs), to_f64(dK), to_f64(dV)
    pos = np.repeat(np.arange(T), k)
    R = T * k
    for b, g in [(0, dims.sg), (B - 1, G - 1)]:
        args = (q[b, g].reshape(R, d), pos, K[b, g], V[b, g], dO[b, g].reshape(R, d), orc.attention_scale(dims),
                o[b, g].reshape(R, d), lse[(b * G + g) * R:(b * G + g + 1) * R])
        a, bk, bv = ob.causal_attention_bwd(*args)
        ma, mk, mv = ob.causal_attention_bwd_error_bound(*args)
        if g == dims.sg:
            ls = lse[B * G * R + b * T:B * G * R + (b + 1) * T]
            args2 = (qs[b], np.arange(T), K[b, g], V[b, g], dOs[b], orc.attention_scale(dims), os_[b], ls)
            a2, bk2, bv2 = ob.causal_attention_bwd(*args2)
            ma2, mk2, mv2 = ob.causal_attention_bwd_error_bound(*args2)
            bk, bv, mk, mv = bk + bk2, bv + bv2, mk + mk2, mv + mv2
            assert_close_grad(g_dqs[b], a2, ma2, "dq_sh")
        assert_close_grad(g_dq[b, g].reshape(R, d), a, ma, "dq_routed")
        assert_close_grad(g_dK[b, g], bk, mk, "dK")
        assert_close_grad(g_dV[b, g], bv, mv, "dV")
    for t in (dq, dqs, dK, dV):
        assert torch.isfinite(t.float()).all()


# ----------------------------------------------------------------------------
# output construction and router backward

@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("dims", [D(B=2, T=70, G=3, E=3, k=2), D(B=1, T=64, G=2, E=4, k=2, d=128, n_shared=0)],
                         ids=["d64", "d128_no_shared"])
def test_combine_bwd(dims, mode):
    dims = dims.replace(output_mode=mode)
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    o = gi.normal_bf16(3, "o", (B, G, T, k, d))
    w = gi.random_weights_simplex(dims, 3)
    dh = gi.normal_bf16(3, "dh", (dims.N, dims.slots * d))
    do = torch.full((B, G, T, k, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    dos = torch.full((B, T, d), float("nan"), dtype=torch.bfloat16, device="cuda") if dims.n_shared else None
    dw = torch.full((dims.N, G, k), float("nan"), dtype=torch.float32, device="cuda")
    gq.gqe_combine_bwd(gq.make_dims(dims), bf16_dev(o), None, torch.from_numpy(w).cuda(), bf16_dev(dh), do, dos, dw)
    torch.cuda.synchronize()
    r_do, r_dos, r_dw = ob.combine_bwd(o, None, w, dh, dims)
    # bf16 output of an fp32 combination of at most two terms: half an ulp plus fp32 rounding
    assert np.all(np.abs(to_f64(do) - r_do) <= 2.0 ** -8 * np.abs(r_do) + 1e-6)
    if dims.n_shared:
        assert np.array_equal(to_f64(dos), r_dos)
    # dw: fp32 dot products of d bf16 pairs
    mag = np.abs(orc.f64(dh)).max() * np.abs(orc.f64(o)).max() * d
    np.testing.assert_allclose(dw.cpu().numpy(), r_dw, atol=1e-6 * mag, rtol=1e-5)


@pytest.mark.parametrize("scope", [0, 1, 2])
@pytest.mark.parametrize("dims", [D(B=2, T=100, D=128, G=3, E=4, k=2), D(B=1, T=300, D=128, G=8, E=2, k=1),
                                  D(B=1, T=90, D=128, G=2, E=8, k=8)], ids=["E4k2", "E2k1", "k_eq_E"])
def test_router_bwd(dims, scope):
    dims = dims.replace(renorm_scope=scope)
    N, G, E, k = dims.N, dims.G, dims.E, dims.k
    x = gi.layer_input(dims, 5)
    Wt = gi.layer_weights(dims, 5)
    dc = gq.make_dims(dims)
    idx = torch.empty((N, G, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((N, G, k), dtype=torch.float32, device="cuda")
    probs = torch.empty((N, G, E), dtype=torch.float32, device="cuda")
    gq.gqe_router_topk(dc, bf16_dev(x), bf16_dev(Wt["Wr"]), None, idx, wt, probs)
    rng = np.random.default_rng(6)
    dw = rng.standard_normal((N, G, k)).astype(np.float32)
    dlog = torch.full((N, G * E), float("nan"), dtype=torch.float32, device="cuda")
    dbias = torch.full((G * E,), float("nan"), dtype=torch.float32, device="cuda")
    gq.gqe_router_bwd(dc, probs, idx, wt, torch.from_numpy(dw).cuda(), dlog, dbias)
    torch.cuda.synchronize()
    p = probs.cpu().numpy().astype(np.float64)
    ref = ob.group_softmax_bwd(p, ob.renormalise_bwd(p, idx.cpu().numpy(), dw, scope)).reshape(N, G * E)
    np.testing.assert_allclose(dlog.cpu().numpy(), ref, atol=1e-6, rtol=1e-4)
    np.testing.assert_allclose(dbias.cpu().numpy(), ref.sum(axis=0), atol=1e-4, rtol=1e-4)
    # softmax gradients sum to zero within each group
    assert np.abs(dlog.cpu().numpy().reshape(N, G, E).sum(axis=-1)).max() < 1e-5


# ----------------------------------------------------------------------------
# the whole layer

LAYER_BWD = {
    "k1_E2": D(B=2, T=256, D=256, G=4, E=2, k=1),
    "k2_E4_ragged": D(B=1, T=200, D=192, G=2, E=4, k=2, sg=1),
    "group_scope": D(B=1, T=128, D=128, G=2, E=3, k=2, renorm_scope=1),
    "weighted_concat": D(B=1, T=128, D=128, G=2, E=2, k=1, output_mode=2, renorm_scope=2),
    "hard_concat_no_shared": D(B=1, T=192, D=128, G=2, E=2, k=1, output_mode=1, n_shared=0),
    "d128_k2_E4": D(B=1, T=256, D=256, G=2, E=4, k=2, d=128),
}

# end to end through every bf16 intermediate (o, h, dh, do, dq, dK, dV, A):
# norm-wise relative error of each gradient tensor.  The router's gradients get
# a wider bound: renormalisation subtracts the selected experts' weighted mean
# of dw = <dh, o> (within a group for renorm scope 1), so the bf16 rounding of
# dh and o is amplified where the selected experts' dw are close (measured:
# ~5e-3 at token scope, ~3e-2 at group scope with k = 2; the call itself is
# held to fp32 accuracy in test_router_bwd).
LAYER_BWD_REL = 2e-2
LAYER_BWD_REL_ROUTER = 5e-2


@pytest.mark.parametrize("case", list(LAYER_BWD))
def test_layer_backward_end_to_end(case):
    dims = LAYER_BWD[case]
    x = gi.layer_input(dims, 4)
    Wt = gi.layer_weights(dims, 4)
    rng = np.random.default_rng(8)
    bias = rng.standard_normal(dims.G * dims.E).astype(np.float32)
    dy = gi.normal_bf16(4, "dy", (dims.B, dims.T, dims.D))
    lay = gq.GQELayer(dims, {kk: torch.from_numpy(v.view(np.int16)) for kk, v in Wt.items()}, bias)
    tx = bf16_dev(x)
    y, saved = lay.forward(tx, keep=True)
    g = lay.backward(tx, bf16_dev(dy), saved)
    torch.cuda.synchronize()
    ref = ob.gqe_backward(x, Wt, dims, dy, bias)
    # tokens whose routing is a near-tie may legitimately differ: none expected at these sizes
    r = orc.router_topk(orc.f64(x).reshape(dims.N, -1), Wt["Wr"], dims.G, dims.E, dims.k, bias, dims.renorm_scope)
    assert np.array_equal(saved["idx"].cpu().numpy(), r["idx"])
    rep = {}
    for name in ["dx", "dWr", "dbias", "dWq", "dWk", "dWv", "dWo"] + (["dWsh"] if dims.n_shared else []):
        got = to_f64(g[name]).reshape(ref[name].shape)
        rel = np.linalg.norm(got - ref[name]) / max(np.linalg.norm(ref[name]), 1e-30)
        rep[name] = rel
        if dims.output_mode == 1 and name in ("dWr", "dbias"):
            assert np.abs(got).max() == 0
            continue
        assert rel <= (LAYER_BWD_REL_ROUTER if name in ("dWr", "dbias") else LAYER_BWD_REL), (name, rel)
    print(f"[layer bwd {case}] norm-wise relative errors:", {k_: f"{v:.2e}" for k_, v in rep.items()})


@pytest.mark.parametrize("rows,cols,ld", [(200, 192, 256), (64, 64, 64), (1000, 70, 1000), (3, 130, 64)])
def test_transpose(rows, cols, ld):
    src = gi.normal_bf16(9, "x", (rows, cols))
    dst = torch.full((cols, ld), float("nan"), dtype=torch.bfloat16, device="cuda")
    gq.gqe_transpose(bf16_dev(src), dst, ld)
    torch.cuda.synchronize()
    got = dst.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got[:, :rows], src.T)
    assert not got[:, rows:].any()


@pytest.mark.parametrize("a_kn,b_kn", [(0, 0), (0, 1), (1, 0), (1, 1)])
@pytest.mark.parametrize("M,N,K", [(200, 192, 104), (2304, 512, 1000), (64, 64, 16384), (4096, 256, 72)],
                         ids=["small_ragged_k", "pair_tiles", "long_k", "pair_short_k"])
def test_gemm_operand_layouts(M, N, K, a_kn, b_kn):
    """C = A B^T with each operand stored either way round; the ragged K tail
    (K not a multiple of 64) is zero-filled by the loads.  Projection
    tolerance: 2^-8 |ref| + 1e-3 (bf16 output of an fp32 accumulation), inputs
    scaled to unit-size outputs."""
    A = gi.normal_bf16(10, "x", (M, K), std=K ** -0.5)
    Bm = gi.normal_bf16(11, "x", (N, K))
    tA = bf16_dev(np.ascontiguousarray(A.T) if a_kn else A)
    tB = bf16_dev(np.ascontiguousarray(Bm.T) if b_kn else Bm)
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    gq.gqe_gemm(tA, a_kn, tB, b_kn, C)
    torch.cuda.synchronize()
    ref = orc.f64(A) @ orc.f64(Bm).T
    got = to_f64(C)
    bad = np.abs(got - ref) > 2.0 ** -8 * np.abs(ref) + 1e-3
    assert not bad.any(), (int(bad.sum()), float(np.abs(got - ref).max()))


@pytest.mark.parametrize("K", [70, 1, 16389])
def test_gemm_any_k_when_k_is_strided(K):
    """With both operands stored [K, *] the contiguous dimensions are M and N,
    so any K works (the token count of a weight gradient)."""
    M, N = 320, 128
    A = gi.normal_bf16(12, "x", (K, M), std=K ** -0.5)
    Bm = gi.normal_bf16(13, "x", (K, N))
    C = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
    gq.gqe_gemm(bf16_dev(A), 1, bf16_dev(Bm), 1, C)
    torch.cuda.synchronize()
    ref = orc.f64(A).T @ orc.f64(Bm)
    got = to_f64(C)
    assert not (np.abs(got - ref) > 2.0 ** -8 * np.abs(ref) + 1e-3).any()


def test_gemm_rejects_unaligned_contiguous_k():
    A = torch.zeros((64, 70), dtype=torch.bfloat16, device="cuda")
    Bm = torch.zeros((64, 70), dtype=torch.bfloat16, device="cuda")
    C = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gq.GQEError):
        gq.gqe_gemm(A, 0, Bm, 0, C)


@pytest.mark.parametrize("a_kn,b_kn", [(1, 1), (0, 1), (0, 0)])
@pytest.mark.parametrize("M,N,K", [(1024, 640, 16384), (2176, 1024, 4104), (200, 64, 72)],
                         ids=["dWo_shape", "pair_split", "small"])
def test_gemm_acc_fp32_split_k(M, N, K, a_kn, b_kn):
    """C (fp32) += A B^T with K split over CTAs and fp32 reduce-add: added onto
    the values already in C; error within fp32 accumulation of bf16 products."""
    A = gi.normal_bf16(14, "x", (M, K), std=K ** -0.5)
    Bm = gi.normal_bf16(15, "x", (N, K))
    tA = bf16_dev(np.ascontiguousarray(A.T) if a_kn else A)
    tB = bf16_dev(np.ascontiguousarray(Bm.T) if b_kn else Bm)
    C0 = np.random.default_rng(3).standard_normal((M, N)).astype(np.float32)
    C = torch.from_numpy(C0).cuda()
    gq.gqe_gemm_acc(tA, a_kn, tB, b_kn, C, accumulate=True)
    torch.cuda.synchronize()
    Af, Bf = orc.f64(A), orc.f64(Bm)
    ref = C0.astype(np.float64) + Af @ Bf.T
    bound = K * 2.0 ** -24 * (np.abs(Af) @ np.abs(Bf).T) + 2.0 ** -23 * np.abs(ref) + 1e-6
    got = C.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= bound), float((np.abs(got - ref) / bound).max())


def test_gemm_acc_overwrites_without_accumulate():
    A = gi.normal_bf16(16, "x", (300, 128), std=128 ** -0.5)
    Bm = gi.normal_bf16(17, "x", (192, 128))
    C = torch.full((300, 192), float("nan"), dtype=torch.float32, device="cuda")
    gq.gqe_gemm_acc(bf16_dev(A), 0, bf16_dev(Bm), 0, C)
    torch.cuda.synchronize()
    ref = orc.f64(A) @ orc.f64(Bm).T
    np.testing.assert_allclose(C.cpu().numpy(), ref, rtol=1e-4, atol=1e-4)


# ----------------------------------------------------------------------------
# the packed projection-gradient matrix (layout only: bit-exact)

PACK_CASES = {
    "main_like": D(B=2, T=300, D=128, G=8, E=2, k=1, d=64),
    "wide_k4_d128": D(B=1, T=130, D=128, G=4, E=8, k=4, d=128),
    "E3_k2_no_shared": D(B=2, T=77, D=128, G=3, E=3, k=2, d=64, n_shared=0),
    "GE64": D(B=1, T=70, D=128, G=16, E=4, k=1, d=64),
}


@pytest.mark.parametrize("case", list(PACK_CASES))
def test_bwd_pack_bit_exact(case):
    """A = [dq in its expert's columns (zeros elsewhere) | dq_sh | dK | dV |
    dlogits as bf16 (round to nearest even), zero padding], compared bit for
    bit with the same packing done on the host."""
    dims = PACK_CASES[case]
    B, T, G, E, k, d, N = dims.B, dims.T, dims.G, dims.E, dims.k, dims.d, dims.N
    idx = gi.random_routing(dims, 2)
    rng = np.random.default_rng(9)
    bits = lambda *shape: gi.f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))  # noqa: E731
    dq, dK, dV = bits(B, G, T, k, d), bits(B, G, T, d), bits(B, G, T, d)
    dqs = bits(B, T, d) if dims.n_shared else None
    dl = rng.standard_normal((N, G * E), dtype=np.float32)
    dc = gq.make_dims(dims)
    Kc = gq.gqe_bwd_pack_cols(dc)
    A = torch.full((N, Kc), float("nan"), dtype=torch.bfloat16, device="cuda")
    gq.gqe_bwd_pack(dc, torch.from_numpy(idx).cuda(), bf16_dev(dq), None if dqs is None else bf16_dev(dqs),
                    bf16_dev(dK), bf16_dev(dV), torch.from_numpy(dl).cuda(), A)
    torch.cuda.synchronize()
    want = np.zeros((N, Kc), dtype=np.uint16)
    n = np.arange(N)
    b, t = n // T, n % T
    for g in range(G):
        for j in range(k):
            cols = (g * E + idx[:, g, j])[:, None] * d + np.arange(d)[None, :]
            want[n[:, None], cols] = dq[b, g, t, j]
    c = G * E * d
    if dqs is not None:
        want[:, c:c + d] = dqs.reshape(N, d)
        c += d
    for src in (dK, dV):
        for g in range(G):
            want[:, c + g * d:c + (g + 1) * d] = src[b, g, t]
        c += G * d
    want[:, c:c + G * E] = gi.f32_to_bf16_bits(dl)
    got = A.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)
