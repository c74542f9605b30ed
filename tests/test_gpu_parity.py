"""Parity of every C-ABI call with the fp64 oracle on the same seeded inputs.

Small shapes span several tiles with ragged tails and are compared element by
element; the full workload sizes are compared on sampled rows the oracle
computes one by one.  Tolerances: TopK indices exact except near-ties (logit
margin < 1e-4, counted, the GPU's choice checked valid); router weights 1e-5;
projections 2^-8 |ref| + 1e-3; attention outputs, h and y max-abs 2e-2 and
mean-abs 2e-3.
"""
import numpy as np
import pytest
import torch

import gqe_inputs as gi
import oracle as orc
from helpers import (ATTN_MAX_ABS, NEAR_TIE, W_TOL, assert_close_attn, assert_close_proj, bf16_dev,
                     to_f64)

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


def dims_c(dims, **over):
    return gq.make_dims(dims, **over)


# ----------------------------------------------------------------------------
# router

ROUTER_CASES = {
    "tiny": (gi.WORKLOADS["tiny_prefill"], None),
    "ragged_odd_GE": (gi.Workload("r", D(B=2, T=77, D=128, G=3, E=3, k=2)), None),
    "group_scope": (gi.Workload("g", D(B=1, T=200, D=192, G=4, E=4, k=2, renorm_scope=1)), None),
    "main": (gi.WORKLOADS["main_prefill"], None),
    "long": (gi.WORKLOADS["long_prefill"], None),
    "wide_skewed": (gi.WORKLOADS["wide_skewed_prefill"], None),
    "no_renorm": (gi.Workload("n0", D(B=1, T=90, D=128, G=2, E=4, k=2, renorm_scope=2)), None),
    "tc_no_renorm": (gi.Workload("n1", D(B=1, T=1500, D=128, G=8, E=2, k=1, renorm_scope=2)), None),
    # 1024 tokens and more take the tcgen05 router: generic E, group scope, ragged last tile
    "tc_E3_group_scope": (gi.Workload("t3", D(B=2, T=640, D=256, G=5, E=3, k=2, renorm_scope=1)), None),
    "tc_E8_k4_ragged": (gi.Workload("t8", D(B=1, T=1100, D=192, G=4, E=8, k=4)), None),
    "tc_E4_GE64": (gi.Workload("t4", D(B=1, T=1536, D=128, G=16, E=4, k=1)), None),
    # the tcgen05 router with Wr read in place at larger d_model
    "tc_K_chunked_GE64": (gi.Workload("tk", D(B=1, T=1100, D=1024, G=8, E=8, k=2)), None),
    "tc_K_chunked_group_scope": (gi.Workload("tg", D(B=2, T=600, D=2048, G=4, E=8, k=3, renorm_scope=1)), None),
    # Wr too large to keep in shared memory and fewer than 1024 tokens (no
    # tcgen05 router): the streaming CUDA-core router, ragged last tile
    "stream_D4096_N500": (gi.Workload("s1", D(B=1, T=500, D=4096, G=4, E=8, k=3)), None),
}


def check_router(w: gi.Workload, seed=0):
    dims = w.dims
    x = gi.layer_input(dims, seed)
    Wt = gi.layer_weights(dims, seed)
    bias = gi.router_bias(w, seed)
    N, G, E, k = dims.N, dims.G, dims.E, dims.k
    idx = torch.empty((N, G, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((N, G, k), dtype=torch.float32, device="cuda")
    probs = torch.empty((N, G, E), dtype=torch.float32, device="cuda")
    gq.gqe_router_topk(dims_c(dims), bf16_dev(x), bf16_dev(Wt["Wr"]),
                       None if bias is None else torch.from_numpy(bias).cuda(), idx, wt, probs)
    torch.cuda.synchronize()
    r = orc.router_topk(orc.f64(x).reshape(N, -1), Wt["Wr"], G, E, k, bias, dims.renorm_scope)
    gi_idx = idx.cpu().numpy()
    tie = r["margin"] < NEAR_TIE
    same = np.all(gi_idx == r["idx"], axis=-1)
    assert np.all(same | tie), f"{int((~same & ~tie).sum())} routing decisions differ outside near-ties"
    # near-ties: the GPU's set must contain every sure expert and only undecided others
    for (t, g), (sure, undecided) in orc.near_tie_alternatives(r, k).items():
        chosen = set(gi_idx[t, g].tolist())
        assert set(sure.tolist()) <= chosen and chosen <= set(sure.tolist()) | set(undecided.tolist())
    assert np.all(np.diff(gi_idx, axis=-1) > 0) if k > 1 else True
    np.testing.assert_allclose(probs.cpu().numpy(), r["probs"], atol=W_TOL)
    tok_ok = ~tie.any(axis=1)
    np.testing.assert_allclose(wt.cpu().numpy()[tok_ok], r["w"][tok_ok], atol=W_TOL)
    return int(tie.sum())


@pytest.mark.parametrize("wname", ["main_prefill", "wide_skewed_prefill"])
def test_router_stats(wname):
    """Per-(group, expert) selection counts (exact) and probability sums
    against the oracle; the skewed workload's expert-0 share shows in both."""
    w = gi.WORKLOADS[wname]
    dims = w.dims
    x = gi.layer_input(dims, 0)
    Wt = gi.layer_weights(dims, 0)
    bias = gi.router_bias(w, 0)
    N, G, E, k = dims.N, dims.G, dims.E, dims.k
    idx = torch.empty((N, G, k), dtype=torch.int32, device="cuda")
    wt = torch.empty((N, G, k), dtype=torch.float32, device="cuda")
    probs = torch.empty((N, G, E), dtype=torch.float32, device="cuda")
    dc = dims_c(dims)
    gq.gqe_router_topk(dc, bf16_dev(x), bf16_dev(Wt["Wr"]), None if bias is None else torch.from_numpy(bias).cuda(),
                       idx, wt, probs)
    counts = torch.full((G * E,), -1, dtype=torch.int32, device="cuda")
    psum = torch.full((G * E,), float("nan"), dtype=torch.float32, device="cuda")
    gq.gqe_router_stats(dc, probs, idx, counts, psum)
    torch.cuda.synchronize()
    c_ref, p_ref = orc.router_stats(probs.cpu().numpy(), idx.cpu().numpy(), G, E)
    np.testing.assert_array_equal(counts.cpu().numpy(), c_ref)
    np.testing.assert_allclose(psum.cpu().numpy(), p_ref, rtol=1e-4)
    assert np.all(counts.cpu().numpy().reshape(G, E).sum(axis=1) == N * k)


@pytest.mark.parametrize("case", list(ROUTER_CASES))
def test_router_topk(case):
    w, _ = ROUTER_CASES[case]
    n_ties = check_router(w)
    print(f"[router {case}] near-ties: {n_ties}")


# ----------------------------------------------------------------------------
# routed + shared query projection

QPROJ_CASES = {
    "tiny": (gi.WORKLOADS["tiny_prefill"].dims, 0.0, None),
    "ragged_k2": (D(B=2, T=77, D=128, G=3, E=4, k=2), 0.0, None),
    "wide_k4_skew_d128": (D(B=1, T=300, D=256, G=2, E=8, k=4, d=128), 0.8, None),
    "no_shared": (D(B=1, T=129, D=64, G=2, E=3, k=1, n_shared=0), 0.0, None),
    "main": (gi.WORKLOADS["main_prefill"].dims, 0.0, None),
    "wide_skewed_sampled": (gi.WORKLOADS["wide_skewed_prefill"].dims, 0.8, 96),
}


@pytest.mark.parametrize("case", list(QPROJ_CASES))
def test_routed_qproj(case):
    dims, skew, n_sample = QPROJ_CASES[case]
    x = gi.layer_input(dims, 1)
    Wt = gi.layer_weights(dims, 1)
    idx = gi.random_routing(dims, 1, skew0=skew)
    N, G, k, d = dims.N, dims.G, dims.k, dims.d
    q = torch.empty((dims.B, G, dims.T, k, d), dtype=torch.bfloat16, device="cuda")
    qs = torch.empty((dims.B, dims.T, d), dtype=torch.bfloat16, device="cuda") if dims.n_shared else None
    cnt = torch.empty((G * dims.E,), dtype=torch.int32, device="cuda")
    dc = dims_c(dims)
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_ROUTED_QPROJ),), dtype=torch.uint8, device="cuda")
    gq.gqe_routed_qproj(dc, bf16_dev(x), bf16_dev(Wt["Wq"]), bf16_dev(Wt["Wsh"]) if dims.n_shared else None,
                        torch.from_numpy(idx).cuda(), q, qs, ws, cnt)
    torch.cuda.synchronize()
    hist = np.bincount((np.arange(G)[None, :, None] * dims.E + idx).reshape(-1), minlength=G * dims.E)
    assert np.array_equal(cnt.cpu().numpy(), hist)
    xf = orc.f64(x).reshape(N, -1)
    rows = np.arange(N) if n_sample is None else np.sort(np.random.default_rng(5).choice(N, n_sample, replace=False))
    sub = gi.GQEDims(B=1, T=len(rows), D=dims.D, G=G, E=dims.E, k=k, d=d, n_shared=dims.n_shared)
    q_ref, qs_ref = orc.routed_qproj(xf[rows], Wt["Wq"], Wt["Wsh"], idx[rows], sub)
    q_gpu = to_f64(q).transpose(0, 2, 1, 3, 4).reshape(N, G, k, d)[rows]
    assert_close_proj(q_gpu, q_ref[0].transpose(1, 0, 2, 3), "q_routed")
    if dims.n_shared:
        assert_close_proj(to_f64(qs).reshape(N, d)[rows], qs_ref[0], "q_sh")


# ----------------------------------------------------------------------------
# dense K/V projection, output projection

@pytest.mark.parametrize("dims", [gi.WORKLOADS["tiny_prefill"].dims, D(B=2, T=77, D=128, G=3, E=2, k=1),
                                  D(B=1, T=130, D=192, G=1, E=2, k=1, d=128),
                                  D(B=3, T=700, D=256, G=4, E=2, k=1),
                                  gi.WORKLOADS["main_prefill"].dims],
                         ids=["tiny", "ragged_G3", "G1_d128", "pair_ragged_M", "main"])
def test_kv_proj(dims):
    x = gi.layer_input(dims, 2)
    Wt = gi.layer_weights(dims, 2)
    K = torch.empty((dims.B, dims.G, dims.T, dims.d), dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    gq.gqe_kv_proj(dims_c(dims), bf16_dev(x), bf16_dev(Wt["Wk"]), bf16_dev(Wt["Wv"]), K, V)
    torch.cuda.synchronize()
    K_ref, V_ref = orc.kv_proj(orc.f64(x).reshape(dims.N, -1), Wt["Wk"], Wt["Wv"], dims)
    assert_close_proj(to_f64(K), K_ref, "K")
    assert_close_proj(to_f64(V), V_ref, "V")


@pytest.mark.parametrize("M,N,K", [(200, 192, 320), (16, 64, 64), (1000, 256, 640), (2125, 512, 192),
                                   (4133, 768, 1024), (16384, 1024, 640)])
def test_linear(M, N, K):
    rng_dims = gi.GQEDims(B=1, T=M, D=K, G=1, E=1, k=1, d=64)
    A = gi.normal_bf16(3, "x", (M, K), 1.0)
    W = gi.normal_bf16(3, "Wo", (N, K), 0.02)
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    gq.gqe_linear(bf16_dev(A), bf16_dev(W), C)
    torch.cuda.synchronize()
    assert_close_proj(to_f64(C), orc.linear(A, W), "linear")
    del rng_dims


# ----------------------------------------------------------------------------
# routed causal attention (prefill)

def _attn_inputs(dims, seed):
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    q = gi.normal_bf16(seed, "q", (B, G, T, k, d))
    qs = gi.normal_bf16(seed, "qsh", (B, T, d))
    K = gi.normal_bf16(seed, "K", (B, G, T, d))
    V = gi.normal_bf16(seed, "V", (B, G, T, d))
    return q, qs, K, V


def _run_prefill(dims, q, qs, K, V, want_lse=True):
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    o = torch.full((B, G, T, k, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    os_ = torch.full((B, T, d), float("nan"), dtype=torch.bfloat16, device="cuda") if dims.n_shared else None
    lse = torch.empty((B * G * T * k + B * T * dims.n_shared,), dtype=torch.float32, device="cuda") if want_lse else None
    gq.gqe_attn_prefill(dims_c(dims), bf16_dev(q), bf16_dev(qs) if dims.n_shared else None, bf16_dev(K),
                        bf16_dev(V), o, os_, lse)
    torch.cuda.synchronize()
    return o, os_, lse


PREFILL_SMALL = {
    "tiny": D(),
    "ragged_k2_sg1": D(B=2, T=300, G=3, E=2, k=2, sg=1),
    "k4_d128_ragged": D(B=1, T=257, G=2, E=4, k=4, d=128),
    "single_token": D(B=2, T=1, G=2, E=2, k=2),
    "k3_no_shared": D(B=2, T=50, G=1, E=3, k=3, n_shared=0),
    "k1_d128_multi_tile": D(B=1, T=520, G=2, E=2, k=1, d=128, sg=1),
    "k8_E8": D(B=1, T=70, G=1, E=8, k=8),
}


@pytest.mark.parametrize("case", list(PREFILL_SMALL))
def test_attn_prefill_small(case):
    dims = PREFILL_SMALL[case]
    q, qs, K, V = _attn_inputs(dims, 7)
    o, os_, lse = _run_prefill(dims, q, qs, K, V)
    o_ref, os_ref, lse_ref, lsesh_ref = orc.attn_prefill(q, qs, K, V, dims)
    assert_close_attn(to_f64(o), o_ref, "o_routed")
    n_r = dims.B * dims.G * dims.T * dims.k
    np.testing.assert_allclose(lse.cpu().numpy()[:n_r], lse_ref.reshape(-1), atol=2e-3, rtol=1e-3)
    if dims.n_shared:
        assert_close_attn(to_f64(os_), os_ref, "o_sh")
        np.testing.assert_allclose(lse.cpu().numpy()[n_r:], lsesh_ref.reshape(-1), atol=2e-3, rtol=1e-3)


def test_attn_prefill_constant_keys_prefix_mean():
    """At any size: equal keys give the causal prefix mean of V."""
    dims = D(B=1, T=1000, G=2, E=2, k=2, d=64)
    q, qs, _, V = _attn_inputs(dims, 8)
    K = np.broadcast_to(gi.normal_bf16(8, "K", (1, 2, 1, 64)), (1, 2, 1000, 64)).copy()
    o, os_, _ = _run_prefill(dims, q, qs, K, V, want_lse=False)
    Vf = orc.f64(V)
    pm = np.cumsum(Vf, axis=2) / np.arange(1, 1001)[None, None, :, None]
    assert_close_attn(to_f64(o), np.repeat(pm[:, :, :, None, :], 2, axis=3), "prefix mean")
    assert_close_attn(to_f64(os_), pm[:, 0], "prefix mean shared")


@pytest.mark.parametrize("d", [64, 128])
def test_attn_prefill_growing_scores(d):
    """Keys whose norm grows along the sequence: later key tiles raise the
    running row maximum far past the lazy-rescale margin, so the rescale of
    P, the row sum and O is exercised on most rows."""
    dims = D(B=1, T=700, G=2, E=2, k=2, d=d)
    q, qs, K, V = _attn_inputs(dims, 12)
    growth = (1.0 + np.arange(dims.T) / 24.0)[None, None, :, None]
    K = gi.f32_to_bf16_bits((gi.bf16_bits_to_f32(K) * growth).astype(np.float32))
    # the softmax becomes nearly one-hot, so o is close to single V rows: V at a
    # quarter scale keeps |o| where bf16 rounding of o stays inside the tolerance
    V = gi.f32_to_bf16_bits((gi.bf16_bits_to_f32(V) * 0.25).astype(np.float32))
    o, os_, lse = _run_prefill(dims, q, qs, K, V)
    o_ref, os_ref, lse_ref, lsesh_ref = orc.attn_prefill(q, qs, K, V, dims)
    assert_close_attn(to_f64(o), o_ref, "o_routed")
    assert_close_attn(to_f64(os_), os_ref, "o_sh")
    n_r = dims.B * dims.G * dims.T * dims.k
    np.testing.assert_allclose(lse.cpu().numpy()[:n_r], lse_ref.reshape(-1), atol=2e-2, rtol=1e-3)


def _boundary_rows(T, extra, rng, B, G):
    """Sampled (b, g, t) rows: t = 0, T-1 and both sides of every 128-row tile
    boundary of one sequence, plus `extra` random rows anywhere."""
    b0, g0 = int(rng.integers(B)), int(rng.integers(G))
    ts = sorted({0, T - 1} | {t for m in range(1, (T + 127) // 128) for t in (128 * m - 1, 128 * m) if t < T})
    picks = [(b0, g0, t) for t in ts]
    picks += [(int(rng.integers(B)), int(rng.integers(G)), int(rng.integers(T))) for _ in range(extra)]
    return picks


@pytest.mark.parametrize("wname,growth", [("main_prefill", 0.0), ("long_prefill", 0.0), ("wide_skewed_prefill", 0.0),
                                          ("long_prefill", 1.0 / 2048)],
                         ids=["main", "long", "wide_skewed", "long_growing_keys"])
def test_attn_prefill_full_size_sampled(wname, growth):
    """Full workload size, bench launch configuration; at least 256 sampled
    rows (every tile boundary of one sequence, t = 0 and T-1, random rows) of
    the routed and shared heads against the oracle, max-abs and mean-abs.
    With growing key norms the running row maximum keeps rising along the
    sequence, so late rows come after many rescales of O and the row sum."""
    dims = gi.WORKLOADS[wname].dims
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    q, qs, K, V = _attn_inputs(dims, 9)
    if growth:
        gr = (1.0 + np.arange(T) * growth)[None, None, :, None]
        K = gi.f32_to_bf16_bits((gi.bf16_bits_to_f32(K) * gr).astype(np.float32))
        V = gi.f32_to_bf16_bits((gi.bf16_bits_to_f32(V) * 0.25).astype(np.float32))
    o, os_, lse = _run_prefill(dims, q, qs, K, V)
    rng = np.random.default_rng(11)
    picks = _boundary_rows(T, max(64, 256 - 2 * (T // 128)), rng, B, G)
    assert len(picks) >= 256
    got = to_f64(o)
    sc = orc.attention_scale(dims)
    g_rows, r_rows = [], []
    for b, g, t in picks:
        r_rows.append(orc.causal_attention(q[b, g, t], np.full(k, t), K[b, g, :t + 1], V[b, g, :t + 1], sc))
        g_rows.append(got[b, g, t])
    assert_close_attn(np.stack(g_rows), np.stack(r_rows), f"{wname} routed rows")
    gsh = to_f64(os_)
    g_rows, r_rows = [], []
    for b, _, t in picks:
        r_rows.append(orc.causal_attention(qs[b, t][None], np.array([t]), K[b, dims.sg, :t + 1],
                                           V[b, dims.sg, :t + 1], sc)[0])
        g_rows.append(gsh[b, t])
    assert_close_attn(np.stack(g_rows), np.stack(r_rows), f"{wname} shared rows")
    assert torch.isfinite(o.float()).all() and torch.isfinite(os_.float()).all()


# ----------------------------------------------------------------------------
# decode attention

def _run_decode(dims, L_max, lens, seed, rows=None, ws_fill=None):
    B, G, k, d = dims.B, dims.G, dims.k, dims.d
    q = gi.normal_bf16(seed, "q", (B, G, k, d))
    qs = gi.normal_bf16(seed, "qsh", (B, d))
    dev_K = torch.empty((B, G, L_max, d), dtype=torch.bfloat16, device="cuda")
    dev_V = torch.empty_like(dev_K)
    host = {}
    gen_rows = range(B) if rows is None else rows
    if rows is not None:
        g_ = torch.Generator(device="cuda").manual_seed(seed)
        dev_K.normal_(generator=g_)
        dev_V.normal_(generator=g_)
    for b in gen_rows:
        Kb = gi.normal_bf16(seed, "Kc", (B, G, L_max, d), rows=[b])[0]
        Vb = gi.normal_bf16(seed, "Vc", (B, G, L_max, d), rows=[b])[0]
        dev_K[b] = bf16_dev(Kb)
        dev_V[b] = bf16_dev(Vb)
        host[b] = (Kb, Vb)
    dc = dims_c(dims)
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_DECODE, L_max),), dtype=torch.uint8, device="cuda")
    if ws_fill is not None:
        ws.view(torch.float32).fill_(ws_fill)
    o = torch.full((B, G, k, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    os_ = torch.full((B, d), float("nan"), dtype=torch.bfloat16, device="cuda") if dims.n_shared else None
    cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    gq.gqe_attn_decode(dc, bf16_dev(q), bf16_dev(qs) if dims.n_shared else None, dev_K, dev_V, L_max, cl, o, os_, ws)
    torch.cuda.synchronize()
    return q, qs, host, to_f64(o), (to_f64(os_) if dims.n_shared else None)


@pytest.mark.parametrize("case", [
    dict(dims=D(B=3, T=1, G=2, E=2, k=2, d=64), L=300, lens=[300, 1, 150]),
    dict(dims=D(B=2, T=1, G=2, E=2, k=1, d=64), L=40000, lens=[40000, 3000], nan_ws=True),
    dict(dims=D(B=2, T=1, G=3, E=4, k=3, d=128, sg=2), L=257, lens=[257, 64]),
    dict(dims=D(B=2, T=1, G=2, E=2, k=1, d=64, n_shared=0), L=4096, lens=[4096, 4000]),
    dict(dims=D(B=1, T=1, G=1, E=8, k=8, d=64), L=1000, lens=[999]),
], ids=["ragged", "short_len_nan_scratch", "d128_sg2", "no_shared_long", "k8"])
def test_attn_decode_small(case):
    dims, L_max, lens = case["dims"], case["L"], case["lens"]
    q, qs, host, o, os_ = _run_decode(dims, L_max, lens, 21, ws_fill=float("nan") if case.get("nan_ws") else None)
    for b in range(dims.B):
        n = lens[b]
        Kb, Vb = host[b]
        for g in range(dims.G):
            ref = orc.causal_attention(q[b, g], np.full(dims.k, n - 1), Kb[g, :n], Vb[g, :n], orc.attention_scale(dims))
            assert_close_attn(o[b, g], ref, f"decode b{b} g{g}")
        if dims.n_shared:
            ref = orc.causal_attention(qs[b][None], np.array([n - 1]), Kb[dims.sg, :n], Vb[dims.sg, :n],
                                       orc.attention_scale(dims))[0]
            assert_close_attn(os_[b], ref, f"decode shared b{b}")


def test_attn_decode_cache_len_out_of_range_is_flagged():
    """cache_len values outside [1, L_max] are a caller error the kernel
    detects without faulting: it records code 0x302 in the device error word
    and clamps, so a length above L_max attends to the whole cache and a
    length of 0 gives zeros."""
    dims = D(B=2, T=1, G=2, E=2, k=1, d=64)
    L_max = 500
    q, qs, host, o, os_ = _run_decode(dims, L_max, [L_max + 7, 0], 23)
    assert gq.gqe_device_error() == 0x302
    Kb, Vb = host[0]
    for g in range(dims.G):
        ref = orc.causal_attention(q[0, g], np.full(dims.k, L_max - 1), Kb[g], Vb[g], orc.attention_scale(dims))
        assert_close_attn(o[0, g], ref, f"clamped to L_max, g{g}")
    assert np.all(o[1] == 0) and np.all(os_[1] == 0)


def test_attn_decode_full_size_sampled():
    """The decode workload (64 x 8 x 32768 x 64 cache): sampled sequences vs the oracle."""
    w = gi.WORKLOADS["decode"]
    dims, L_max = w.dims, w.L
    rows = [0, 37, 63]
    q, qs, host, o, os_ = _run_decode(dims, L_max, [L_max] * dims.B, 31, rows=rows)
    for b in rows:
        Kb, Vb = host[b]
        for g in range(dims.G):
            ref = orc.causal_attention(q[b, g], np.full(dims.k, L_max - 1), Kb[g], Vb[g], orc.attention_scale(dims))
            assert_close_attn(o[b, g], ref, f"decode b{b} g{g}")
        ref = orc.causal_attention(qs[b][None], np.array([L_max - 1]), Kb[dims.sg], Vb[dims.sg], orc.attention_scale(dims))[0]
        assert_close_attn(os_[b], ref, f"decode shared b{b}")
    assert np.isfinite(o).all()


# ----------------------------------------------------------------------------
# output construction

@pytest.mark.parametrize("dims", [D(), D(B=2, T=33, G=3, E=4, k=2, d=128), D(B=1, T=10, G=2, E=2, k=1, n_shared=0),
                                  gi.WORKLOADS["main_prefill"].dims], ids=["tiny", "k2_d128", "no_shared", "main"])
def test_combine(dims):
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    o = gi.normal_bf16(4, "o", (B, G, T, k, d))
    osh = gi.normal_bf16(4, "osh", (B, T, d))
    w = gi.random_weights_simplex(dims, 4)
    h = torch.full((dims.N, dims.slots * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    gq.gqe_combine(dims_c(dims), bf16_dev(o), bf16_dev(osh) if dims.n_shared else None,
                   torch.from_numpy(w).cuda(), h)
    torch.cuda.synchronize()
    ref = orc.combine(o, osh, w.astype(np.float64), dims)
    got = to_f64(h)
    hard = G * k * d
    assert np.array_equal(got[:, :hard], ref[:, :hard])                       # copies: exact
    if dims.n_shared:
        assert np.array_equal(got[:, hard + d:], ref[:, hard + d:])
    np.testing.assert_allclose(got[:, hard:hard + d], ref[:, hard:hard + d], rtol=2 ** -8, atol=1e-6)


@pytest.mark.parametrize("dims", [gi.WORKLOADS["main_prefill"].dims,
                                  D(B=2, T=1024, D=512, G=3, E=4, k=2, n_shared=0),
                                  D(B=1, T=2048, D=256, G=2, E=2, k=1, d=128),
                                  D(B=3, T=896, D=256, G=4, E=2, k=1, sg=2),
                                  D(B=2, T=77, D=128, G=3, E=2, k=1)],
                         ids=["main_direct", "k2_no_shared_direct", "d128_direct", "B3_ragged_pair_direct",
                              "T77_through_h"])
def test_combine_out_proj(dims):
    """Output construction + projection in one call, against the oracle's
    h = combine(o, o_sh, w) and y = h Wo^T (h is never written when T % 128 == 0)."""
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    o = gi.normal_bf16(6, "o", (B, G, T, k, d))
    osh = gi.normal_bf16(6, "osh", (B, T, d))
    w = gi.random_weights_simplex(dims, 6)
    Wo = gi.normal_bf16(6, "Wo", (dims.D, dims.slots * d), 0.02)
    y = torch.full((dims.N, dims.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    dc = dims_c(dims)
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_COMBINE_OUT_PROJ),), dtype=torch.uint8, device="cuda")
    gq.gqe_combine_out_proj(dc, bf16_dev(o), bf16_dev(osh) if dims.n_shared else None,
                            torch.from_numpy(w).cuda(), bf16_dev(Wo), y, ws)
    torch.cuda.synchronize()
    # y carries the bf16 rounding of the weighted-sum slot (as h does) and of y
    # itself: the layer-output tolerance applies, not the single-GEMM one
    h_ref = orc.combine(o, osh, w.astype(np.float64), dims)
    assert_close_attn(to_f64(y), orc.out_proj(h_ref, Wo), "y")
    # the same MMAs over the same bf16 operands as building h and projecting it
    h = torch.empty((dims.N, dims.slots * d), dtype=torch.bfloat16, device="cuda")
    gq.gqe_combine(dc, bf16_dev(o), bf16_dev(osh) if dims.n_shared else None, torch.from_numpy(w).cuda(), h)
    y2 = torch.empty_like(y)
    gq.gqe_linear(h, bf16_dev(Wo), y2)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)


@pytest.mark.parametrize("mode", [1, 2])
@pytest.mark.parametrize("dims", [D(B=2, T=33, G=3, E=4, k=2, d=128), D(B=1, T=256, G=4, E=2, k=1, n_shared=0),
                                  D(B=1, T=2048, D=512, G=4, E=2, k=1)],
                         ids=["k2_d128", "no_shared_T256", "T2048_direct"])
def test_output_modes(dims, mode):
    """The ablation output constructions: h from gqe_combine and y from
    gqe_combine_out_proj (which reads the hard slots in place for mode 1 when
    T % 128 == 0) against the oracle."""
    dims = dims.replace(output_mode=mode)
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    o = gi.normal_bf16(13, "o", (B, G, T, k, d))
    osh = gi.normal_bf16(13, "osh", (B, T, d))
    w = gi.random_weights_simplex(dims, 13)
    dc = dims_c(dims)
    wt = torch.from_numpy(w).cuda()
    osh_d = bf16_dev(osh) if dims.n_shared else None
    h = torch.full((dims.N, dims.slots * d), float("nan"), dtype=torch.bfloat16, device="cuda")
    gq.gqe_combine(dc, bf16_dev(o), osh_d, wt, h)
    Wo = gi.normal_bf16(13, "Wo", (dims.D, dims.slots * d), 0.02)
    y = torch.full((dims.N, dims.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_COMBINE_OUT_PROJ),), dtype=torch.uint8, device="cuda")
    gq.gqe_combine_out_proj(dc, bf16_dev(o), osh_d, wt, bf16_dev(Wo), y, ws)
    torch.cuda.synchronize()
    h_ref = orc.combine(o, osh, w.astype(np.float64), dims)
    got = to_f64(h)
    if mode == 1:
        assert np.array_equal(got, h_ref)                  # copies: exact
    else:
        np.testing.assert_allclose(got, h_ref, rtol=2 ** -8, atol=1e-6)
    assert_close_attn(to_f64(y), orc.out_proj(h_ref, Wo), "y")


# ----------------------------------------------------------------------------
# whole layer

def _layer(w: gi.Workload, seed=0):
    dims = w.dims
    x = gi.layer_input(dims, seed)
    Wt = gi.layer_weights(dims, seed)
    bias = gi.router_bias(w, seed)
    layer = gq.GQELayer(dims, {k_: torch.from_numpy(v.view(np.int16)) for k_, v in Wt.items()}, bias)
    return dims, x, Wt, bias, layer


def test_layer_dense_gqa_mode():
    """k = E with no shared head is dense GQA through the same kernels: every
    query head of every group is computed, and the hard slots of h are the GQA
    heads in order g*E + e (the oracle reduces to dense GQA there, pinned on
    the CPU); y against the oracle layer."""
    dims = D(B=2, T=300, D=256, G=4, E=2, k=2, n_shared=0)
    w = gi.Workload("dense_gqa", dims)
    dims, x, Wt, bias, layer = _layer(w, seed=8)
    y, inter = layer.forward(bf16_dev(x), keep=True)
    torch.cuda.synchronize()
    ref = orc.gqe_forward(x, Wt, dims, bias)
    assert np.array_equal(inter["idx"].cpu().numpy(), np.broadcast_to(np.arange(2), (dims.N, 4, 2)))
    assert_close_attn(to_f64(y).reshape(dims.N, -1), ref["y"], "y")
    assert_close_attn(to_f64(inter["h"]), ref["h"], "h")


@pytest.mark.parametrize("mode,scope", [(1, 0), (2, 2)], ids=["hard_concat", "weighted_concat_no_renorm"])
def test_layer_ablation_modes(mode, scope):
    """The two ablation layers of the accuracy table end to end."""
    dims = D(B=2, T=256, D=256, G=4, E=2, k=1, n_shared=0, renorm_scope=scope, output_mode=mode)
    w = gi.Workload("ablation", dims)
    dims, x, Wt, bias, layer = _layer(w, seed=9)
    y, inter = layer.forward(bf16_dev(x), keep=True)
    torch.cuda.synchronize()
    ref = orc.gqe_forward(x, Wt, dims, bias)
    r = ref["router"]
    tie_tok = (r["margin"] < NEAR_TIE).any(axis=1)
    agree = np.all(inter["idx"].cpu().numpy() == r["idx"], axis=(1, 2))
    assert np.all(agree | tie_tok)
    assert_close_attn(to_f64(y).reshape(dims.N, -1)[agree], ref["y"][agree], "y")
    assert_close_attn(to_f64(inter["h"])[agree], ref["h"][agree], "h")


def test_layer_decode_step_end_to_end():
    w = gi.Workload("dec_small", D(B=4, T=1, D=256, G=2, E=4, k=2, d=64), decode=True, L=700)
    dims = w.dims
    x = gi.normal_bf16(0, "xdec", (dims.B, dims.D))
    Wt = gi.layer_weights(dims, 0)
    layer = gq.GQELayer(dims, {k_: torch.from_numpy(v.view(np.int16)) for k_, v in Wt.items()})
    L_max = 700
    lens = np.array([700, 1, 333, 512])
    Kc = gi.normal_bf16(0, "Kc", (dims.B, dims.G, L_max, dims.d))
    Vc = gi.normal_bf16(0, "Vc", (dims.B, dims.G, L_max, dims.d))
    dK, dV = bf16_dev(Kc), bf16_dev(Vc)
    y, inter = layer.decode_step(bf16_dev(x), dK, dV, torch.from_numpy(lens.astype(np.int32)).cuda(), keep=True)
    torch.cuda.synchronize()
    ref = orc.decode_step(x, Wt, Kc, Vc, lens, dims)
    # the cache rows written by the step
    for b in range(dims.B):
        assert_close_attn(to_f64(dK[b, :, lens[b] - 1]), ref["Knew"][b, :, 0], "K append")
    gi_idx = inter["idx"].cpu().numpy()
    agree = np.all(gi_idx == ref["router"]["idx"], axis=(1, 2))
    assert np.all(agree | (ref["router"]["margin"] < NEAR_TIE).any(axis=1))
    assert_close_attn(to_f64(y)[agree], ref["y"][agree], "decode y")


# ----------------------------------------------------------------------------
# the exponential helpers of the attention kernel

def test_device_exp2_helpers():
    xs = np.concatenate([np.linspace(-120, 20, 20001), np.linspace(-1, 1, 4001)]).astype(np.float32)
    x = torch.from_numpy(xs).cuda()
    yp, y2, yh = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
    gq.gqe_debug_exp2(x, yp, y2, yh)
    torch.cuda.synchronize()
    ref = np.exp2(xs.astype(np.float64))
    rel_poly = np.abs(yp.cpu().numpy() - ref) / ref
    rel_hw = np.abs(yh.cpu().numpy() - ref) / ref
    assert rel_poly.max() < 1e-4, rel_poly.max()
    assert rel_hw.max() < 1e-5, rel_hw.max()
    assert torch.equal(yp, y2)
    ninf = torch.tensor([-float("inf"), -500.0], device="cuda")
    a, b, c = torch.empty_like(ninf), torch.empty_like(ninf), torch.empty_like(ninf)
    gq.gqe_debug_exp2(ninf, a, b, c)
    torch.cuda.synchronize()
    assert (a.cpu() < 2.0 ** -124).all() and (a.cpu() > 0).all()
    assert c.cpu()[0] == 0


def test_layer_graph_replay_matches_eager():
    w = gi.WORKLOADS["tiny_prefill"]
    dims, x, Wt, bias, layer = _layer(w, seed=3)
    xd = bf16_dev(x)
    y_eager = layer.forward(xd).clone()
    y_graph = layer.forward_graph(xd).clone()
    y_graph2 = layer.forward_graph(xd).clone()
    torch.cuda.synchronize()
    assert torch.equal(y_eager, y_graph) and torch.equal(y_graph, y_graph2)
    x_pin = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    y_pin = torch.empty((dims.B, dims.T, dims.D), dtype=torch.bfloat16).pin_memory()
    layer.forward_host(x_pin, y_pin)
    torch.cuda.synchronize()
    assert torch.equal(y_pin, y_eager.cpu())


def test_layer_concurrent_kv_matches_sequential():
    """The K/V projection on a side stream gives the same bits as the calls in
    sequence on one stream."""
    w = gi.WORKLOADS["main_prefill"]
    dims, x, Wt, bias, layer = _layer(w, seed=5)
    xd = bf16_dev(x)
    layer.concurrent_kv = False
    y_seq = layer.forward(xd).clone()
    layer.concurrent_kv = True
    y_con = layer.forward(xd).clone()
    torch.cuda.synchronize()
    assert torch.equal(y_seq, y_con)


def test_layer_host_pipeline_matches_eager():
    """Five batches through the three-stream host pipeline: each output equals
    the eager forward of its own input (no slot reuse races)."""
    w = gi.WORKLOADS["tiny_prefill"]
    dims, x, Wt, bias, layer = _layer(w, seed=4)
    xs = [gi.layer_input(dims, seed=10 + i) for i in range(5)]
    x_pins = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for a in xs]
    y_pins = [torch.full((dims.B, dims.T, dims.D), float("nan"), dtype=torch.bfloat16).pin_memory() for _ in xs]
    layer.forward_host_pipelined(x_pins, y_pins)
    torch.cuda.synchronize()
    for a, yp in zip(xs, y_pins):
        y_ref = layer.forward(bf16_dev(a)).clone()
        torch.cuda.synchronize()
        assert torch.equal(yp, y_ref.cpu())
