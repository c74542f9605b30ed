"""The whole GQE layer on every workload, end to end against the fp64 oracle.

Prefill: GQELayer.forward(keep=True) runs router -> routed/shared query
projection -> K/V projection -> attention -> output construction and
projection through the C ABI, in the launch configuration the benchmark
times.  The tiny and main-layer workloads are compared on every row; the
long-context (T = 32768, biased router) and wide/skewed (d_model 4096, E = 8,
k = 4, d = 128, 80 % of top-1 on expert 0) workloads on at least 256 sampled
token rows that the oracle computes one by one from the row's own routing and
its sequence's K/V prefix (oracle.gqe_forward_rows): t = 0, T-1, both sides of
every 128-token tile boundary, tokens routed to the rarest expert, random rows.
Decode: GQELayer.decode_step on the full decode workload (64 sequences against
a [64, 8, 32768, 64] cache), sampled sequences against oracle.decode_step.

Checks: TopK exact outside the router's near-ties (tests/golden/near_ties.json,
written by the oracle alone), the GPU's choice at a near-tie valid; y and h
within max-abs 2e-2 and mean-abs 2e-3.  Rows whose routing differs at a
near-tie are valid alternatives and are left out of the numeric comparison
(routing of token t only changes row t).  With GQE_PARITY_REPORT set to a
path, one JSON line per workload (rows compared, errors, near-ties, differing
decisions) is appended there.
"""
import json
import os

import numpy as np
import pytest
import torch

import gqe_inputs as gi
import oracle as orc
from helpers import NEAR_TIE, assert_close_attn, assert_close_proj, bf16_dev, to_f64

pytestmark = pytest.mark.gpu

gq = pytest.importorskip("moe_gqa_query_b200")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "near_ties.json")


@pytest.fixture(autouse=True)
def _cuda_and_error_word():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    yield
    torch.cuda.synchronize()
    assert gq.gqe_device_error() == 0
    torch.cuda.empty_cache()


def _report(**kw):
    path = os.environ.get("GQE_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(kw) + "\n")


def _golden(wname):
    with open(GOLDEN) as f:
        return json.load(f)["workloads"][wname]


def _check_routing_all_tokens(wname, gpu_idx, r_full):
    """GPU TopK over every token against the oracle: differences only at the
    golden near-ties, and there only valid alternatives."""
    gold = _golden(wname)
    tie_set = {tuple(p) for p in gold["near_tie_pairs"]}
    assert gold["near_ties"] == int((r_full["margin"] < NEAR_TIE).sum())
    same = np.all(gpu_idx == r_full["idx"], axis=-1)
    diff = [tuple(map(int, p)) for p in np.argwhere(~same)]
    assert set(diff) <= tie_set, f"{len(set(diff) - tie_set)} decisions differ outside near-ties"
    k = gpu_idx.shape[-1]
    for (t, g), (sure, undecided) in orc.near_tie_alternatives(r_full, k).items():
        chosen = set(gpu_idx[t, g].tolist())
        assert set(sure.tolist()) <= chosen <= set(sure.tolist()) | set(undecided.tolist())
    return gold["near_ties"], len(diff)


def _layer(w, seed=0):
    dims = w.dims
    Wt = gi.layer_weights(dims, seed)
    bias = gi.router_bias(w, seed)
    layer = gq.GQELayer(dims, {k_: torch.from_numpy(v.view(np.int16)) for k_, v in Wt.items()}, bias)
    return Wt, bias, layer


def _sample_rows(dims, counts_ge, idx_full, rng):
    """(b, t) rows: t = 0, T-1 and both sides of every tile boundary of
    sequence 0 (and of sequence 1 when one sequence gives fewer than 200), 32
    tokens routed to the rarest selected expert, 32 random rows."""
    B, T = dims.B, dims.T
    rows = []
    for b in range(min(B, 2)):
        rows += [(b, t) for t in sorted({0, T - 1} | {t for m in range(1, T // 128) for t in (128 * m - 1, 128 * m)})]
        if len(rows) >= 200:
            break
    G, E = dims.G, dims.E
    c = np.asarray(counts_ge).reshape(G, E)
    g_r, e_r = np.unravel_index(np.argmin(np.where(c > 0, c, np.iinfo(np.int64).max)), c.shape)
    toks = np.nonzero(np.any(idx_full[:, g_r, :] == e_r, axis=-1))[0]
    for n in rng.choice(toks, min(32, len(toks)), replace=False):
        rows.append((int(n) // T, int(n) % T))
    for n in rng.choice(dims.N, 32, replace=False):
        rows.append((int(n) // T, int(n) % T))
    seen, out = set(), []
    for r in rows:
        if r not in seen:
            seen.add(r)
            out.append(r)
    return out, (int(g_r), int(e_r), int(c[g_r, e_r]))


@pytest.mark.parametrize("wname", ["tiny_prefill", "main_prefill", "long_prefill", "wide_skewed_prefill"])
def test_layer_forward_every_workload(wname):
    w = gi.WORKLOADS[wname]
    dims = w.dims
    Wt, bias, layer = _layer(w)
    x = gi.layer_input(dims, 0)
    y, inter = layer.forward(bf16_dev(x), keep=True)
    torch.cuda.synchronize()
    gpu_idx = inter["idx"].cpu().numpy()
    # router over every token (cheap in fp64 even at the largest workload)
    r_full = orc.router_topk(x.reshape(dims.N, dims.D), Wt["Wr"], dims.G, dims.E, dims.k, bias, dims.renorm_scope)
    n_ties, n_diff = _check_routing_all_tokens(wname, gpu_idx, r_full)
    counts, _ = orc.router_stats(r_full["probs"], r_full["idx"], dims.G, dims.E)
    assert [int(c) for c in counts] == _golden(wname)["expert_counts"]
    if dims.N <= 16384 and dims.D <= 1024:
        ref = orc.gqe_forward(x, Wt, dims, bias)
        flat = np.arange(dims.N)
        y_ref, h_ref = ref["y"], ref["h"]
        rare = None
    else:
        rng = np.random.default_rng(17)
        rows, rare = _sample_rows(dims, counts, r_full["idx"], rng)
        assert len(rows) >= 256
        ref = orc.gqe_forward_rows(x, Wt, dims, rows, bias)
        flat = np.array([b * dims.T + t for b, t in rows])
        y_ref, h_ref = ref["y"], ref["h"]
        assert np.array_equal(ref["router"]["idx"], r_full["idx"][flat])
    agree = np.all(gpu_idx[flat] == r_full["idx"][flat], axis=(1, 2))
    yg = to_f64(y).reshape(dims.N, -1)[flat]
    hg = to_f64(inter["h"])[flat]
    ymx, ymean = assert_close_attn(yg[agree], y_ref[agree], f"{wname} y")
    hmx, hmean = assert_close_attn(hg[agree], h_ref[agree], f"{wname} h")
    # router weights of the compared rows (token scope: the whole token's selection must agree)
    np.testing.assert_allclose(inter["w"].cpu().numpy()[flat][agree], r_full["w"][flat][agree], atol=1e-5)
    share0 = top1_0 = None
    if w.bias == "expert0":
        share0 = float(np.mean(gpu_idx[:, :, 0] == 0))          # ascending slots: expert 0 is slot 0 when chosen
        top1_0 = float(np.mean(np.argmax(r_full["logits"], axis=-1) == 0))
        assert 0.75 <= top1_0 <= 0.85                           # the workload's ~80 % top-1 skew
    _report(test="layer_forward", workload=wname, rows_compared=int(agree.sum()), rows_total=int(dims.N),
            y_max_abs=ymx, y_mean_abs=ymean, h_max_abs=hmx, h_mean_abs=hmean, near_ties=n_ties,
            near_tie_decisions_differing=n_diff, rarest_expert=rare, expert0_in_topk_share=share0,
            expert0_top1_share=top1_0)
    print(f"[{wname}] rows {int(agree.sum())}: y max-abs {ymx:.3e} mean-abs {ymean:.3e}; near-ties {n_ties}, "
          f"GPU chose the other expert at {n_diff}")


def test_layer_decode_step_full_size_sampled():
    """The decode workload end to end through GQELayer.decode_step: router,
    query projection, the new token's K/V rows appended to the 32768-entry
    cache, attention over the whole cache, output construction and
    projection; four sequences regenerated on the host and checked against
    oracle.decode_step."""
    w = gi.WORKLOADS["decode"]
    dims, L_max = w.dims, w.L
    B, G, d = dims.B, dims.G, dims.d
    Wt, bias, layer = _layer(w)
    x = gi.normal_bf16(0, "xdec", (B, dims.D))
    gen = torch.Generator(device="cuda").manual_seed(5)
    Kc = torch.empty((B, G, L_max, d), dtype=torch.bfloat16, device="cuda").normal_(generator=gen)
    Vc = torch.empty_like(Kc).normal_(generator=gen)
    rows = [0, 21, 42, 63]
    host_K, host_V = [], []
    for b in rows:
        Kb = gi.normal_bf16(0, "Kc", (B, G, L_max, d), rows=[b])
        Vb = gi.normal_bf16(0, "Vc", (B, G, L_max, d), rows=[b])
        Kc[b] = bf16_dev(Kb[0])
        Vc[b] = bf16_dev(Vb[0])
        host_K.append(Kb[0])
        host_V.append(Vb[0])
    lens = np.full(B, L_max, dtype=np.int32)
    lens[21] = L_max - 1000           # one shorter cache among the sampled ones
    y, inter = layer.decode_step(bf16_dev(x), Kc, Vc, torch.from_numpy(lens).cuda(), keep=True)
    torch.cuda.synchronize()
    r_full = orc.router_topk(x, Wt["Wr"], G, dims.E, dims.k, bias, dims.renorm_scope)
    n_ties, n_diff = _check_routing_all_tokens("decode", inter["idx"].cpu().numpy(), r_full)
    sub = dims.replace(B=len(rows))
    ref = orc.decode_step(x[rows], Wt, np.stack(host_K), np.stack(host_V), lens[rows], sub, bias)
    for i, b in enumerate(rows):
        n = int(lens[b])
        assert_close_proj(to_f64(Kc[b, :, n - 1]), ref["Knew"][i, :, 0], f"K row appended, b{b}")
        assert_close_proj(to_f64(Vc[b, :, n - 1]), ref["Vnew"][i, :, 0], f"V row appended, b{b}")
    agree = np.all(inter["idx"].cpu().numpy()[rows] == ref["router"]["idx"], axis=(1, 2))
    ymx, ymean = assert_close_attn(to_f64(y)[rows][agree], ref["y"][agree], "decode y")
    hmx, hmean = assert_close_attn(to_f64(inter["h"])[rows][agree], ref["h"][agree], "decode h")
    _report(test="decode_step", workload="decode", rows_compared=int(agree.sum()), rows_total=B,
            y_max_abs=ymx, y_mean_abs=ymean, h_max_abs=hmx, h_mean_abs=hmean, near_ties=n_ties,
            near_tie_decisions_differing=n_diff)


# ----------------------------------------------------------------------------
# single calls at the largest workloads' shapes

def test_routed_qproj_long_biased_routing():
    """The routed projection fed the long-context workload's own biased
    routing (uneven segment sizes at T = 32768), sampled rows vs the oracle,
    per-expert counts exact."""
    w = gi.WORKLOADS["long_prefill"]
    dims = w.dims
    x = gi.layer_input(dims, 0)
    Wt = gi.layer_weights(dims, 0)
    r = orc.router_topk(x.reshape(dims.N, dims.D), Wt["Wr"], dims.G, dims.E, dims.k, gi.router_bias(w, 0))
    idx = r["idx"]
    hist = np.bincount((np.arange(dims.G)[None, :, None] * dims.E + idx).reshape(-1), minlength=dims.G * dims.E)
    assert hist.max() > 1.5 * hist.min()          # the bias makes the load uneven
    q = torch.empty((dims.B, dims.G, dims.T, dims.k, dims.d), dtype=torch.bfloat16, device="cuda")
    qs = torch.empty((dims.B, dims.T, dims.d), dtype=torch.bfloat16, device="cuda")
    cnt = torch.empty((dims.G * dims.E,), dtype=torch.int32, device="cuda")
    dc = gq.make_dims(dims)
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_ROUTED_QPROJ),), dtype=torch.uint8, device="cuda")
    gq.gqe_routed_qproj(dc, bf16_dev(x), bf16_dev(Wt["Wq"]), bf16_dev(Wt["Wsh"]), torch.from_numpy(idx).cuda(),
                        q, qs, ws, cnt)
    torch.cuda.synchronize()
    assert np.array_equal(cnt.cpu().numpy(), hist)
    rows = np.sort(np.random.default_rng(3).choice(dims.N, 512, replace=False))
    sub = gi.GQEDims(B=1, T=len(rows), D=dims.D, G=dims.G, E=dims.E, k=dims.k, d=dims.d)
    q_ref, qs_ref = orc.routed_qproj(x.reshape(dims.N, -1)[rows], Wt["Wq"], Wt["Wsh"], idx[rows], sub)
    q_gpu = to_f64(q).transpose(0, 2, 1, 3, 4).reshape(dims.N, dims.G, dims.k, dims.d)[rows]
    assert_close_proj(q_gpu, q_ref[0].transpose(1, 0, 2, 3), "q_routed")
    assert_close_proj(to_f64(qs).reshape(dims.N, dims.d)[rows], qs_ref[0], "q_sh")


def test_kv_proj_wide():
    """K/V projection at d_model 4096, 4 groups of d = 128 (the wide workload)."""
    dims = gi.WORKLOADS["wide_skewed_prefill"].dims
    x = gi.layer_input(dims, 2)
    Wt = gi.layer_weights(dims, 2)
    K = torch.empty((dims.B, dims.G, dims.T, dims.d), dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    gq.gqe_kv_proj(gq.make_dims(dims), bf16_dev(x), bf16_dev(Wt["Wk"]), bf16_dev(Wt["Wv"]), K, V)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(4).choice(dims.N, 1024, replace=False))
    sub = dims.replace(B=1, T=len(rows))
    K_ref, V_ref = orc.kv_proj(x.reshape(dims.N, -1)[rows], Wt["Wk"], Wt["Wv"], sub)
    Kg = to_f64(K).transpose(0, 2, 1, 3).reshape(dims.N, dims.G, dims.d)[rows]
    Vg = to_f64(V).transpose(0, 2, 1, 3).reshape(dims.N, dims.G, dims.d)[rows]
    assert_close_proj(Kg, K_ref[0].transpose(1, 0, 2), "K")
    assert_close_proj(Vg, V_ref[0].transpose(1, 0, 2), "V")


def test_combine_out_proj_wide():
    """Output construction + projection over 18 slots of d = 128 into d_model
    4096 (the wide workload), slots read in place; sampled rows of y vs the
    oracle, and the whole y bit-identical to gqe_combine + gqe_linear."""
    dims = gi.WORKLOADS["wide_skewed_prefill"].dims
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    assert dims.slots == 18
    o = gi.normal_bf16(6, "o", (B, G, T, k, d))
    osh = gi.normal_bf16(6, "osh", (B, T, d))
    w = gi.random_weights_simplex(dims, 6)
    Wo = gi.normal_bf16(6, "Wo", (dims.D, dims.slots * d), 0.02)
    dc = gq.make_dims(dims)
    y = torch.full((dims.N, dims.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_COMBINE_OUT_PROJ),), dtype=torch.uint8, device="cuda")
    od, oshd, wd, Wod = bf16_dev(o), bf16_dev(osh), torch.from_numpy(w).cuda(), bf16_dev(Wo)
    gq.gqe_combine_out_proj(dc, od, oshd, wd, Wod, y, ws)
    h = torch.empty((dims.N, dims.slots * d), dtype=torch.bfloat16, device="cuda")
    gq.gqe_combine(dc, od, oshd, wd, h)
    y2 = torch.empty_like(y)
    gq.gqe_linear(h, Wod, y2)
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    rows = np.sort(np.random.default_rng(6).choice(dims.N, 512, replace=False))
    h_ref = orc.combine(o, osh, w.astype(np.float64), dims)
    assert_close_attn(to_f64(y)[rows], orc.out_proj(h_ref[rows], Wo), "y")
    np.testing.assert_array_equal(to_f64(h)[:, :G * k * d], h_ref[:, :G * k * d])     # hard slots: copies


def test_linear_wide_output_projection_shape():
    """gqe_linear at the wide workload's output projection: [16384, 2304] x
    [4096, 2304]^T, sampled rows vs the oracle."""
    M, N, K = 16384, 4096, 2304
    A = gi.normal_bf16(3, "x", (M, K), 1.0)
    W = gi.normal_bf16(3, "Wo", (N, K), 0.02)
    C = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    gq.gqe_linear(bf16_dev(A), bf16_dev(W), C)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(8).choice(M, 512, replace=False))
    assert_close_proj(to_f64(C)[rows], orc.linear(A[rows], W), "linear")
