"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something the GQE pages or mathematics fix:
brute force, closed forms, invariants, or reductions to a library attention
routine.  A plausible slip in the oracle (a dropped term, a transposed operand,
a wrong slot order, a wrong group for the shared head, an off-by-one causal
mask, a wrong renormalisation sum) fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import gqe_inputs as gi
import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _dims(**kw):
    base = dict(B=1, T=8, D=16, G=2, E=3, k=2, d=4)
    base.update(kw)
    return gi.GQEDims(**base)


def _rand(rng, *shape, std=1.0):
    return rng.standard_normal(shape) * std


# ----------------------------------------------------------------------------
# router: GQE study note §3-2 2)

@pytest.mark.parametrize("E,k", [(2, 1), (3, 2), (4, 2), (5, 3), (8, 4), (8, 1), (4, 4)])
def test_topk_matches_brute_force(E, k):
    """TopK == the lexicographically smallest k-subset with the largest logit sum.

    Integer logits make sums exact and plant many ties (tie rule: lower index).
    """
    rng = np.random.default_rng(E * 10 + k)
    N, G = 64, 3
    s = rng.integers(-2, 3, size=(N, G, E)).astype(np.float64)
    sel = orc.topk_select(orc.group_softmax(s), k)
    for t in range(N):
        for g in range(G):
            best, best_sum = None, -np.inf
            for c in itertools.combinations(range(E), k):   # lexicographic order
                sm = s[t, g, list(c)].sum()
                if sm > best_sum:
                    best, best_sum = c, sm
            assert tuple(sel[t, g]) == best


def test_softmax_and_renormalisation_sums():
    rng = np.random.default_rng(1)
    N, D, G, E, k = 50, 16, 4, 5, 2
    x = _rand(rng, N, D)
    Wr = _rand(rng, D, G * E)
    r = orc.router_topk(x, Wr, G, E, k)
    np.testing.assert_allclose(r["probs"].sum(-1), 1.0, atol=1e-14)
    # token scope: sum over all k*G selections of a token is 1
    np.testing.assert_allclose(r["w"].sum(axis=(1, 2)), 1.0, atol=1e-14)
    # group scope: 1 within each group
    r1 = orc.router_topk(x, Wr, G, E, k, scope=1)
    np.testing.assert_allclose(r1["w"].sum(axis=2), 1.0, atol=1e-14)
    # k = 1 with group scope: every weight is exactly 1
    r2 = orc.router_topk(x, Wr, G, E, 1, scope=1)
    assert np.all(r2["w"] == 1.0)
    # selected weights are the selected probabilities, rescaled by one factor per token
    psel = np.take_along_axis(r["probs"], r["idx"].astype(np.int64), -1)
    ratio = r["w"] / psel
    np.testing.assert_allclose(ratio, ratio[:, :1, :1] * np.ones_like(ratio), rtol=1e-13)


def test_router_selects_largest_probabilities():
    """Every selected expert's probability is >= every unselected one's."""
    rng = np.random.default_rng(2)
    x = _rand(rng, 40, 8)
    Wr = _rand(rng, 8, 3 * 6)
    r = orc.router_topk(x, Wr, 3, 6, 3)
    p, idx = r["probs"], r["idx"]
    for t in range(40):
        for g in range(3):
            chosen = set(idx[t, g])
            lo = min(p[t, g, e] for e in chosen)
            hi = max((p[t, g, e] for e in range(6) if e not in chosen), default=-1)
            assert lo >= hi
            assert list(idx[t, g]) == sorted(chosen)


def test_margin_definition():
    s = np.array([[[0.5, 2.0, 1.0, 1.75]]])
    np.testing.assert_allclose(orc.selection_margin(s, 1), [[0.25]])
    np.testing.assert_allclose(orc.selection_margin(s, 2), [[0.75]])
    assert np.isinf(orc.selection_margin(s, 4)).all()


def test_near_tie_alternatives_sets():
    """The near-tie helper the router parity tests use: for a (token, group)
    whose k-th/(k+1)-th logit margin is under 1e-4, the experts within 1e-4 of
    the k-th logit are undecided and those clearly above it are sure; clear
    groups and k = E give no entry."""
    s = np.array([[[1.0, 1.00005, 0.2, -0.3],      # k=1: a two-way tie on top
                   [3.0, 0.0, -1.0, 0.5]],         # clear
                  [[2.0, 1.0, 1.00003, 0.0],       # k=2: expert 0 sure, 1 and 2 tied for 2nd
                   [0.1, 0.1, 0.1, 0.1]]])         # four-way tie
    r1 = {"logits": s, "margin": orc.selection_margin(s, 1)}
    alt1 = orc.near_tie_alternatives(r1, 1)
    assert set(alt1) == {(0, 0), (1, 1)}
    sure, und = alt1[(0, 0)]
    assert sure.tolist() == [] and und.tolist() == [0, 1]
    sure, und = alt1[(1, 1)]
    assert sure.tolist() == [] and und.tolist() == [0, 1, 2, 3]
    r2 = {"logits": s, "margin": orc.selection_margin(s, 2)}
    alt2 = orc.near_tie_alternatives(r2, 2)
    assert set(alt2) == {(1, 0), (1, 1)}
    sure, und = alt2[(1, 0)]
    assert sure.tolist() == [0] and und.tolist() == [1, 2]
    assert orc.near_tie_alternatives({"logits": s, "margin": orc.selection_margin(s, 4)}, 4) == {}


def test_router_bias_is_added_per_expert():
    rng = np.random.default_rng(3)
    x = _rand(rng, 10, 6)
    Wr = _rand(rng, 6, 4)
    b = np.array([0.0, 10.0, -3.0, 1.0])
    s0 = orc.router_logits(x, Wr)
    s1 = orc.router_logits(x, Wr, b)
    np.testing.assert_allclose(s1 - s0, np.broadcast_to(b, s0.shape), atol=1e-12)


# ----------------------------------------------------------------------------
# attention closed forms: GQE study note §1-1

def _scalar_attention(q, K, V, t, scale):
    """Pure-Python loops: o = sum_j<=t exp(s_j - max) V_j / sum_j exp(s_j - max)."""
    s = [sum(q[a] * K[j][a] for a in range(len(q))) * scale for j in range(t + 1)]
    m = max(s)
    z = [math.exp(v - m) for v in s]
    den = sum(z)
    return [sum(z[j] * V[j][c] for j in range(t + 1)) / den for c in range(len(V[0]))]


def test_attention_matches_scalar_loops():
    rng = np.random.default_rng(4)
    T, d = 9, 5
    q = _rand(rng, T, d)
    K = _rand(rng, T, d)
    V = _rand(rng, T, d)
    o = orc.causal_attention(q, np.arange(T), K, V, 0.37, chunk=4)
    for t in range(T):
        ref = _scalar_attention(q[t].tolist(), K.tolist(), V.tolist(), t, 0.37)
        np.testing.assert_allclose(o[t], ref, rtol=1e-12, atol=1e-13)


def test_position_zero_returns_own_value_row():
    dims = _dims(B=2, T=6, G=3, E=2, k=2, d=4)
    rng = np.random.default_rng(5)
    q = _rand(rng, 2, 3, 6, 2, 4) * 5
    qs = _rand(rng, 2, 6, 4) * 5
    K = _rand(rng, 2, 3, 6, 4)
    V = _rand(rng, 2, 3, 6, 4)
    o, osh, _, _ = orc.attn_prefill(q, qs, K, V, dims)
    for b in range(2):
        for g in range(3):
            for j in range(2):
                np.testing.assert_allclose(o[b, g, 0, j], V[b, g, 0], atol=1e-14)
        np.testing.assert_allclose(osh[b, 0], V[b, dims.sg, 0], atol=1e-14)


def test_constant_keys_give_causal_prefix_mean():
    dims = _dims(B=1, T=7, G=2, E=2, k=1, d=3, sg=1)
    rng = np.random.default_rng(6)
    q = _rand(rng, 1, 2, 7, 1, 3)
    qs = _rand(rng, 1, 7, 3)
    K = np.broadcast_to(_rand(rng, 1, 2, 1, 3), (1, 2, 7, 3)).copy()
    V = _rand(rng, 1, 2, 7, 3)
    o, osh, _, _ = orc.attn_prefill(q, qs, K, V, dims)
    for t in range(7):
        for g in range(2):
            np.testing.assert_allclose(o[0, g, t, 0], V[0, g, : t + 1].mean(0), atol=1e-13)
        # the shared head reads KV group sg = 1
        np.testing.assert_allclose(osh[0, t], V[0, 1, : t + 1].mean(0), atol=1e-13)


def test_packed_rows_each_use_their_own_token_position():
    """With k > 1 the k rows of token t see exactly keys 0..t (no more, no fewer)."""
    dims = _dims(B=1, T=5, G=1, E=3, k=3, d=2, n_shared=0)
    rng = np.random.default_rng(7)
    q = _rand(rng, 1, 1, 5, 3, 2)
    K = _rand(rng, 1, 1, 5, 2)
    V = _rand(rng, 1, 1, 5, 2)
    o, _, lse, _ = orc.attn_prefill(q, None, K, V, dims)
    for t in range(5):
        for j in range(3):
            ref = _scalar_attention(q[0, 0, t, j].tolist(), K[0, 0].tolist(), V[0, 0].tolist(),
                                    t, 1.0 / math.sqrt(dims.d))
            np.testing.assert_allclose(o[0, 0, t, j], ref, rtol=1e-12)
            s = [float(q[0, 0, t, j] @ K[0, 0, i]) * 1.0 / math.sqrt(dims.d) for i in range(t + 1)]
            np.testing.assert_allclose(lse[0, 0, t, j], math.log(sum(math.exp(v) for v in s)),
                                       rtol=1e-12)


# ----------------------------------------------------------------------------
# reductions to dense attention (library routine: torch SDPA, fp64 on CPU)

def _sdpa(q, k, v, scale):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        is_causal=True, scale=scale).numpy()


def test_single_expert_is_standard_multi_head_attention():
    """E = 1 (k = 1): every group's one expert is a plain causal attention head."""
    dims = gi.GQEDims(B=2, T=12, D=10, G=3, E=1, k=1, d=4, n_shared=1, sg=2)
    rng = np.random.default_rng(8)
    x = _rand(rng, 2, 12, 10)
    Wt = dict(Wr=_rand(rng, 10, 3), Wq=_rand(rng, 3, 1, 4, 10) * 0.5,
              Wk=_rand(rng, 12, 10) * 0.5, Wv=_rand(rng, 12, 10), Wsh=_rand(rng, 4, 10) * 0.5,
              Wo=_rand(rng, 10, 5 * 4))
    out = orc.gqe_forward(x, Wt, dims)
    assert np.all(out["router"]["idx"] == 0)
    q = np.einsum("btD,gdD->bgtd", x, Wt["Wq"][:, 0])
    k = np.einsum("btD,gdD->bgtd", x, Wt["Wk"].reshape(3, 4, 10))
    v = np.einsum("btD,gdD->bgtd", x, Wt["Wv"].reshape(3, 4, 10))
    ref = _sdpa(q, k, v, 0.5)
    np.testing.assert_allclose(out["o"][:, :, :, 0], ref, atol=1e-12)
    qs = np.einsum("btD,dD->btd", x, Wt["Wsh"])[:, None]
    ref_sh = _sdpa(qs, k[:, 2:3], v[:, 2:3], 0.5)[:, 0]
    np.testing.assert_allclose(out["o_sh"], ref_sh, atol=1e-12)
    # token-scope weights with k=1, E=1: every p = 1, so p~ = 1/G and the
    # route slot is the mean of the G head outputs
    h = out["h"].reshape(2, 12, -1)
    np.testing.assert_allclose(h[..., 3 * 4: 4 * 4], ref.mean(axis=1), atol=1e-12)


def test_all_experts_selected_is_dense_gqa():
    """k = E, no shared head, uniform router: hard slots equal dense GQA heads.

    Dense GQA per the freeguideonline tutorial's recipe (K/V repeated so query
    head i reads KV group floor(i / (h/g))), then a library causal attention.
    Head order g*E + e; the route slot is the mean of all G*E heads.
    """
    G, E, d, D, T, B = 3, 2, 4, 8, 10, 2
    dims = gi.GQEDims(B=B, T=T, D=D, G=G, E=E, k=E, d=d, n_shared=0)
    rng = np.random.default_rng(9)
    x = _rand(rng, B, T, D)
    Wq = _rand(rng, G, E, d, D) * 0.5
    Wk = _rand(rng, G * d, D) * 0.5
    Wv = _rand(rng, G * d, D)
    Wt = dict(Wr=np.zeros((D, G * E)), Wq=Wq, Wk=Wk, Wv=Wv, Wsh=np.zeros((0, D)),
              Wo=_rand(rng, D, (G * E + 1) * d))
    out = orc.gqe_forward(x, Wt, dims)
    h = G * E
    q = torch.from_numpy(x @ Wq.reshape(h * d, D).T).view(B, T, h, d).transpose(1, 2)
    k = torch.from_numpy(x @ Wk.T).view(B, T, G, d).transpose(1, 2)
    v = torch.from_numpy(x @ Wv.T).view(B, T, G, d).transpose(1, 2)
    k = k.repeat_interleave(h // G, dim=1)
    v = v.repeat_interleave(h // G, dim=1)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).numpy()
    ref_rows = ref.transpose(0, 2, 1, 3).reshape(B * T, h * d)      # concat heads per token
    np.testing.assert_allclose(out["h"][:, : h * d], ref_rows, atol=1e-12)
    np.testing.assert_allclose(out["h"][:, h * d:], ref.mean(axis=1).transpose(0, 1, 2).reshape(B * T, d),
                               atol=1e-12)
    assert out["h"].shape[1] == (G * E + 1) * d


def test_decode_equals_last_prefill_row():
    """A decode step for token T-1 over the cache of tokens 0..T-1 reproduces
    row T-1 of the prefill output (cache write at row cache_len-1, causal read)."""
    T = 9
    dims = gi.GQEDims(B=3, T=T, D=12, G=2, E=3, k=2, d=4, n_shared=1, sg=1)
    rng = np.random.default_rng(10)
    x = _rand(rng, 3, T, 12)
    Wt = dict(Wr=_rand(rng, 12, 6), Wq=_rand(rng, 2, 3, 4, 12) * 0.4, Wk=_rand(rng, 8, 12) * 0.4,
              Wv=_rand(rng, 8, 12), Wsh=_rand(rng, 4, 12) * 0.4, Wo=_rand(rng, 12, 6 * 4))
    pre = orc.gqe_forward(x, Wt, dims)
    L = T + 3
    Kc = _rand(rng, 3, 2, L, 4)
    Vc = _rand(rng, 3, 2, L, 4)
    Kc[:, :, : T - 1] = pre["K"][:, :, : T - 1]
    Vc[:, :, : T - 1] = pre["V"][:, :, : T - 1]
    ddims = dims.replace(T=1)
    dec = orc.decode_step(x[:, T - 1], Wt, Kc, Vc, np.full(3, T), ddims)
    y_pre = pre["y"].reshape(3, T, -1)[:, T - 1]
    np.testing.assert_allclose(dec["y"], y_pre, atol=1e-12)
    # rows beyond cache_len are never read: changing them changes nothing
    Kc2, Vc2 = Kc.copy(), Vc.copy()
    Kc2[:, :, T:] = 1e3
    Vc2[:, :, T:] = -1e3
    dec2 = orc.decode_step(x[:, T - 1], Wt, Kc2, Vc2, np.full(3, T), ddims)
    np.testing.assert_allclose(dec2["y"], dec["y"], atol=0)


def test_decode_ragged_cache_lengths_match_scalar_loops():
    """Decode attention with a different cache length per sequence: every
    routed row of sequence b attends to rows 0..cache_len[b]-1 of its own
    group's cache and the shared row to group sg's, written out as scalar
    loops (GQA tutorial, decode with a KV cache; study note §3-2 5))."""
    rng = np.random.default_rng(12)
    B, G, k, d, L = 3, 3, 2, 4, 11
    dims = gi.GQEDims(B=B, T=1, D=8, G=G, E=3, k=k, d=d, n_shared=1, sg=2)
    q = _rand(rng, B, G, k, d)
    qs = _rand(rng, B, d)
    Kc = _rand(rng, B, G, L, d)
    Vc = _rand(rng, B, G, L, d)
    lens = np.array([L, 1, 6])
    o, o_sh = orc.attn_decode(q, qs, Kc, Vc, lens, dims)
    sc = 1.0 / math.sqrt(d)
    for b in range(B):
        n = int(lens[b])
        for g in range(G):
            for j in range(k):
                ref = _scalar_attention(q[b, g, j].tolist(), Kc[b, g, :n].tolist(), Vc[b, g, :n].tolist(), n - 1, sc)
                np.testing.assert_allclose(o[b, g, j], ref, rtol=1e-12, atol=1e-13)
        ref = _scalar_attention(qs[b].tolist(), Kc[b, 2, :n].tolist(), Vc[b, 2, :n].tolist(), n - 1, sc)
        np.testing.assert_allclose(o_sh[b], ref, rtol=1e-12, atol=1e-13)
    # a cache of one row returns that row's value
    np.testing.assert_allclose(o[1], np.broadcast_to(Vc[1, :, 0][:, None, :], (G, k, d)), atol=1e-15)


# ----------------------------------------------------------------------------
# output construction and locality: GQE study note §3-2 3)-5)

def test_routing_of_one_token_changes_only_its_row():
    dims = gi.GQEDims(B=1, T=10, D=8, G=2, E=4, k=2, d=3)
    rng = np.random.default_rng(11)
    x = _rand(rng, 10, 8)
    Wq = _rand(rng, 2, 4, 3, 8)
    Wsh = _rand(rng, 3, 8)
    Wk = _rand(rng, 6, 8)
    Wv = _rand(rng, 6, 8)
    idx = gi.random_routing(dims, seed=1)
    w = gi.random_weights_simplex(dims, seed=1).astype(np.float64)
    idx2 = idx.copy()
    idx2[4, 1] = [0, 3] if list(idx[4, 1]) != [0, 3] else [1, 2]
    hs = []
    for ii in (idx, idx2):
        q, qs = orc.routed_qproj(x, Wq, Wsh, ii, dims)
        K, V = orc.kv_proj(x, Wk, Wv, dims)
        o, osh, _, _ = orc.attn_prefill(q, qs, K, V, dims)
        hs.append(orc.combine(o, osh, w, dims))
    diff = np.abs(hs[0] - hs[1]).max(axis=1)
    assert diff[4] > 1e-3
    assert np.all(np.delete(diff, 4) == 0)


def test_slot_counts_closed_forms():
    main = gi.WORKLOADS["main_prefill"].dims
    assert main.slots == 10          # 8 hard + weighted + shared
    assert main.h_active == 9        # 8 routed + 1 shared
    assert main.k / main.E == 0.5    # active routed fraction kG/N = k/E
    wide = gi.WORKLOADS["wide_skewed_prefill"].dims
    assert wide.slots == 18 and wide.h_active == 17


def _load_hand_worked():
    with open(os.path.join(GOLDEN, "hand_worked_layer.json")) as f:
        g = json.load(f)
    sub = {"SQRT2_LN3": math.sqrt(2) * math.log(3), "SQRT2_LN2": math.sqrt(2) * math.log(2)}

    def arr(v):
        if isinstance(v, list):
            return [arr(u) for u in v]
        return sub[v] if isinstance(v, str) else float(v)
    Wt = {k: np.array(arr(g[k]), dtype=np.float64) for k in ("Wr", "Wq", "Wsh", "Wk", "Wv", "Wo")}
    return gi.GQEDims(**g["dims"]), np.array(g["x"], dtype=np.float64)[None], Wt


def test_hand_worked_layer():
    """Closed-form outputs of the two-token layer in tests/golden/hand_worked_layer.json."""
    dims, x, Wt = _load_hand_worked()
    out = orc.gqe_forward(x, Wt, dims)
    e = math.e
    # router: token 0 picks (g0,e0), (g1,e1); token 1 picks (g0,e1), (g1,e0)
    assert out["router"]["idx"][:, :, 0].tolist() == [[0, 1], [1, 0]]
    pA, pB = e / (1 + e), e ** 2 / (1 + e ** 2)           # token 0
    pC, pD = e ** 3 / (1 + e ** 3), e / (1 + e)           # token 1
    V0 = {0: np.array([1.0, 2.0]), 1: np.array([3.0, -1.0])}   # group 0 values by token
    V1 = {0: np.array([0.0, 1.0]), 1: np.array([2.0, 2.0])}    # group 1
    # token 0 attends only to itself
    h0 = np.concatenate([V0[0], V1[0], (pA * V0[0] + pB * V1[0]) / (pA + pB), V0[0]])
    # token 1: weight on key 1 is logistic(score): ln3 -> 3/4, 0 -> 1/2, ln2 (shared) -> 2/3
    o_g0 = 0.25 * V0[0] + 0.75 * V0[1]
    o_g1 = 0.5 * V1[0] + 0.5 * V1[1]
    o_sh = V0[0] / 3 + 2 * V0[1] / 3
    h1 = np.concatenate([o_g0, o_g1, (pC * o_g0 + pD * o_g1) / (pC + pD), o_sh])
    np.testing.assert_allclose(out["h"], np.stack([h0, h1]), atol=1e-12)
    y = np.stack([[h[0], h[2], h[4] + h[5], h[6] - h[7]] for h in (h0, h1)])
    np.testing.assert_allclose(out["y"], y, atol=1e-12)


def test_planted_mistakes_are_caught():
    """Mutations of the oracle's steps, planted here on the CPU, fail the pins.

    A transposed slot order, a shared head on the wrong group and a group-scope
    renormalisation each change the hand-worked layer's outputs.
    """
    dims, x, Wt = _load_hand_worked()
    ref = orc.gqe_forward(x, Wt, dims)["h"]
    # shared head on group 1 instead of sg = 0
    bad = orc.gqe_forward(x, Wt, dims.replace(sg=1))["h"]
    assert np.abs(bad - ref).max() > 0.1
    # group-scope renormalisation (k = 1 gives p~ = 1 per group: the slot becomes a sum)
    bad = orc.gqe_forward(x, Wt, dims.replace(renorm_scope=1))["h"]
    assert np.abs(bad - ref).max() > 0.1
    # transposed query weight
    Wt2 = dict(Wt)
    Wt2["Wq"] = Wt["Wq"].transpose(1, 0, 2, 3).copy()
    bad = orc.gqe_forward(x, Wt2, dims)["h"]
    assert np.abs(bad - ref).max() > 0.1


# ----------------------------------------------------------------------------
# inputs module: recipe properties (not method arithmetic)

def test_bf16_rounding_is_nearest_even():
    vals = np.array([1.0, 1.00390625, 1.005859375, 1.0078125 + 2 ** -9, -3.14159], dtype=np.float32)
    bits = gi.f32_to_bf16_bits(vals)
    back = gi.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins
    assert back[1] == 1.0
    assert back[2] == np.float32(1.0078125)
    assert abs(back[4] - vals[4]) <= 2 ** -8 * abs(vals[4])
    assert np.array_equal(orc.f64(bits), back.astype(np.float64))


def test_inputs_are_reproducible_per_leading_index():
    dims = gi.GQEDims(B=3, T=4, D=8, G=2, E=2, k=1, d=4)
    full = gi.layer_input(dims, seed=5)
    part = gi.layer_input(dims, seed=5, rows=[2])
    assert np.array_equal(full[2], part[0])
    assert not np.array_equal(gi.layer_input(dims, seed=6), full)


def test_skewed_router_bias_realises_expert0_share():
    """Wide/skewed workload: with the +3 bias, expert 0 is top-1 for most tokens."""
    w = gi.WORKLOADS["wide_skewed_prefill"]
    dims = w.dims.replace(B=1, T=512)
    x = gi.layer_input(dims)
    Wt = gi.layer_weights(dims)
    r = orc.router_topk(orc.f64(x).reshape(-1, dims.D), Wt["Wr"], dims.G, dims.E, dims.k,
                        gi.router_bias(w))
    top1 = r["logits"].argmax(-1)
    frac0 = float((top1 == 0).mean())
    in_topk = float((r["idx"] == 0).any(-1).mean())
    assert 0.7 < frac0 < 0.9
    assert in_topk > 0.95


# ----------------------------------------------------------------------------
# output-construction variants ("GQE" study note §5-1, ablation rows) and the
# un-renormalised router weights


def _brute_force_h(o, osh, w, dims):
    """h token by token and slot by slot with plain Python loops."""
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    rows = []
    for b in range(B):
        for t in range(T):
            row = []
            route = [0.0] * d
            for g in range(G):
                for j in range(k):
                    v = [float(gi.bf16_bits_to_f32(o[b, g, t, j, c:c + 1])[0]) for c in range(d)]
                    wt = float(w[b * T + t, g, j])
                    row += [wt * x for x in v] if dims.output_mode == 2 else v
                    route = [r + wt * x for r, x in zip(route, v)]
            if dims.output_mode == 0:
                row += route
            if dims.n_shared:
                row += [float(gi.bf16_bits_to_f32(osh[b, t, c:c + 1])[0]) for c in range(d)]
            rows.append(row)
    return np.array(rows)


@pytest.mark.parametrize("mode", [0, 1, 2])
@pytest.mark.parametrize("n_shared", [0, 1])
def test_output_modes_match_brute_force(mode, n_shared):
    dims = gi.GQEDims(B=2, T=3, D=64, G=3, E=3, k=2, d=4, n_shared=n_shared, output_mode=mode)
    o = gi.normal_bf16(21, "o", (dims.B, dims.G, dims.T, dims.k, dims.d))
    osh = gi.normal_bf16(21, "osh", (dims.B, dims.T, dims.d))
    w = gi.random_weights_simplex(dims, 21).astype(np.float64)
    h = orc.combine(o, osh, w, dims)
    assert h.shape == (dims.N, dims.slots * dims.d)
    np.testing.assert_allclose(h, _brute_force_h(o, osh, w, dims), rtol=0, atol=1e-12)


def test_weighted_concat_slots_sum_to_the_weighted_sum_slot():
    """Mode 2's weighted hard slots, added over the slots, give mode 0's
    weighted-sum slot; mode 1's h is mode 0's without that slot."""
    base = gi.GQEDims(B=1, T=5, D=64, G=4, E=2, k=1, d=8, n_shared=1)
    o = gi.normal_bf16(22, "o", (1, 4, 5, 1, 8))
    osh = gi.normal_bf16(22, "osh", (1, 5, 8))
    w = gi.random_weights_simplex(base, 22).astype(np.float64)
    h0 = orc.combine(o, osh, w, base)
    h1 = orc.combine(o, osh, w, base.replace(output_mode=1))
    h2 = orc.combine(o, osh, w, base.replace(output_mode=2))
    G, k, d = 4, 1, 8
    route = h0[:, G * k * d:(G * k + 1) * d]
    np.testing.assert_allclose(h2[:, :G * k * d].reshape(5, G * k, d).sum(axis=1), route, atol=1e-12)
    np.testing.assert_array_equal(h1, np.delete(h0, np.s_[G * k * d:(G * k + 1) * d], axis=1))
    np.testing.assert_array_equal(h1[:, -d:], h2[:, -d:])


def test_renorm_scope_none_keeps_group_softmax_probabilities():
    rng = np.random.default_rng(23)
    x = gi.f32_to_bf16_bits(rng.normal(size=(6, 32)).astype(np.float32))
    Wr = gi.f32_to_bf16_bits(rng.normal(size=(32, 8), scale=0.3).astype(np.float32))
    r = orc.router_topk(orc.f64(x), Wr, 2, 4, 2, None, 2)
    xs, W = orc.f64(x), orc.f64(Wr)
    for t in range(6):
        for g in range(2):
            s = xs[t] @ W[:, g * 4:(g + 1) * 4]
            p = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
            np.testing.assert_allclose(r["w"][t, g], p[r["idx"][t, g]], rtol=1e-12)
    # a single expert per group: the weight is exactly 1
    r1 = orc.router_topk(orc.f64(x), Wr[:, :2], 2, 1, 1, None, 2)
    assert np.all(r1["w"] == 1.0)


def test_router_stats_closed_forms_and_brute_force():
    """Per group the selection counts add to N*k and the probability sums to N
    (each token's in-group probabilities add to 1); counts match a loop."""
    rng = np.random.default_rng(24)
    N, G, E, k, D = 40, 3, 4, 2, 32
    x = gi.f32_to_bf16_bits(rng.normal(size=(N, D)).astype(np.float32))
    Wr = gi.f32_to_bf16_bits(rng.normal(size=(D, G * E), scale=0.3).astype(np.float32))
    r = orc.router_topk(orc.f64(x), Wr, G, E, k)
    counts, psum = orc.router_stats(r["probs"], r["idx"], G, E)
    for g in range(G):
        assert counts[g * E:(g + 1) * E].sum() == N * k
        assert abs(psum[g * E:(g + 1) * E].sum() - N) < 1e-9
    loop = np.zeros(G * E, dtype=np.int64)
    for t in range(N):
        for g in range(G):
            for e in r["idx"][t, g]:
                loop[g * E + int(e)] += 1
    np.testing.assert_array_equal(counts, loop)


# ----------------------------------------------------------------------------
# the layer at chosen rows equals the whole layer at those rows

@pytest.mark.parametrize("kw", [
    dict(B=2, T=19, D=24, G=3, E=4, k=2, d=4, sg=1),
    dict(B=1, T=33, D=16, G=2, E=2, k=1, d=8),
    dict(B=3, T=7, D=16, G=2, E=3, k=3, d=4, n_shared=0),
    dict(B=2, T=12, D=16, G=2, E=4, k=2, d=4, renorm_scope=1, output_mode=2),
    dict(B=1, T=10, D=16, G=4, E=2, k=1, d=4, output_mode=1),
])
def test_forward_rows_equals_full_layer(kw):
    """gqe_forward_rows (used for sampled rows of the large workloads) gives
    the full oracle layer's router decision, h and y at every requested row,
    in the requested order, repeated rows included."""
    dims = gi.GQEDims(**kw)
    rng = np.random.default_rng(sum(kw.values()))
    x = gi.f32_to_bf16_bits(rng.standard_normal((dims.B, dims.T, dims.D)).astype(np.float32))
    Wt = {n: gi.f32_to_bf16_bits((rng.standard_normal(v.shape) * 0.3).astype(np.float32))
          for n, v in gi.layer_weights(dims).items()}
    bias = rng.standard_normal(dims.G * dims.E).astype(np.float32)
    full = orc.gqe_forward(x, Wt, dims, bias)
    rows = [(b, t) for b in range(dims.B) for t in range(dims.T)]
    rows = rows[::-1] + rows[:3]
    part = orc.gqe_forward_rows(x, Wt, dims, rows, bias)
    flat = [b * dims.T + t for b, t in rows]
    assert np.array_equal(part["router"]["idx"], full["router"]["idx"][flat])
    np.testing.assert_allclose(part["router"]["w"], full["router"]["w"][flat], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(part["h"], full["h"][flat], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(part["y"], full["y"][flat], rtol=1e-11, atol=1e-13)
