"""Plain fp64 CPU oracle of the Grouped Query Experts (GQE) attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or run
this module: only the test suite, the smoke check and the benchmark's timed
CPU-baseline leg use it.  It shares no code with the CUDA library.

Every function follows one passage of the pages that describe GQE and names
it.  Pages cited:
  [SN]  "GQE" study note (dimensionstp.github.io/study-concept/gqe), the
        detailed walkthrough: §1-1 (attention equation, GQA notation),
        §3-2 items 1)-7) (router, TopK, hard slots, weighted-sum slot, shared
        head, final concat, compute profile, output projection).
  [AF]  ai-feeds summary "Grouped Query Experts: GQA自注意力上的混合专家",
        "方法" section (unselected query heads are skipped; KV unchanged).
  [FG]  freeguideonline tutorial "分组查询注意力 GQA", "GQA 核心原理与计算流程"
        (head i reads KV group floor(i/(h/g))) and "自回归推理中的内存带宽优势"
        (a decode step reads the whole KV cache).

Readings where the pages leave a step open (each one is listed in the design
notes of the repository):
  * p~ is normalised over all k*G selections of a token (scope 0); scope 1
    normalises within a group; scope 2 leaves the in-group softmax
    probability p as it is (for the ablation variants below).
  * the two ablation variants of [SN] §5-1 (accuracy table), which the pages
    name but do not define, read plainly: "hard concat only" (output_mode 1)
    drops the weighted-sum slot, h = [hard slots, shared]; "weighted concat,
    no renormalised slot" (output_mode 2) scales each hard slot by its router
    weight and has no weighted-sum slot, h = [w * hard slots, shared].
  * hard slots are group-major, and inside a group in ascending expert index.
  * TopK ties go to the lower expert index.
  * the shared head has no K/V of its own and reads KV group ``sg``.
  * no positional encoding, biases, norms or dropout; scale 1/sqrt(d); causal.
  * decode: the cache holds ``cache_len`` valid rows including the new token.

Pinned by the tests in tests/test_oracle_pins.py: brute-force TopK, softmax and
renormalisation sums, position-0 and constant-key closed forms, the E=1 and
k=E (dense GQA) reductions against a library attention routine, per-token
locality, a hand-derived worked example of the whole layer, and a scalar
pure-Python attention on tiny inputs.  Parity of the full composition beyond
those parts rests on these pins (no page prints a numeric example).

Arrays: bf16 inputs arrive as uint16 bit patterns and are widened exactly to
float64; everything is computed in float64.
"""
from __future__ import annotations

import math

import numpy as np


# ----------------------------------------------------------------------------
# storage

def f64(a) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64; float arrays pass through."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ----------------------------------------------------------------------------
# router: [SN] §3-2 2)

def router_logits(x, Wr, bias=None):
    """s_{t,g,e} = r_g(x_t)_e with r a linear map x_t -> x_t Wr (+ bias).

    x [N, D], Wr [D, G*E] -> s [N, G*E]  ([SN] §3-2 2), score equation).
    """
    s = f64(x) @ f64(Wr)
    if bias is not None:
        s = s + f64(bias)[None, :]
    return s


def group_softmax(s):
    """p_{t,g,e} = exp(s_{t,g,e}) / sum_{e'} exp(s_{t,g,e'}) within each group.

    s [N, G, E] -> p [N, G, E]  ([SN] §3-2 2), softmax equation).
    """
    m = s.max(axis=-1, keepdims=True)
    z = np.exp(s - m)
    return z / z.sum(axis=-1, keepdims=True)


def topk_select(p, k):
    """S_{t,g} = TopK(p_{t,g,1:E}, k), ties to the lower index, returned ascending.

    p [N, G, E] -> int32 [N, G, k]  ([SN] §3-2 2), TopK equation).
    """
    N, G, E = p.shape
    e_idx = np.broadcast_to(np.arange(E), p.shape)
    # order by (-p, e): lexsort keys are given last-major
    order = np.lexsort((e_idx, -p), axis=-1)
    sel = np.sort(order[..., :k], axis=-1)
    return sel.astype(np.int32)


def selection_margin(s, k):
    """k-th minus (k+1)-th largest logit per (token, group); +inf when k == E."""
    E = s.shape[-1]
    if k >= E:
        return np.full(s.shape[:-1], np.inf)
    srt = -np.sort(-s, axis=-1)
    return srt[..., k - 1] - srt[..., k]


def renormalise(p, sel, scope=0):
    """p~ over the selected experts ([SN] §3-2 4), "normalised over the selected outputs").

    scope 0: p~_{t,g,e} = p_{t,g,e} / sum_{g'} sum_{e' in S_{t,g'}} p_{t,g',e'}
    scope 1: the same sum restricted to the token's own group g.
    scope 2: no renormalisation, p~ = p (ablation variants).
    Returns float64 [N, G, k] aligned with ``sel``.
    """
    psel = np.take_along_axis(p, sel.astype(np.int64), axis=-1)
    if scope == 2:
        return psel.copy()
    if scope == 0:
        den = psel.sum(axis=(1, 2), keepdims=True)
    else:
        den = psel.sum(axis=2, keepdims=True)
    return psel / den


def router_topk(x, Wr, G, E, k, bias=None, scope=0):
    """The router step: logits, in-group softmax, TopK, renormalised weights."""
    s = router_logits(x, Wr, bias).reshape(-1, G, E)
    p = group_softmax(s)
    sel = topk_select(p, k)
    w = renormalise(p, sel, scope)
    return dict(logits=s, probs=p, idx=sel, w=w, margin=selection_margin(s, k))


# ----------------------------------------------------------------------------
# projections: [SN] §3-2 2) (selected experts compute their query projection),
# [AF] 方法 (unselected query heads take no part), [SN] §1-2 3) (KV dense)

def linear(x, W):
    """x W^T with W in [out, in] layout."""
    return f64(x) @ f64(W).T


def router_stats(probs, idx, G, E):
    """Per (group, expert): tokens that selected it and the sum of its in-group
    probability over the tokens ([SN] §4-3, §4-4: load balance and collapse
    monitoring; the loss built from them is not given).  probs [N, G, E],
    idx [N, G, k] -> (counts int64 [G*E], prob_sum float64 [G*E])."""
    N = probs.shape[0]
    counts = np.zeros(G * E, dtype=np.int64)
    for g in range(G):
        for e in range(E):
            counts[g * E + e] = int(np.sum(idx[:, g, :] == e))
    prob_sum = np.asarray(probs, dtype=np.float64).reshape(N, G * E).sum(axis=0)
    return counts, prob_sum


def routed_qproj(x, Wq, Wsh, idx, dims):
    """q_{t,g,e} = x_t Wq[g,e]^T for e in S_{t,g} only; q_sh = x_t Wsh^T.

    x [N, D]; Wq [G, E, d, D]; Wsh [n_shared*d, D]; idx [N, G, k]
    -> q_routed [B, G, T, k, d] (slot j holds expert idx[t, g, j]),
       q_sh [B, T, d] (or None without a shared head).
    """
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    xf = f64(x).reshape(B * T, -1)
    Wqf = f64(Wq)
    q = np.empty((B * T, G, k, d))
    for g in range(G):
        for j in range(k):
            e_of_row = idx[:, g, j]
            for e in np.unique(e_of_row):
                rows = np.nonzero(e_of_row == e)[0]
                q[rows, g, j] = xf[rows] @ Wqf[g, e].T
    q_routed = q.reshape(B, T, G, k, d).transpose(0, 2, 1, 3, 4)
    q_sh = None
    if dims.n_shared:
        q_sh = (xf @ f64(Wsh).T).reshape(B, T, d)
    return np.ascontiguousarray(q_routed), q_sh


def kv_proj(x, Wk, Wv, dims):
    """Dense, unchanged GQA K/V: K_g = x Wk[g]^T, V_g = x Wv[g]^T -> [B, G, T, d]."""
    B, T, G, d = dims.B, dims.T, dims.G, dims.d
    xf = f64(x).reshape(B * T, -1)
    K = (xf @ f64(Wk).T).reshape(B, T, G, d).transpose(0, 2, 1, 3)
    V = (xf @ f64(Wv).T).reshape(B, T, G, d).transpose(0, 2, 1, 3)
    return np.ascontiguousarray(K), np.ascontiguousarray(V)


# ----------------------------------------------------------------------------
# attention: [SN] §1-1 (softmax(QK^T/sqrt(d))V), causal

def attention_scale(dims) -> float:
    """Factor applied to q.K before the softmax: the layer's explicit scale
    when it sets one, else 1/sqrt(d) ([SN] §1-1, the attention equation)."""
    return float(dims.scale) if dims.scale else 1.0 / math.sqrt(dims.d)


def causal_attention(q, pos, K, V, scale, chunk=2048, want_lse=False):
    """o_r = sum_{j <= pos_r} softmax_j(q_r . K_j * scale) V_j.

    q [R, d] query rows, pos [R] the token position of each row, K, V [L, d].
    Rows are processed in chunks (exact: each row's softmax is its own).
    Returns o [R, d] (and the natural-log LSE of the scaled scores).
    """
    q = f64(q)
    K = f64(K)
    V = f64(V)
    R = q.shape[0]
    o = np.empty((R, V.shape[1]))
    lse = np.empty(R)
    for r0 in range(0, R, chunk):
        r1 = min(R, r0 + chunk)
        pmax = int(pos[r0:r1].max())
        s = (q[r0:r1] @ K[: pmax + 1].T) * scale
        mask = np.arange(pmax + 1)[None, :] > pos[r0:r1, None]
        s[mask] = -np.inf
        m = s.max(axis=1, keepdims=True)
        z = np.exp(s - m)
        den = z.sum(axis=1, keepdims=True)
        o[r0:r1] = (z @ V[: pmax + 1]) / den
        lse[r0:r1] = (m + np.log(den))[:, 0]
    return (o, lse) if want_lse else o


def attn_prefill(q_routed, q_sh, K, V, dims, chunk=2048):
    """Every selected expert and the shared head attend causally to its group's K/V.

    q_routed [B, G, T, k, d] against K, V [B, G, T, d] of the same group
    ([SN] §3-2 2), "selected experts ... attend to the same dense KV head");
    q_sh [B, T, d] against group sg ([SN] §3-2 5), reading: KV group sg).
    Returns o_routed [B, G, T, k, d], o_sh [B, T, d] or None, and the LSEs.
    """
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    sc = attention_scale(dims)
    o = np.empty((B, G, T, k, d))
    lse = np.empty((B, G, T, k))
    pos = np.repeat(np.arange(T), k)
    for b in range(B):
        for g in range(G):
            ob, lb = causal_attention(np.asarray(q_routed[b, g]).reshape(T * k, d), pos,
                                      K[b, g], V[b, g], sc, chunk, want_lse=True)
            o[b, g] = ob.reshape(T, k, d)
            lse[b, g] = lb.reshape(T, k)
    o_sh = lse_sh = None
    if dims.n_shared:
        o_sh = np.empty((B, T, d))
        lse_sh = np.empty((B, T))
        for b in range(B):
            o_sh[b], lse_sh[b] = causal_attention(q_sh[b], np.arange(T), K[b, dims.sg],
                                                  V[b, dims.sg], sc, chunk, want_lse=True)
    return o, o_sh, lse, lse_sh


def attn_decode(q_routed, q_sh, Kc, Vc, cache_len, dims):
    """One new query row per sequence against the whole cache ([FG] decode note).

    q_routed [B, G, k, d], q_sh [B, d]; Kc, Vc [B, G, L_max, d];
    cache_len [B] valid rows (the new token's own K/V included, at row
    cache_len-1).  Returns o_routed [B, G, k, d], o_sh [B, d] or None.
    """
    B, G, k, d = q_routed.shape
    sc = attention_scale(dims)
    o = np.empty((B, G, k, d))
    o_sh = np.empty((B, d)) if dims.n_shared else None
    for b in range(B):
        n = int(cache_len[b])
        pos = np.full(k, n - 1)
        for g in range(G):
            o[b, g] = causal_attention(q_routed[b, g], pos, Kc[b, g, :n], Vc[b, g, :n], sc)
        if dims.n_shared:
            o_sh[b] = causal_attention(np.asarray(q_sh[b])[None, :], np.array([n - 1]),
                                       Kc[b, dims.sg, :n], Vc[b, dims.sg, :n], sc)[0]
    return o, o_sh


# ----------------------------------------------------------------------------
# output construction: [SN] §3-2 3) 4) 5) and the final concat

def combine(o_routed, o_sh, w, dims):
    """h_t = Concat(h_hard, h_route, h_shared).

    h_hard  = the selected o_{t,g,e}, group by group, each in its own slot
              ([SN] §3-2 3), never averaged);
    h_route = sum_g sum_{e in S} p~_{t,g,e} o_{t,g,e}  ([SN] §3-2 4));
    h_shared = the shared head's output ([SN] §3-2 5)).
    o_routed [B, G, T, k, d] (or decode [B, G, k, d] with T=1), w [N, G, k]
    -> h [N, slots * d], slots = k*G + 1 + n_shared.

    output_mode 1 ([SN] §5-1, "hard concat only"): h = [h_hard, h_shared];
    output_mode 2 ([SN] §5-1, "weighted concat, no renormalised slot"):
    h = [w_{t,g,e} o_{t,g,e} slot by slot, h_shared].
    """
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    mode = getattr(dims, "output_mode", 0)
    o = f64(o_routed).reshape(B, G, T, k, d).transpose(0, 2, 1, 3, 4).reshape(B * T, G, k, d)
    if mode == 2:
        parts = [(f64(w)[..., None] * o).reshape(B * T, G * k * d)]
    else:
        parts = [o.reshape(B * T, G * k * d)]
    if mode == 0:
        parts.append(np.einsum("ngk,ngkd->nd", f64(w), o))
    if dims.n_shared:
        parts.append(f64(o_sh).reshape(B * T, d))
    return np.concatenate(parts, axis=1)


def out_proj(h, Wo):
    """y = h Wo^T over the slots of h ([SN] §3-2 7))."""
    return linear(h, Wo)


# ----------------------------------------------------------------------------
# whole layer

def gqe_forward(x, Wt, dims, bias=None):
    """The full prefill layer in fp64, no intermediate rounding.

    x [B, T, D] (bf16 bits or float); Wt: dict of Wr, Wq, Wk, Wv, Wsh, Wo.
    """
    B, T = dims.B, dims.T
    xf = f64(x).reshape(B * T, -1)
    r = router_topk(xf, Wt["Wr"], dims.G, dims.E, dims.k, bias, dims.renorm_scope)
    q_routed, q_sh = routed_qproj(xf, Wt["Wq"], Wt["Wsh"], r["idx"], dims)
    K, V = kv_proj(xf, Wt["Wk"], Wt["Wv"], dims)
    o, o_sh, _, _ = attn_prefill(q_routed, q_sh, K, V, dims)
    h = combine(o, o_sh, r["w"], dims)
    y = out_proj(h, Wt["Wo"])
    return dict(router=r, q_routed=q_routed, q_sh=q_sh, K=K, V=V, o=o, o_sh=o_sh, h=h, y=y)


def gqe_forward_rows(x, Wt, dims, rows, bias=None, chunk=2048):
    """The prefill layer at chosen token rows only, in fp64.

    A token's row of h and y is made of its own router decision, its own
    query projections, and attention of those queries over the keys and
    values of tokens 0..t of its own sequence; K and V are the dense GQA
    projections of that prefix ([SN] §1-2 3), KV unchanged).  Nothing else of
    the batch enters the row, so each requested row is the full layer's row,
    computed from x[b, :t+1] alone.  This is the full-layer definition
    restricted to those rows; used where gqe_forward over a whole workload
    would take too long.

    x [B, T, D]; rows: iterable of (b, t).  Returns dict(router over the rows,
    h [R, slots*d], y [R, D]) in the order of ``rows``.
    """
    rows = [(int(b), int(t)) for b, t in rows]
    R = len(rows)
    G, E, k, d = dims.G, dims.E, dims.k, dims.d
    x = np.asarray(x)
    xr = np.stack([f64(x[b, t]) for b, t in rows])
    r = router_topk(xr, Wt["Wr"], G, E, k, bias, dims.renorm_scope)
    one = _Shape(B=R, T=1, G=G, k=k, d=d, n_shared=dims.n_shared, output_mode=getattr(dims, "output_mode", 0))
    q_routed, q_sh = routed_qproj(xr, Wt["Wq"], Wt["Wsh"], r["idx"], one)     # [R, G, 1, k, d], [R, 1, d]
    sc = attention_scale(dims)
    o = np.empty((R, G, 1, k, d))
    o_sh = np.empty((R, 1, d)) if dims.n_shared else None
    for b in sorted({b for b, _ in rows}):
        mine = [i for i, (bb, _) in enumerate(rows) if bb == b]
        t_end = max(rows[i][1] for i in mine) + 1
        pre = _Shape(B=1, T=t_end, G=G, d=d)
        K, V = kv_proj(x[b, :t_end], Wt["Wk"], Wt["Wv"], pre)                 # [1, G, t_end, d]
        for i in mine:
            t = rows[i][1]
            for g in range(G):
                o[i, g, 0] = causal_attention(q_routed[i, g, 0], np.full(k, t), K[0, g, :t + 1],
                                              V[0, g, :t + 1], sc, chunk)
            if dims.n_shared:
                o_sh[i] = causal_attention(q_sh[i], np.array([t]), K[0, dims.sg, :t + 1],
                                           V[0, dims.sg, :t + 1], sc, chunk)
    h = combine(o, o_sh, r["w"], one)
    y = out_proj(h, Wt["Wo"])
    return dict(router=r, h=h, y=y)


class _Shape:
    """The shape fields the helpers above read, for a sub-batch of rows."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def decode_step(x_new, Wt, Kc, Vc, cache_len, dims, bias=None):
    """One decode step for B sequences (T = 1).

    The new token's K/V rows are projected and written at row cache_len-1 of
    a copy of the cache; every selected expert and the shared head then attend
    over rows [0, cache_len).
    """
    B = dims.B
    xf = f64(x_new).reshape(B, -1)
    r = router_topk(xf, Wt["Wr"], dims.G, dims.E, dims.k, bias, dims.renorm_scope)
    q_routed, q_sh = routed_qproj(xf, Wt["Wq"], Wt["Wsh"], r["idx"], dims)   # [B,G,1,k,d]
    Knew, Vnew = kv_proj(xf, Wt["Wk"], Wt["Wv"], dims)                        # [B,G,1,d]
    Kc = f64(Kc).copy()
    Vc = f64(Vc).copy()
    for b in range(B):
        n = int(cache_len[b])
        Kc[b, :, n - 1] = Knew[b, :, 0]
        Vc[b, :, n - 1] = Vnew[b, :, 0]
    o, o_sh = attn_decode(q_routed[:, :, 0], None if q_sh is None else q_sh[:, 0],
                          Kc, Vc, cache_len, dims)
    h = combine(o[:, :, None], o_sh, r["w"], dims)
    y = out_proj(h, Wt["Wo"])
    return dict(router=r, q_routed=q_routed, q_sh=q_sh, Knew=Knew, Vnew=Vnew,
                o=o, o_sh=o_sh, h=h, y=y)


def near_tie_alternatives(r, k):
    """For (token, group) pairs whose k-th/(k+1)-th logit margin is below 1e-4,
    the set of experts whose choice is numerically undecided.

    Returns a dict (t, g) -> (sure experts, undecided experts).
    """
    out = {}
    s = r["logits"]
    E = s.shape[-1]
    if k >= E:
        return out
    for t, g in zip(*np.nonzero(r["margin"] < 1e-4)):
        srt = -np.sort(-s[t, g])
        kth = srt[k - 1]
        close = np.abs(s[t, g] - kth) < 1e-4
        sure = np.nonzero((s[t, g] > kth) & ~close)[0]
        out[(int(t), int(g))] = (sure, np.nonzero(close)[0])
    return out
