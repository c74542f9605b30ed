"""Plain fp64 CPU oracle of the GQE layer's backward pass.

TEST INFRASTRUCTURE ONLY, like the forward oracle beside it: only the test
suite, the smoke check and the benchmark's CPU legs use it, and it shares no
code with the CUDA library.

Each function is the derivative of one forward step of gqe_oracle.py, written
out by the chain rule from that step's definition ([SN] "GQE" study note
§3-2 items 2)-7) and §1-1; [SN] §4-1 for the reason the weighted-sum slot
exists: it is the path on which the router receives a gradient).  Readings
where the pages leave the backward open:
  * TopK is piecewise constant: the selection S_{t,g} receives no gradient,
    the router learns only through the selected probabilities in the
    weighted-sum slot (output_mode 0) or the weighted hard slots (mode 2).
    In output_mode 1 the router receives no gradient at all.
  * the shared head has no K/V of its own, so its dK/dV land in group sg.

Pinned by tests/test_oracle_backward_pins.py: central finite differences in
fp64 of every forward step and of the whole layer (inputs chosen with TopK
margins far above the step size, so the selection does not move), torch
autograd through a library attention, and closed forms (constant values give
dq = dK = 0; in-group softmax gradients sum to zero; renormalisation is scale
invariant; output_mode 1 gives the router nothing).
"""
from __future__ import annotations

import numpy as np

from .gqe_oracle import (
    f64, router_logits, group_softmax, topk_select, renormalise, routed_qproj,
    kv_proj, attn_prefill, attention_scale, combine,
)


# ----------------------------------------------------------------------------
# attention: [SN] §1-1, o = softmax(q K^T * scale) V, causal

def causal_attention_bwd(q, pos, K, V, dO, scale, O=None, lse=None):
    """Gradients of o_r = sum_{j <= pos_r} P_rj V_j, P = softmax_j(q_r . K_j * scale).

    With S = q K^T * scale (masked to j <= pos_r) and P its row softmax:
      dV = P^T dO,   dP = dO V^T,
      dS_rj = P_rj (dP_rj - Delta_r)                    (softmax Jacobian),
      Delta_r = sum_i P_ri dP_ri = dO_r . o_r,
      dq = scale * dS K,   dK = scale * dS^T q.
    Delta is the first sum unless the forward output O is given, then the
    second; P is the softmax unless the forward's log-sum-exp is given, then
    exp(S - lse) (both identical for the exact O and lse; a call that
    receives rounded ones computes from those).
    q, dO [R, d]; pos [R]; K, V [L, d].  Returns dq [R, d], dK, dV [L, d].
    """
    q, K, V, dO = f64(q), f64(K), f64(V), f64(dO)
    P = _probs(q, pos, K, scale, lse)
    dV = P.T @ dO
    dP = dO @ V.T
    if O is None:
        delta = np.sum(P * dP, axis=1, keepdims=True)
    else:
        delta = np.sum(dO * f64(O), axis=1, keepdims=True)
    dS = P * (dP - delta)
    return scale * (dS @ K), scale * (dS.T @ q), dV


def _probs(q, pos, K, scale, lse=None):
    s = (q @ K.T) * scale
    s[np.arange(K.shape[0])[None, :] > np.asarray(pos)[:, None]] = -np.inf
    if lse is not None:
        return np.exp(s - np.asarray(lse, dtype=np.float64)[:, None])
    z = np.exp(s - s.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def causal_attention_bwd_error_bound(q, pos, K, V, dO, scale, O=None, lse=None):
    """Worst-case error of causal_attention_bwd's outputs when computed as a
    tensor-core kernel does it: S, dP, Delta and the three gradient products
    accumulated in fp32, the MMA operands P and dS rounded to bf16.  Before
    the final bf16 rounding of the results (which adds 2^-8 |result|).

    With u = 2^-8 (bf16 rounding) and g_n = n 2^-24 (an fp32 sum of n
    products errs by at most g_n times the sum of their magnitudes):
      err P    <= P scale g_d sum|q||K|                      (S in fp32)
      err dS   <= scale (|dP - Delta| err P + P g_d (sum|dO||V| + sum|dO||O|))
      dq: sum_j ((u + g_L) |scale dS| + err dS) |K_j|,  dK likewise with |q_r|,
      dV: sum_r ((u + g_R) P + err P) |dO_r|.
    Returns (bound_dq, bound_dK, bound_dV), absolute, shaped like the outputs.
    """
    q, K, V, dO = f64(q), f64(K), f64(V), f64(dO)
    R, d = q.shape
    L = K.shape[0]
    P = _probs(q, pos, K, scale, lse)
    dP = dO @ V.T
    Of = f64(O) if O is not None else P @ V
    delta = np.sum(dO * Of, axis=1, keepdims=True)
    gd, gL, gR = d * 2.0 ** -24, L * 2.0 ** -24, R * 2.0 ** -24
    u = 2.0 ** -8
    aq, aK, aV, adO = np.abs(q), np.abs(K), np.abs(V), np.abs(dO)
    eP = P * scale * gd * (aq @ aK.T)
    edS = scale * (np.abs(dP - delta) * eP + P * gd * (adO @ aV.T + np.sum(adO * np.abs(Of), axis=1, keepdims=True)))
    aS = np.abs(scale * P * (dP - delta))
    b_dq = ((u + gL) * aS + edS) @ aK
    b_dK = ((u + gR) * aS + edS).T @ aq
    b_dV = ((u + gR) * P + eP).T @ adO
    return b_dq, b_dK, b_dV


def attn_prefill_bwd_error_bound(q_routed, q_sh, K, V, do_routed, do_sh, dims, o_routed=None, o_sh=None,
                                 lse=None):
    """causal_attention_bwd_error_bound laid out like attn_prefill_bwd's
    outputs.  lse: the forward's fp32 log-sum-exp in gqe_attn_prefill's layout
    (routed rows, then shared rows), or None."""
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    sc = attention_scale(dims)
    R = T * k
    pos = np.repeat(np.arange(T), k)
    mq = np.empty((B, G, T, k, d))
    mK = np.zeros((B, G, T, d))
    mV = np.zeros((B, G, T, d))
    for b in range(B):
        for g in range(G):
            o_rows = None if o_routed is None else np.asarray(o_routed[b, g]).reshape(R, d)
            l_rows = None if lse is None else np.asarray(lse)[(b * G + g) * R:(b * G + g + 1) * R]
            a, bk, bv = causal_attention_bwd_error_bound(np.asarray(q_routed[b, g]).reshape(R, d), pos, K[b, g],
                                                         V[b, g], np.asarray(do_routed[b, g]).reshape(R, d), sc,
                                                         o_rows, l_rows)
            mq[b, g] = a.reshape(T, k, d)
            mK[b, g] += bk
            mV[b, g] += bv
    mqs = None
    if dims.n_shared:
        mqs = np.empty((B, T, d))
        for b in range(B):
            l_rows = None if lse is None else np.asarray(lse)[B * G * R + b * T:B * G * R + (b + 1) * T]
            a, bk, bv = causal_attention_bwd_error_bound(q_sh[b], np.arange(T), K[b, dims.sg], V[b, dims.sg],
                                                         do_sh[b], sc, None if o_sh is None else o_sh[b], l_rows)
            mqs[b] = a
            mK[b, dims.sg] += bk
            mV[b, dims.sg] += bv
    return mq, mqs, mK, mV


def attn_prefill_bwd(q_routed, q_sh, K, V, do_routed, do_sh, dims, o_routed=None, o_sh=None, lse=None):
    """Backward of attn_prefill: every selected expert's rows and the shared
    head's rows send their dK/dV into the KV group they read ([SN] §3-2 2), 5)).

    q_routed, do_routed [B, G, T, k, d]; q_sh, do_sh [B, T, d] or None;
    K, V [B, G, T, d]; o_routed, o_sh: the forward output to take Delta from,
    lse: the forward's log-sum-exp in gqe_attn_prefill's layout to take P
    from (see causal_attention_bwd), or None.  Returns dq_routed, dq_sh, dK, dV.
    """
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    sc = attention_scale(dims)
    R = T * k
    pos = np.repeat(np.arange(T), k)
    dq = np.empty((B, G, T, k, d))
    dK = np.zeros((B, G, T, d))
    dV = np.zeros((B, G, T, d))
    for b in range(B):
        for g in range(G):
            o_rows = None if o_routed is None else np.asarray(o_routed[b, g]).reshape(R, d)
            l_rows = None if lse is None else np.asarray(lse)[(b * G + g) * R:(b * G + g + 1) * R]
            a, bk, bv = causal_attention_bwd(np.asarray(q_routed[b, g]).reshape(R, d), pos, K[b, g], V[b, g],
                                             np.asarray(do_routed[b, g]).reshape(R, d), sc, o_rows, l_rows)
            dq[b, g] = a.reshape(T, k, d)
            dK[b, g] += bk
            dV[b, g] += bv
    dq_sh = None
    if dims.n_shared:
        dq_sh = np.empty((B, T, d))
        for b in range(B):
            l_rows = None if lse is None else np.asarray(lse)[B * G * R + b * T:B * G * R + (b + 1) * T]
            a, bk, bv = causal_attention_bwd(q_sh[b], np.arange(T), K[b, dims.sg], V[b, dims.sg], do_sh[b], sc,
                                             None if o_sh is None else o_sh[b], l_rows)
            dq_sh[b] = a
            dK[b, dims.sg] += bk
            dV[b, dims.sg] += bv
    return dq, dq_sh, dK, dV


# ----------------------------------------------------------------------------
# output construction: [SN] §3-2 3) 4) 5)

def combine_bwd(o_routed, o_sh, w, dh, dims):
    """Backward of combine.

    output_mode 0: the hard slot of (t, g, j) passes dh straight to o_{t,g,j};
      the weighted-sum slot h_route = sum p~ o gives o_{t,g,j} another
      p~_{t,g,j} dh_route and p~_{t,g,j} the gradient <dh_route, o_{t,g,j}>.
    output_mode 1: hard slots only, p~ receives nothing.
    output_mode 2: slot (t, g, j) holds p~ o, so o gets p~ dh_slot and p~ gets
      <dh_slot, o>.
    The shared slot passes its gradient to o_sh.
    dh [N, slots*d] -> do_routed [B, G, T, k, d], do_sh [B, T, d] or None, dw [N, G, k].
    """
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    mode = getattr(dims, "output_mode", 0)
    N = B * T
    o = f64(o_routed).reshape(B, G, T, k, d).transpose(0, 2, 1, 3, 4).reshape(N, G, k, d)
    wf = f64(w)
    dhf = f64(dh)
    hard = dhf[:, : G * k * d].reshape(N, G, k, d)
    col = G * k * d
    if mode == 2:
        do = wf[..., None] * hard
        dw = np.einsum("ngkd,ngkd->ngk", hard, o)
    else:
        do = hard.copy()
        dw = np.zeros((N, G, k))
    if mode == 0:
        dr = dhf[:, col: col + d]
        col += d
        do = do + wf[..., None] * dr[:, None, None, :]
        dw = np.einsum("nd,ngkd->ngk", dr, o)
    do_sh = None
    if dims.n_shared:
        do_sh = dhf[:, col: col + d].reshape(B, T, d).copy()
    do_routed = np.ascontiguousarray(do.reshape(B, T, G, k, d).transpose(0, 2, 1, 3, 4))
    return do_routed, do_sh, dw


# ----------------------------------------------------------------------------
# router: [SN] §3-2 2) and 4)

def renormalise_bwd(p, sel, dw, scope=0):
    """Backward of renormalise: dw [N, G, k] on p~ -> dp [N, G, E] on p.

    p~_i = p_i / Z with Z the sum over the scope's selected p; hence
    dp_i = (dw_i - sum_{j in scope} dw_j p~_j) / Z for selected i, 0 for the
    rest.  Scope 2 (no renormalisation): dp_i = dw_i.
    """
    N, G, E = p.shape
    sel = sel.astype(np.int64)
    psel = np.take_along_axis(p, sel, axis=-1)
    dw = f64(dw)
    if scope == 2:
        dsel = dw
    else:
        axes = (1, 2) if scope == 0 else (2,)
        Z = psel.sum(axis=axes, keepdims=True)
        wt = psel / Z
        dsel = (dw - np.sum(dw * wt, axis=axes, keepdims=True)) / Z
    dp = np.zeros((N, G, E))
    np.put_along_axis(dp, sel, dsel, axis=-1)
    return dp


def group_softmax_bwd(p, dp):
    """Backward of group_softmax: ds_e = p_e (dp_e - sum_e' p_e' dp_e') per group."""
    return p * (dp - np.sum(p * dp, axis=-1, keepdims=True))


def router_bwd(x, Wr, probs, idx, dw, scope=0):
    """dw on the router weights -> (dx, dWr, dbias) through renormalisation,
    the in-group softmax and the linear map s = x Wr + bias.  TopK passes no
    gradient (its output is a set)."""
    N, G, E = probs.shape
    ds = group_softmax_bwd(probs, renormalise_bwd(probs, idx, dw, scope)).reshape(N, G * E)
    xf = f64(x)
    return ds @ f64(Wr).T, xf.T @ ds, ds.sum(axis=0)


# ----------------------------------------------------------------------------
# projections: y = x W^T

def linear_bwd(x, W, dy):
    """y = x W^T: dx = dy W, dW = dy^T x."""
    dy = f64(dy)
    return dy @ f64(W), dy.T @ f64(x)


def routed_qproj_bwd(x, Wq, Wsh, idx, dq_routed, dq_sh, dims):
    """Backward of routed_qproj: a selected (t, g, j) with expert e sends
    dq W_q[g,e] to dx_t and dq^T x_t to dW_q[g,e]; unselected experts receive
    nothing.  Returns dx [N, D], dWq [G, E, d, D], dWsh or None."""
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    xf = f64(x).reshape(B * T, -1)
    Wqf = f64(Wq)
    dq = f64(dq_routed).reshape(B, G, T, k, d).transpose(0, 2, 1, 3, 4).reshape(B * T, G, k, d)
    dx = np.zeros_like(xf)
    dWq = np.zeros_like(Wqf)
    for g in range(G):
        for j in range(k):
            e_of_row = idx[:, g, j]
            for e in np.unique(e_of_row):
                rows = np.nonzero(e_of_row == e)[0]
                dx[rows] += dq[rows, g, j] @ Wqf[g, e]
                dWq[g, e] += dq[rows, g, j].T @ xf[rows]
    dWsh = None
    if dims.n_shared:
        a, dWsh = linear_bwd(xf, Wsh, f64(dq_sh).reshape(B * T, d))
        dx += a
    return dx, dWq, dWsh


def kv_proj_bwd(x, Wk, Wv, dK, dV, dims):
    """Backward of kv_proj (K_g = x Wk[g]^T, V_g = x Wv[g]^T)."""
    B, T, G, d = dims.B, dims.T, dims.G, dims.d
    xf = f64(x).reshape(B * T, -1)
    dKf = f64(dK).transpose(0, 2, 1, 3).reshape(B * T, G * d)
    dVf = f64(dV).transpose(0, 2, 1, 3).reshape(B * T, G * d)
    a, dWk = linear_bwd(xf, Wk, dKf)
    b, dWv = linear_bwd(xf, Wv, dVf)
    return a + b, dWk, dWv


# ----------------------------------------------------------------------------
# whole layer

def gqe_backward(x, Wt, dims, dy, bias=None):
    """Gradients of L = <y, dy> for the prefill layer (fp64, no rounding).

    Returns a dict with dx [N, D] and dWr, dbias, dWq, dWk, dWv, dWsh, dWo,
    plus the intermediate gradients (dh, do_routed, do_sh, dw, dq_routed,
    dq_sh, dK, dV) for per-step comparisons.
    """
    B, T = dims.B, dims.T
    xf = f64(x).reshape(B * T, -1)
    G, E, k = dims.G, dims.E, dims.k
    s = router_logits(xf, Wt["Wr"], bias).reshape(-1, G, E)
    p = group_softmax(s)
    idx = topk_select(p, k)
    w = renormalise(p, idx, dims.renorm_scope)
    q_routed, q_sh = routed_qproj(xf, Wt["Wq"], Wt["Wsh"], idx, dims)
    K, V = kv_proj(xf, Wt["Wk"], Wt["Wv"], dims)
    o, o_sh, _, _ = attn_prefill(q_routed, q_sh, K, V, dims)
    h = combine(o, o_sh, w, dims)

    dyf = f64(dy).reshape(B * T, -1)
    dh, dWo = linear_bwd(h, Wt["Wo"], dyf)
    do_routed, do_sh, dw = combine_bwd(o, o_sh, w, dh, dims)
    dq_routed, dq_sh, dK, dV = attn_prefill_bwd(q_routed, q_sh, K, V, do_routed, do_sh, dims)
    dx_q, dWq, dWsh = routed_qproj_bwd(xf, Wt["Wq"], Wt["Wsh"], idx, dq_routed, dq_sh, dims)
    dx_kv, dWk, dWv = kv_proj_bwd(xf, Wt["Wk"], Wt["Wv"], dK, dV, dims)
    dx_r, dWr, dbias = router_bwd(xf, Wt["Wr"], p, idx, dw, dims.renorm_scope)
    return dict(dx=dx_q + dx_kv + dx_r, dWr=dWr, dbias=dbias, dWq=dWq, dWk=dWk, dWv=dWv, dWsh=dWsh,
                dWo=dWo, dh=dh, do_routed=do_routed, do_sh=do_sh, dw=dw, dq_routed=dq_routed,
                dq_sh=dq_sh, dK=dK, dV=dV, probs=p, idx=idx, w=w, o=o, o_sh=o_sh, h=h,
                q_routed=q_routed, q_sh=q_sh, K=K, V=V)
