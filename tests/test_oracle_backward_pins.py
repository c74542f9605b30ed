"""Pins of the fp64 backward oracle (CPU only).

Every gradient the oracle writes out by the chain rule is checked against
central finite differences of the pinned forward oracle, along random
directions, in fp64: a dropped term, a wrong sign, a transposed operand or a
gradient sent to the wrong KV group fails one of them.  A few closed forms
(constant values, scale invariance of the renormalisation, zero-sum softmax
gradients) and a library autograd attention pin the same functions from a
second side.
"""
import numpy as np
import pytest
import torch

import gqe_inputs as gi
import oracle as orc
from oracle import gqe_backward as ob


def _dims(**kw):
    base = dict(B=2, T=8, D=16, G=2, E=3, k=2, d=4)
    base.update(kw)
    return gi.GQEDims(**base)


def _fd(f, x, v, eps=1e-5):
    """Central difference of the scalar f along direction v at x."""
    return (f(x + eps * v) - f(x - eps * v)) / (2 * eps)


def _check(f, x, grad, rng, n_dir=3, rtol=1e-6):
    for _ in range(n_dir):
        v = rng.standard_normal(x.shape)
        num = _fd(f, x, v)
        ana = float(np.sum(grad * v))
        assert abs(num - ana) <= rtol * max(1.0, abs(num)), (num, ana)


# ----------------------------------------------------------------------------
# attention: GQE study note §1-1

@pytest.mark.parametrize("k", [1, 3])
def test_attention_gradients_match_finite_differences(k):
    rng = np.random.default_rng(10 + k)
    T, d = 6, 4
    R = T * k
    pos = np.repeat(np.arange(T), k)
    q, K, V, dO = (rng.standard_normal(s) for s in [(R, d), (T, d), (T, d), (R, d)])
    sc = 0.7
    dq, dK, dV = ob.causal_attention_bwd(q, pos, K, V, dO, sc)
    L = lambda q_, K_, V_: float(np.sum(orc.causal_attention(q_, pos, K_, V_, sc) * dO))
    _check(lambda a: L(a, K, V), q, dq, rng)
    _check(lambda a: L(q, a, V), K, dK, rng)
    _check(lambda a: L(q, K, a), V, dV, rng)


def test_delta_and_p_from_the_forward_outputs_are_the_same():
    """Delta_r = sum_j P_rj dP_rj equals dO_r . o_r, and exp(S - lse) equals the
    softmax, for the exact forward output and log-sum-exp."""
    rng = np.random.default_rng(6)
    T, d, k = 7, 4, 2
    pos = np.repeat(np.arange(T), k)
    q, dO = rng.standard_normal((T * k, d)), rng.standard_normal((T * k, d))
    K, V = rng.standard_normal((T, d)), rng.standard_normal((T, d))
    o, lse = orc.causal_attention(q, pos, K, V, 0.6, want_lse=True)
    for a, b in zip(ob.causal_attention_bwd(q, pos, K, V, dO, 0.6),
                    ob.causal_attention_bwd(q, pos, K, V, dO, 0.6, O=o, lse=lse)):
        np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


def test_backward_error_bound_covers_an_emulated_bf16_kernel():
    """The error bound holds for an emulation of the kernel's arithmetic
    (P and dS rounded to bf16 before the products, results rounded to bf16)."""
    rng = np.random.default_rng(7)
    T, d, k = 40, 16, 2
    pos = np.repeat(np.arange(T), k)
    bf = lambda a: gi.bf16_bits_to_f32(gi.f32_to_bf16_bits(np.asarray(a, np.float32))).astype(np.float64)
    q, dO = bf(rng.standard_normal((T * k, d))), bf(rng.standard_normal((T * k, d)))
    K, V = bf(rng.standard_normal((T, d))), bf(rng.standard_normal((T, d)))
    sc = d ** -0.5
    o, lse = orc.causal_attention(q, pos, K, V, sc, want_lse=True)
    o = bf(o)
    ref = ob.causal_attention_bwd(q, pos, K, V, dO, sc, O=o, lse=lse)
    bound = ob.causal_attention_bwd_error_bound(q, pos, K, V, dO, sc, O=o, lse=lse)
    P = np.exp(np.where(np.arange(T)[None, :] > pos[:, None], -np.inf, q @ K.T * sc) - lse[:, None])
    dS = bf(sc * P * (dO @ V.T - np.sum(dO * o, axis=1, keepdims=True)))
    emu = (bf(dS @ K), bf(dS.T @ q), bf(bf(P).T @ dO))
    for e, r, b in zip(emu, ref, bound):
        assert np.all(np.abs(e - r) <= 2.0 ** -8 * np.abs(r) + b + 1e-12)


def test_attention_gradients_match_library_autograd():
    """Standard causal attention (one row per position) against torch autograd
    through scaled_dot_product_attention in float64."""
    rng = np.random.default_rng(3)
    T, d = 9, 8
    q, K, V, dO = (rng.standard_normal((T, d)) for _ in range(4))
    dq, dK, dV = ob.causal_attention_bwd(q, np.arange(T), K, V, dO, 1 / np.sqrt(d))
    tq, tK, tV = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, K, V))
    o = torch.nn.functional.scaled_dot_product_attention(tq[None, None], tK[None, None], tV[None, None],
                                                         is_causal=True)[0, 0]
    o.backward(torch.tensor(dO))
    np.testing.assert_allclose(dq, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, tK.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, tV.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_constant_values_give_zero_query_and_key_gradients():
    """With every V row equal to v, o = v whatever q and K are: dq = dK = 0,
    and dV_j = sum of dO over the rows that see key j weighted by P."""
    rng = np.random.default_rng(4)
    T, d = 7, 4
    q, K, dO = (rng.standard_normal((T, d)) for _ in range(3))
    V = np.tile(rng.standard_normal(d), (T, 1))
    dq, dK, dV = ob.causal_attention_bwd(q, np.arange(T), K, V, dO, 0.5)
    assert np.abs(dq).max() < 1e-13 and np.abs(dK).max() < 1e-13
    # the sum over keys of dV is the sum over rows of dO (rows of P sum to 1)
    np.testing.assert_allclose(dV.sum(axis=0), dO.sum(axis=0), rtol=1e-12)
    # the last key is seen by the last row only
    s = q[-1] @ K.T * 0.5
    p_last = np.exp(s - s.max())
    p_last /= p_last.sum()
    np.testing.assert_allclose(dV[-1], p_last[-1] * dO[-1], rtol=1e-12)


def test_shared_head_gradients_land_in_group_sg():
    rng = np.random.default_rng(5)
    dims = _dims(B=1, T=5, G=3, E=2, k=1, d=4, sg=2)
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    q = rng.standard_normal((B, G, T, k, d))
    qs = rng.standard_normal((B, T, d))
    K, V = rng.standard_normal((B, G, T, d)), rng.standard_normal((B, G, T, d))
    do = np.zeros((B, G, T, k, d))
    dos = rng.standard_normal((B, T, d))
    dq, dqs, dK, dV = ob.attn_prefill_bwd(q, qs, K, V, do, dos, dims)
    assert np.abs(dq).max() == 0
    for g in range(G):
        nz = np.abs(dK[0, g]).max() > 0 and np.abs(dV[0, g]).max() > 0
        assert nz == (g == dims.sg)


# ----------------------------------------------------------------------------
# output construction: GQE study note §3-2 3) 4) 5)

@pytest.mark.parametrize("mode", [0, 1, 2])
def test_combine_gradients_match_finite_differences(mode):
    rng = np.random.default_rng(20 + mode)
    dims = _dims(output_mode=mode)
    B, T, G, k, d = dims.B, dims.T, dims.G, dims.k, dims.d
    o = rng.standard_normal((B, G, T, k, d))
    os_ = rng.standard_normal((B, T, d))
    w = rng.random((B * T, G, k))
    dh = rng.standard_normal((B * T, dims.slots * d))
    do, dos, dw = ob.combine_bwd(o, os_, w, dh, dims)
    L = lambda o_, os2, w_: float(np.sum(orc.combine(o_, os2, w_, dims) * dh))
    _check(lambda a: L(a, os_, w), o, do, rng)
    _check(lambda a: L(o, a, w), os_, dos, rng)
    _check(lambda a: L(o, os_, a), w, dw, rng)
    if mode == 1:
        assert np.abs(dw).max() == 0


# ----------------------------------------------------------------------------
# router: GQE study note §3-2 2) and 4)

@pytest.mark.parametrize("scope", [0, 1, 2])
def test_renormalisation_gradient_matches_finite_differences(scope):
    rng = np.random.default_rng(30 + scope)
    N, G, E, k = 6, 3, 4, 2
    p = rng.random((N, G, E)) + 0.1
    sel = np.sort(np.argsort(rng.random((N, G, E)), axis=-1)[..., :k], axis=-1).astype(np.int32)
    dw = rng.standard_normal((N, G, k))
    dp = ob.renormalise_bwd(p, sel, dw, scope)
    _check(lambda a: float(np.sum(orc.renormalise(a, sel, scope) * dw)), p, dp, rng)
    # unselected experts receive nothing
    mask = np.zeros((N, G, E), bool)
    np.put_along_axis(mask, sel.astype(np.int64), True, axis=-1)
    assert np.abs(dp[~mask]).max() == 0
    if scope in (0, 1):
        # p~ is invariant under scaling p (within the scope): sum_i dp_i p_i = 0
        axes = (1, 2) if scope == 0 else (2,)
        np.testing.assert_allclose(np.sum(dp * p, axis=axes), 0, atol=1e-12)


def test_group_softmax_gradient_matches_finite_differences_and_sums_to_zero():
    rng = np.random.default_rng(40)
    s = rng.standard_normal((5, 3, 4))
    dp = rng.standard_normal(s.shape)
    ds = ob.group_softmax_bwd(orc.group_softmax(s), dp)
    _check(lambda a: float(np.sum(orc.group_softmax(a) * dp)), s, ds, rng)
    np.testing.assert_allclose(ds.sum(axis=-1), 0, atol=1e-13)


# ----------------------------------------------------------------------------
# the whole layer

def _layer_case(seed, **kw):
    dims = _dims(**kw)
    rng = np.random.default_rng(seed)
    D, G, E, d = dims.D, dims.G, dims.E, dims.d
    Wt = dict(Wr=rng.standard_normal((D, G * E)) * 0.5, Wq=rng.standard_normal((G, E, d, D)) * 0.3,
              Wk=rng.standard_normal((G * d, D)) * 0.3, Wv=rng.standard_normal((G * d, D)) * 0.3,
              Wsh=rng.standard_normal((dims.n_shared * d, D)) * 0.3,
              Wo=rng.standard_normal((D, dims.slots * d)) * 0.3)
    x = rng.standard_normal((dims.B, dims.T, D))
    bias = rng.standard_normal(G * E)
    dy = rng.standard_normal((dims.N, D))
    r = orc.router_topk(x.reshape(dims.N, D), Wt["Wr"], G, E, dims.k, bias, dims.renorm_scope)
    assert r["margin"].min() > 1e-3          # the step size cannot move the selection
    return dims, Wt, x, bias, dy, rng


@pytest.mark.parametrize("kw", [dict(), dict(renorm_scope=1), dict(output_mode=2), dict(output_mode=1),
                                dict(n_shared=0, k=1, E=2), dict(sg=1)])
def test_layer_gradients_match_finite_differences(kw):
    dims, Wt, x, bias, dy, rng = _layer_case(50 + len(kw), **kw)
    g = ob.gqe_backward(x, Wt, dims, dy, bias)

    def L(x_=x, b_=bias, **over):
        W = dict(Wt)
        W.update(over)
        return float(np.sum(orc.gqe_forward(x_, W, dims, b_)["y"] * dy))

    _check(lambda a: L(x_=a), x, g["dx"].reshape(x.shape), rng)
    _check(lambda a: L(b_=a), bias, g["dbias"], rng)
    for name in ["Wr", "Wq", "Wk", "Wv", "Wo"] + (["Wsh"] if dims.n_shared else []):
        _check(lambda a, n=name: L(**{n: a}), Wt[name], g["d" + name], rng)
    if dims.output_mode == 1:
        # no path from the router to y: the router weights receive nothing
        assert np.abs(g["dWr"]).max() == 0 and np.abs(g["dbias"]).max() == 0
