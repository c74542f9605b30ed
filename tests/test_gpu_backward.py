"""Parity of the backward calls with the fp64 backward oracle (GPU).

The backward oracle is pinned by finite differences of the forward oracle
(tests/test_oracle_backward_pins.py).  Each call gets the same bf16 inputs as
the oracle.  Gradients are held to the rounding bound of their arithmetic
(helpers.assert_close_grad): per element 2^-8 (|ref| + sum of the magnitudes
of its products), i.e. half an ulp of bf16 on every MMA operand and on the
output, plus a mean-abs check of 2e-3 of the reference's rms.
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
    return dq, dqs, dK, dV, to_f64(o), to_f64(os_) if sh else None


ATTN_BWD_SMALL = {
    "tiny": D(),
    "ragged_k2_sg1": D(B=2, T=200, G=3, E=3, k=2, sg=1),
    "k1_multi_tile": D(B=1, T=520, G=2, E=2, k=1, sg=1),
    "k3_no_shared": D(B=2, T=50, G=1, E=3, k=3, n_shared=0),
    "single_token": D(B=2, T=1, G=2, E=2, k=2),
    "k8_E8": D(B=1, T=70, G=1, E=8, k=8),
    "k4_E8_ragged": D(B=1, T=300, G=2, E=8, k=4),
}


@pytest.mark.parametrize("case", list(ATTN_BWD_SMALL))
def test_attn_bwd_small(case):
    dims = ATTN_BWD_SMALL[case]
    q, qs, K, V, dO, dOs = _attn_bwd_inputs(dims, 21)
    dq, dqs, dK, dV, o, os_ = _run_attn_bwd(dims, q, qs, K, V, dO, dOs)
    # per-call parity: Delta from the bf16 forward output the call received
    args = (q, qs if dims.n_shared else None, K, V, dO, dOs if dims.n_shared else None, dims, o, os_)
    r_dq, r_dqs, r_dK, r_dV = ob.attn_prefill_bwd(*args)
    m_dq, m_dqs, m_dK, m_dV = ob.attn_prefill_bwd_magnitudes(*args)
    errs = [assert_close_grad(to_f64(dq), r_dq, m_dq, "dq_routed"), assert_close_grad(to_f64(dK), r_dK, m_dK, "dK"),
            assert_close_grad(to_f64(dV), r_dV, m_dV, "dV")]
    if dims.n_shared:
        errs.append(assert_close_grad(to_f64(dqs), r_dqs, m_dqs, "dq_sh"))
    print(f"[attn bwd {case}] err/bound, mean/rms:", [(f"{a:.2f}", f"{b:.2e}") for a, b in errs])


def test_attn_bwd_full_size_sampled():
    """The main prefill workload in the bench's launch configuration; dK, dV and
    dq of two whole KV sequences (one of them the shared head's group) against
    the oracle computed per sequence."""
    dims = gi.WORKLOADS["main_prefill"].dims
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    q, qs, K, V, dO, dOs = _attn_bwd_inputs(dims, 22)
    dq, dqs, dK, dV, o, os_ = _run_attn_bwd(dims, q, qs, K, V, dO, dOs)
    g_dq, g_dqs, g_dK, g_dV = to_f64(dq), to_f64(dqs), to_f64(dK), to_f64(dV)
    pos = np.repeat(np.arange(T), k)
    for b, g in [(0, dims.sg), (B - 1, G - 1)]:
        args = (q[b, g].reshape(T * k, d), pos, K[b, g], V[b, g], dO[b, g].reshape(T * k, d), dims.sm_scale,
                o[b, g].reshape(T * k, d))
        a, bk, bv = ob.causal_attention_bwd(*args)
        ma, mk, mv = ob.causal_attention_bwd_magnitudes(*args)
        if g == dims.sg:
            args2 = (qs[b], np.arange(T), K[b, g], V[b, g], dOs[b], dims.sm_scale, os_[b])
            a2, bk2, bv2 = ob.causal_attention_bwd(*args2)
            ma2, mk2, mv2 = ob.causal_attention_bwd_magnitudes(*args2)
            bk, bv, mk, mv = bk + bk2, bv + bv2, mk + mk2, mv + mv2
            assert_close_grad(g_dqs[b], a2, ma2, "dq_sh")
        assert_close_grad(g_dq[b, g].reshape(T * k, d), a, ma, "dq_routed")
        assert_close_grad(g_dK[b, g], bk, mk, "dK")
        assert_close_grad(g_dV[b, g], bv, mv, "dV")
    for t in (dq, dqs, dK, dV):
        assert torch.isfinite(t.float()).all()
