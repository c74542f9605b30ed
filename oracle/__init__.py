"""fp64 CPU oracle of the GQE attention forward and backward (test infrastructure only).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package; the product path never does.
"""
from .gqe_oracle import (  # noqa: F401
    f64, router_logits, group_softmax, topk_select, selection_margin, renormalise,
    router_topk, router_stats, linear, routed_qproj, kv_proj, causal_attention, attn_prefill,
    attn_decode, attention_scale, combine, out_proj, gqe_forward, gqe_forward_rows, decode_step, near_tie_alternatives,
)
from . import gqe_backward  # noqa: F401,E402
