"""ctypes binding of libgqe.so (include/gqe.h): argument marshalling only.

Every function here has the name of the C entry point it calls, takes torch
tensors that already live on the GPU (or raw integer pointers), passes their
device pointers, the shape struct and the current CUDA stream to the library,
and raises GQEError on a non-zero status.  No step of the computation happens
in Python.  The library must be built (python moe_gqa_query_b200/build.py);
importing this module without it raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
# GQE_LIB_PATH selects another build of the library (the traced diagnostic
# build, libgqe_trace.so); by default the package's own libgqe.so.
LIB_PATH = os.environ.get("GQE_LIB_PATH") or os.path.join(_PKG, "libgqe.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "gqe.h")

GQE_OK = 0
GQE_OP_ROUTED_QPROJ = 1
GQE_OP_ATTN_DECODE = 2
GQE_OP_COMBINE_OUT_PROJ = 3
GQE_OP_ATTN_BWD = 4
GQE_OP_LAYER_FORWARD = 5
GQE_OP_LAYER_FORWARD_HOST = 6
STATUS_NAMES = {0: "GQE_OK", 1: "GQE_ERR_INVALID_ARG", 2: "GQE_ERR_UNSUPPORTED",
                3: "GQE_ERR_WORKSPACE", 4: "GQE_ERR_CUDA", 5: "GQE_ERR_DEVICE_CHECK"}


class GQEError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


class gqe_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("d_model", ctypes.c_int),
                ("G", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int),
                ("d_head", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("shared_kv_group", ctypes.c_int), ("renorm_scope", ctypes.c_int),
                ("scale", ctypes.c_float), ("output_mode", ctypes.c_int)]


class gqe_layer_weights(ctypes.Structure):
    _fields_ = [("Wr", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("Wq", ctypes.c_void_p),
                ("Wsh", ctypes.c_void_p), ("Wk", ctypes.c_void_p), ("Wv", ctypes.c_void_p),
                ("Wo", ctypes.c_void_p)]


def make_dims(cfg, **override) -> gqe_dims:
    """Shape struct from any object with B, T, D, G, E, k, d (+ n_shared, sg,
    renorm_scope, scale, output_mode) attributes."""
    v = dict(B=cfg.B, T=cfg.T, d_model=cfg.D, G=cfg.G, E=cfg.E, k=cfg.k, d_head=cfg.d,
             n_shared=getattr(cfg, "n_shared", 1), shared_kv_group=getattr(cfg, "sg", 0),
             renorm_scope=getattr(cfg, "renorm_scope", 0), scale=float(getattr(cfg, "scale", 0.0)),
             output_mode=getattr(cfg, "output_mode", 0))
    v.update(override)
    return gqe_dims(**v)


_P = ctypes.c_void_p
_I = ctypes.c_int
_SZ = ctypes.c_size_t
_D = ctypes.POINTER(gqe_dims)
_LW = ctypes.POINTER(gqe_layer_weights)

SIGNATURES = {
    "gqe_workspace_size": [_D, _I, _I, ctypes.POINTER(_SZ)],
    "gqe_router_topk": [_D, _P, _P, _P, _P, _P, _P, _P],
    "gqe_router_stats": [_D, _P, _P, _P, _P, _P],
    "gqe_routed_qproj": [_D, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "gqe_kv_proj": [_D, _P, _P, _P, _P, _P, _P],
    "gqe_kv_append": [_D, _P, _P, _P, _P, _P, _I, _P, _P],
    "gqe_attn_prefill": [_D, _P, _P, _P, _P, _P, _P, _P, _P],
    "gqe_attn_prefill_bwd": [_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "gqe_attn_decode": [_D, _P, _P, _P, _P, _I, _P, _P, _P, _P, _SZ, _P],
    "gqe_attn_decode_noalloc": [_D, _P, _P, _P, _P, _I, _P, _P, _P, _P],
    "gqe_combine": [_D, _P, _P, _P, _P, _P],
    "gqe_combine_out_proj": [_D, _P, _P, _P, _P, _P, _P, _SZ, _P],
    "gqe_layer_forward": [_D, _LW, _P, _P, _P, _SZ, _P],
    "gqe_layer_forward_host": [_D, _LW, _P, _P, _I, _P, _SZ, _P, _P, _P],
    "gqe_linear": [_I, _I, _I, _P, _P, _P, _P],
    "gqe_gemm": [_I, _I, _I, _P, _I, _P, _I, _P, _P],
    "gqe_gemm_acc": [_I, _I, _I, _P, _I, _P, _I, _P, _I, _P],
    "gqe_transpose_f32": [_I, _I, _P, _P, _I, _P],
    "gqe_combine_bwd": [_D, _P, _P, _P, _P, _P, _P, _P, _P],
    "gqe_router_bwd": [_D, _P, _P, _P, _P, _P, _P, _P],
    "gqe_bwd_pack_cols": [_D, ctypes.POINTER(_I)],
    "gqe_bwd_pack": [_D, _P, _P, _P, _P, _P, _P, _P, _P],
    "gqe_bwd_pack_weights": [_D, _P, _P, _P, _P, _P, _P, _P],
    "gqe_transpose": [_I, _I, _P, _P, _I, _P],
    "gqe_device_error": [ctypes.POINTER(_I), _P],
    "gqe_debug_exp2": [_P, _P, _P, _P, _I, _P],
    "gqe_debug_wait_timeout": [_P],
    "gqe_status_string": [_I],
}


def header_functions(path: str = HEADER_PATH):
    """Names of the functions include/gqe.h declares."""
    with open(path) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(gqe_\w+)\s*\(", text, flags=re.M)))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python moe_gqa_query_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, args in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "gqe_status_string" else ctypes.c_int
    return lib


lib = _load()


# ----------------------------------------------------------------------------
# marshalling helpers

def _ptr(t, name="tensor", dtype=None, optional=False):
    if t is None:
        if optional:
            return None
        raise ValueError(f"{name} is required")
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn, st):
    if st != GQE_OK:
        raise GQEError(fn, st)


def _bf16():
    import torch
    return torch.bfloat16


# ----------------------------------------------------------------------------
# the entry points

def gqe_workspace_size(dims: gqe_dims, op: int, L_max: int = 0) -> int:
    n = _SZ(0)
    _check("gqe_workspace_size", lib.gqe_workspace_size(ctypes.byref(dims), op, L_max, ctypes.byref(n)))
    return int(n.value)


def gqe_router_topk(dims, x, Wr, bias, topk_idx, topk_w, probs=None, stream=None):
    import torch
    _check("gqe_router_topk", lib.gqe_router_topk(
        ctypes.byref(dims), _ptr(x, "x", _bf16()), _ptr(Wr, "Wr", _bf16()),
        _ptr(bias, "bias", torch.float32, optional=True), _ptr(topk_idx, "topk_idx", torch.int32),
        _ptr(topk_w, "topk_w", torch.float32), _ptr(probs, "probs", torch.float32, optional=True),
        _stream(stream)))


def gqe_router_stats(dims, probs, topk_idx, counts, prob_sum, stream=None):
    import torch
    _check("gqe_router_stats", lib.gqe_router_stats(
        ctypes.byref(dims), _ptr(probs, "probs", torch.float32), _ptr(topk_idx, "topk_idx", torch.int32),
        _ptr(counts, "counts", torch.int32), _ptr(prob_sum, "prob_sum", torch.float32), _stream(stream)))


def gqe_routed_qproj(dims, x, Wq, Wsh, topk_idx, q_routed, q_sh, ws, expert_counts=None, stream=None):
    import torch
    ws_bytes = ws.numel() * ws.element_size()
    _check("gqe_routed_qproj", lib.gqe_routed_qproj(
        ctypes.byref(dims), _ptr(x, "x", _bf16()), _ptr(Wq, "Wq", _bf16()),
        _ptr(Wsh, "Wsh", _bf16(), optional=True), _ptr(topk_idx, "topk_idx", torch.int32),
        _ptr(q_routed, "q_routed", _bf16()), _ptr(q_sh, "q_sh", _bf16(), optional=True),
        _ptr(expert_counts, "expert_counts", torch.int32, optional=True),
        _ptr(ws, "ws"), ws_bytes, _stream(stream)))


def gqe_kv_proj(dims, x, Wk, Wv, K, V, stream=None):
    b = _bf16()
    _check("gqe_kv_proj", lib.gqe_kv_proj(
        ctypes.byref(dims), _ptr(x, "x", b), _ptr(Wk, "Wk", b), _ptr(Wv, "Wv", b),
        _ptr(K, "K", b), _ptr(V, "V", b), _stream(stream)))


def gqe_kv_append(dims, x, Wk, Wv, Kc, Vc, L_max, cache_len, stream=None):
    import torch
    b = _bf16()
    _check("gqe_kv_append", lib.gqe_kv_append(
        ctypes.byref(dims), _ptr(x, "x", b), _ptr(Wk, "Wk", b), _ptr(Wv, "Wv", b),
        _ptr(Kc, "Kc", b), _ptr(Vc, "Vc", b), int(L_max), _ptr(cache_len, "cache_len", torch.int32),
        _stream(stream)))


def gqe_attn_prefill(dims, q_routed, q_sh, K, V, o_routed, o_sh, lse=None, stream=None):
    import torch
    b = _bf16()
    _check("gqe_attn_prefill", lib.gqe_attn_prefill(
        ctypes.byref(dims), _ptr(q_routed, "q_routed", b), _ptr(q_sh, "q_sh", b, optional=True),
        _ptr(K, "K", b), _ptr(V, "V", b), _ptr(o_routed, "o_routed", b),
        _ptr(o_sh, "o_sh", b, optional=True), _ptr(lse, "lse", torch.float32, optional=True),
        _stream(stream)))


def gqe_attn_prefill_bwd(dims, q_routed, q_sh, K, V, o_routed, o_sh, lse, do_routed, do_sh,
                         dq_routed, dq_sh, dK, dV, ws, stream=None):
    import torch
    b = _bf16()
    ws_bytes = ws.numel() * ws.element_size()
    _check("gqe_attn_prefill_bwd", lib.gqe_attn_prefill_bwd(
        ctypes.byref(dims), _ptr(q_routed, "q_routed", b), _ptr(q_sh, "q_sh", b, optional=True),
        _ptr(K, "K", b), _ptr(V, "V", b), _ptr(o_routed, "o_routed", b), _ptr(o_sh, "o_sh", b, optional=True),
        _ptr(lse, "lse", torch.float32), _ptr(do_routed, "do_routed", b), _ptr(do_sh, "do_sh", b, optional=True),
        _ptr(dq_routed, "dq_routed", b), _ptr(dq_sh, "dq_sh", b, optional=True), _ptr(dK, "dK", b),
        _ptr(dV, "dV", b), _ptr(ws, "ws"), ws_bytes, _stream(stream)))


def gqe_attn_decode(dims, q_routed, q_sh, Kc, Vc, L_max, cache_len, o_routed, o_sh, ws, stream=None):
    import torch
    b = _bf16()
    ws_bytes = ws.numel() * ws.element_size()
    _check("gqe_attn_decode", lib.gqe_attn_decode(
        ctypes.byref(dims), _ptr(q_routed, "q_routed", b), _ptr(q_sh, "q_sh", b, optional=True),
        _ptr(Kc, "Kc", b), _ptr(Vc, "Vc", b), int(L_max), _ptr(cache_len, "cache_len", torch.int32),
        _ptr(o_routed, "o_routed", b), _ptr(o_sh, "o_sh", b, optional=True), _ptr(ws, "ws"), ws_bytes,
        _stream(stream)))


def gqe_attn_decode_noalloc(dims, q_routed, q_sh, Kc, Vc, L_max, cache_len, o_routed, o_sh, stream=None):
    """gqe_attn_decode with the partial states in the library's fixed device
    array instead of a caller workspace: for callers that cannot allocate
    device memory at decode time.  Calls must not overlap on the GPU."""
    import torch
    b = _bf16()
    _check("gqe_attn_decode_noalloc", lib.gqe_attn_decode_noalloc(
        ctypes.byref(dims), _ptr(q_routed, "q_routed", b), _ptr(q_sh, "q_sh", b, optional=True),
        _ptr(Kc, "Kc", b), _ptr(Vc, "Vc", b), int(L_max), _ptr(cache_len, "cache_len", torch.int32),
        _ptr(o_routed, "o_routed", b), _ptr(o_sh, "o_sh", b, optional=True), _stream(stream)))


DECODE_NOALLOC_MAX_BYTES = 8 << 20


def gqe_combine(dims, o_routed, o_sh, topk_w, h, stream=None):
    import torch
    b = _bf16()
    _check("gqe_combine", lib.gqe_combine(
        ctypes.byref(dims), _ptr(o_routed, "o_routed", b), _ptr(o_sh, "o_sh", b, optional=True),
        _ptr(topk_w, "topk_w", torch.float32), _ptr(h, "h", b), _stream(stream)))


def gqe_combine_out_proj(dims, o_routed, o_sh, topk_w, Wo, y, ws, stream=None):
    import torch
    b = _bf16()
    ws_bytes = ws.numel() * ws.element_size()
    _check("gqe_combine_out_proj", lib.gqe_combine_out_proj(
        ctypes.byref(dims), _ptr(o_routed, "o_routed", b), _ptr(o_sh, "o_sh", b, optional=True),
        _ptr(topk_w, "topk_w", torch.float32), _ptr(Wo, "Wo", b), _ptr(y, "y", b),
        _ptr(ws, "ws"), ws_bytes, _stream(stream)))


def layer_weights(src) -> gqe_layer_weights:
    """The weight struct of gqe_layer_forward[_host] from an object (e.g. a
    GQELayer) or dict holding the device tensors Wr, bias, Wq, Wsh, Wk, Wv, Wo
    (bias and Wsh may be None).  The struct holds raw pointers: keep the
    tensors alive while it is in use."""
    import torch
    get = src.get if isinstance(src, dict) else (lambda k: getattr(src, k, None))
    b = _bf16()
    return gqe_layer_weights(
        Wr=_ptr(get("Wr"), "Wr", b), bias=_ptr(get("bias"), "bias", torch.float32, optional=True),
        Wq=_ptr(get("Wq"), "Wq", b), Wsh=_ptr(get("Wsh"), "Wsh", b, optional=True),
        Wk=_ptr(get("Wk"), "Wk", b), Wv=_ptr(get("Wv"), "Wv", b), Wo=_ptr(get("Wo"), "Wo", b))


def _host_ptr(t, name):
    if t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.dtype != _bf16():
        raise ValueError(f"{name} must be {_bf16()}, got {t.dtype}")
    return t.data_ptr()


def gqe_layer_forward(dims, weights, x, y, ws, stream=None):
    """Whole prefill forward, device x [B, T, D] -> y; weights from layer_weights()."""
    b = _bf16()
    ws_bytes = ws.numel() * ws.element_size()
    _check("gqe_layer_forward", lib.gqe_layer_forward(
        ctypes.byref(dims), ctypes.byref(weights), _ptr(x, "x", b), _ptr(y, "y", b), _ptr(ws, "ws"), ws_bytes,
        _stream(stream)))


def gqe_layer_forward_host(dims, weights, x_host, y_host, chunk_seqs, ws, stream_in=None, stream_compute=None,
                           stream_out=None):
    """Whole prefill forward on host x_host [B, T, D] -> y_host (pinned for
    overlap), chunk_seqs sequences per chunk; streams default to the current
    one.  y_host is written once stream_compute reaches this point."""
    ws_bytes = ws.numel() * ws.element_size()
    _check("gqe_layer_forward_host", lib.gqe_layer_forward_host(
        ctypes.byref(dims), ctypes.byref(weights), _host_ptr(x_host, "x_host"), _host_ptr(y_host, "y_host"),
        int(chunk_seqs), _ptr(ws, "ws"), ws_bytes, _stream(stream_in), _stream(stream_compute),
        _stream(stream_out)))


def gqe_linear(A, W, C, stream=None):
    b = _bf16()
    M, K = A.shape[-2] if A.dim() > 1 else 1, A.shape[-1]
    M = A.numel() // K
    N = W.shape[0]
    _check("gqe_linear", lib.gqe_linear(M, N, K, _ptr(A, "A", b), _ptr(W, "W", b), _ptr(C, "C", b),
                                        _stream(stream)))


def gqe_gemm(A, a_kn, B, b_kn, C, stream=None):
    """C [M, N] = A B^T over K, with A stored [M, K] (a_kn=0) or [K, M] (a_kn=1)
    and B stored [N, K] (b_kn=0) or [K, N] (b_kn=1)."""
    b = _bf16()
    A2 = A.reshape(-1, A.shape[-1])
    B2 = B.reshape(-1, B.shape[-1])
    M, K = (A2.shape[1], A2.shape[0]) if a_kn else (A2.shape[0], A2.shape[1])
    N, Kb = (B2.shape[1], B2.shape[0]) if b_kn else (B2.shape[0], B2.shape[1])
    if K != Kb:
        raise ValueError(f"K mismatch: {K} vs {Kb}")
    if C.numel() != M * N:
        raise ValueError(f"C has {C.numel()} elements, expected {M}x{N}")
    _check("gqe_gemm", lib.gqe_gemm(M, N, K, _ptr(A, "A", b), int(a_kn), _ptr(B, "B", b), int(b_kn),
                                    _ptr(C, "C", b), _stream(stream)))


def gqe_gemm_acc(A, a_kn, B, b_kn, C, accumulate=False, stream=None):
    """C [M, N] fp32 = (C if accumulate else 0) + A B^T over K (layouts as gqe_gemm)."""
    import torch
    b = _bf16()
    A2 = A.reshape(-1, A.shape[-1])
    B2 = B.reshape(-1, B.shape[-1])
    M, K = (A2.shape[1], A2.shape[0]) if a_kn else (A2.shape[0], A2.shape[1])
    N, Kb = (B2.shape[1], B2.shape[0]) if b_kn else (B2.shape[0], B2.shape[1])
    if K != Kb:
        raise ValueError(f"K mismatch: {K} vs {Kb}")
    if C.numel() != M * N:
        raise ValueError(f"C has {C.numel()} elements, expected {M}x{N}")
    _check("gqe_gemm_acc", lib.gqe_gemm_acc(M, N, K, _ptr(A, "A", b), int(a_kn), _ptr(B, "B", b), int(b_kn),
                                            _ptr(C, "C", torch.float32), int(bool(accumulate)), _stream(stream)))


def gqe_combine_bwd(dims, o_routed, o_sh, topk_w, dh, do_routed, do_sh, dtopk_w, stream=None):
    import torch
    b = _bf16()
    _check("gqe_combine_bwd", lib.gqe_combine_bwd(
        ctypes.byref(dims), _ptr(o_routed, "o_routed", b), _ptr(o_sh, "o_sh", b, optional=True),
        _ptr(topk_w, "topk_w", torch.float32), _ptr(dh, "dh", b), _ptr(do_routed, "do_routed", b),
        _ptr(do_sh, "do_sh", b, optional=True), _ptr(dtopk_w, "dtopk_w", torch.float32), _stream(stream)))


def gqe_router_bwd(dims, probs, topk_idx, topk_w, dtopk_w, dlogits, dbias=None, stream=None):
    import torch
    f = torch.float32
    _check("gqe_router_bwd", lib.gqe_router_bwd(
        ctypes.byref(dims), _ptr(probs, "probs", f), _ptr(topk_idx, "topk_idx", torch.int32),
        _ptr(topk_w, "topk_w", f), _ptr(dtopk_w, "dtopk_w", f), _ptr(dlogits, "dlogits", f),
        _ptr(dbias, "dbias", f, optional=True), _stream(stream)))


def gqe_bwd_pack_cols(dims) -> int:
    n = _I(0)
    _check("gqe_bwd_pack_cols", lib.gqe_bwd_pack_cols(ctypes.byref(dims), ctypes.byref(n)))
    return int(n.value)


def gqe_bwd_pack(dims, topk_idx, dq_routed, dq_sh, dK, dV, dlogits, A, stream=None):
    import torch
    b = _bf16()
    _check("gqe_bwd_pack", lib.gqe_bwd_pack(
        ctypes.byref(dims), _ptr(topk_idx, "topk_idx", torch.int32), _ptr(dq_routed, "dq_routed", b),
        _ptr(dq_sh, "dq_sh", b, optional=True), _ptr(dK, "dK", b), _ptr(dV, "dV", b),
        _ptr(dlogits, "dlogits", torch.float32), _ptr(A, "A", b), _stream(stream)))


def gqe_bwd_pack_weights(dims, Wr, Wq, Wsh, Wk, Wv, Wcat, stream=None):
    b = _bf16()
    _check("gqe_bwd_pack_weights", lib.gqe_bwd_pack_weights(
        ctypes.byref(dims), _ptr(Wr, "Wr", b), _ptr(Wq, "Wq", b), _ptr(Wsh, "Wsh", b, optional=True),
        _ptr(Wk, "Wk", b), _ptr(Wv, "Wv", b), _ptr(Wcat, "Wcat", b), _stream(stream)))


def gqe_transpose(src, dst, ld_dst=None, stream=None):
    """dst [cols, ld_dst] <- src [rows, cols]^T (columns past rows zeroed)."""
    b = _bf16()
    rows, cols = src.shape[0], src.numel() // src.shape[0]
    ld = rows if ld_dst is None else int(ld_dst)
    _check("gqe_transpose", lib.gqe_transpose(rows, cols, _ptr(src, "src", b), _ptr(dst, "dst", b), ld,
                                              _stream(stream)))


def gqe_transpose_f32(src, dst, ld_dst=None, stream=None):
    """dst [cols, ld_dst] <- src [rows, cols]^T, fp32."""
    import torch
    rows, cols = src.shape[0], src.numel() // src.shape[0]
    ld = rows if ld_dst is None else int(ld_dst)
    _check("gqe_transpose_f32", lib.gqe_transpose_f32(rows, cols, _ptr(src, "src", torch.float32),
                                                      _ptr(dst, "dst", torch.float32), ld, _stream(stream)))


def gqe_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    _check("gqe_device_error", lib.gqe_device_error(ctypes.byref(code), _stream(stream)))
    return int(code.value)


def gqe_debug_wait_timeout(stream=None):
    _check("gqe_debug_wait_timeout", lib.gqe_debug_wait_timeout(_stream(stream)))


def gqe_debug_exp2(x, y_poly, y_pair, y_hw, stream=None):
    import torch
    f = torch.float32
    _check("gqe_debug_exp2", lib.gqe_debug_exp2(_ptr(x, "x", f), _ptr(y_poly, "y_poly", f), _ptr(y_pair, "y_pair", f),
                                                _ptr(y_hw, "y_hw", f), x.numel(), _stream(stream)))


def gqe_status_string(status: int) -> str:
    return lib.gqe_status_string(int(status)).decode()
