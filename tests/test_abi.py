"""The C-ABI library builds for sm_100a, loads, exports every declared symbol and
rejects bad arguments before launching anything (CPU only: no compute call)."""
import ctypes
import os

import numpy as np
import pytest

import moe_gqa_query_b200 as gq
from moe_gqa_query_b200 import _lib


def test_library_exports_every_header_function():
    names = gq.header_functions()
    assert len(names) >= 11
    raw = ctypes.CDLL(gq.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    # the five calls of the method's hot path
    for n in ("gqe_router_topk", "gqe_routed_qproj", "gqe_attn_prefill", "gqe_attn_decode", "gqe_combine"):
        assert n in names


def _header_prototypes():
    """name -> list of parameter declarations, from include/gqe.h."""
    import re
    with open(_lib.HEADER_PATH) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    out = {}
    for m in re.finditer(r"^\s*(?:const\s+)?\w+\*?\s+\*?(gqe_\w+)\s*\(([^)]*)\)\s*;", text, flags=re.M):
        params = [p.strip() for p in m.group(2).replace("\n", " ").split(",") if p.strip()]
        out[m.group(1)] = [] if params == ["void"] else params
    return out


def test_bindings_match_header_prototypes():
    """Every declared function has a ctypes signature with the same number of
    parameters, and each parameter's kind agrees: pointers (and the stream
    handle) as pointers, size_t as size_t, int (and the status enum) as int."""
    protos = _header_prototypes()
    assert set(protos) == set(gq.header_functions())
    for name, params in protos.items():
        sig = _lib.SIGNATURES.get(name)
        assert sig is not None, f"{name} has no binding"
        assert len(sig) == len(params), f"{name}: header {len(params)} parameters, binding {len(sig)}"
        for decl, t in zip(params, sig):
            if "*" in decl or decl.startswith("gqe_stream"):
                assert t is ctypes.c_void_p or issubclass(t, ctypes._Pointer), f"{name}: {decl}"
            elif decl.startswith("size_t"):
                assert t is ctypes.c_size_t, f"{name}: {decl}"
            elif decl.startswith("int") or decl.startswith("gqe_status"):   # the status enum is an int
                assert t is ctypes.c_int, f"{name}: {decl}"
            else:
                raise AssertionError(f"{name}: unexpected parameter {decl}")


def test_library_build_targets_sm100a_only():
    """The build compiles every source for sm_100a and for nothing else (read
    from the build script's flags, not from the built binary)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("gqe_build", os.path.join(os.path.dirname(gq.LIB_PATH), "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    flags = mod.NVCC_FLAGS
    archs = [flags[i + 1] for i, f in enumerate(flags) if f == "-gencode"]
    assert archs == ["arch=compute_100a,code=sm_100a"]
    assert not any(f.startswith("-arch") for f in flags)


def test_noalloc_limit_matches_header():
    """The binding's size limit of gqe_attn_decode_noalloc is the header's."""
    import re
    with open(_lib.HEADER_PATH) as f:
        m = re.search(r"#define\s+GQE_DECODE_NOALLOC_MAX_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", f.read())
    assert m, "GQE_DECODE_NOALLOC_MAX_BYTES not found in the header"
    assert gq.DECODE_NOALLOC_MAX_BYTES == int(m.group(1)) << int(m.group(2))


def _cfg(**kw):
    base = dict(B=1, T=128, D=256, G=2, E=2, k=1, d=64)
    base.update(kw)
    return type("C", (), base)()


@pytest.mark.parametrize("bad,status", [
    (dict(k=3, E=2), 1),            # k > E
    (dict(k=0), 1),
    (dict(B=0), 1),
    (dict(d=96), 2),                # unsupported head width
    (dict(E=9, k=1), 2),            # E > 8
    (dict(D=100), 2),               # d_model not a multiple of 64
    (dict(G=9, E=8, k=1), 2),       # G*E > 64
])
def test_bad_dims_are_rejected(bad, status):
    d = gq.make_dims(_cfg(**bad))
    with pytest.raises(gq.GQEError) as ei:
        gq.gqe_workspace_size(d, gq.GQE_OP_ROUTED_QPROJ)
    assert ei.value.status == status


def test_bad_shared_group_and_scope():
    with pytest.raises(gq.GQEError):
        gq.gqe_workspace_size(gq.make_dims(_cfg(), shared_kv_group=2), 1)
    with pytest.raises(gq.GQEError):
        gq.gqe_workspace_size(gq.make_dims(_cfg(), renorm_scope=3), 1)
    with pytest.raises(gq.GQEError):
        gq.gqe_workspace_size(gq.make_dims(_cfg(), output_mode=3), 1)
    with pytest.raises(gq.GQEError):
        gq.gqe_workspace_size(gq.make_dims(_cfg(), output_mode=-1), 1)
    with pytest.raises(gq.GQEError):
        gq.gqe_workspace_size(gq.make_dims(_cfg(), scale=-1.0), 1)


def test_output_mode_changes_the_fused_projection_scratch():
    base = _cfg(B=2, T=256, D=256, G=4, E=2, k=1)
    sizes = [gq.gqe_workspace_size(gq.make_dims(base, output_mode=m), gq.GQE_OP_COMBINE_OUT_PROJ) for m in range(3)]
    # h has k*G + 1 + n_shared slots in mode 0 and one fewer in the ablation modes
    assert sizes[0] == 512 * (4 + 1 + 1) * 64 * 2
    assert sizes[1] == sizes[2] == 512 * (4 + 1) * 64 * 2


def test_workspace_sizes():
    d = gq.make_dims(_cfg(B=8, T=2048, D=1024, G=8, E=2, k=1))
    n = gq.gqe_workspace_size(d, gq.GQE_OP_ROUTED_QPROJ)
    # at least the two permutation index arrays (source and destination row)
    assert n >= 2 * 4 * 8 * 2048 * 8
    dd = gq.make_dims(_cfg(B=64, T=1, D=1024, G=8, E=2, k=1))
    m = gq.gqe_workspace_size(dd, gq.GQE_OP_ATTN_DECODE, 32768)
    assert m >= 64 * 8 * 2 * 66 * 4
    with pytest.raises(gq.GQEError):
        gq.gqe_workspace_size(dd, gq.GQE_OP_ATTN_DECODE, 0)
    with pytest.raises(gq.GQEError):
        gq.gqe_workspace_size(d, 99)


def test_null_pointers_rejected_before_launch():
    d = gq.make_dims(_cfg())
    lib = _lib.lib
    st = lib.gqe_router_topk(ctypes.byref(d), None, None, None, None, None, None, None)
    assert st == 1
    st = lib.gqe_attn_prefill(ctypes.byref(d), None, None, None, None, None, None, None, None)
    assert st == 1
    st = lib.gqe_combine(ctypes.byref(d), None, None, None, None, None)
    assert st == 1
    st = lib.gqe_linear(0, 64, 64, None, None, None, None)
    assert st == 1
    st = lib.gqe_linear(4, 64, 60, 16, 16, 16, None)     # K not a multiple of 64
    assert st == 2


def test_misaligned_pointers_rejected_before_launch():
    d = gq.make_dims(_cfg())
    lib = _lib.lib
    st = lib.gqe_kv_proj(ctypes.byref(d), 18, 32, 48, 64, 80, None)   # x not 16-byte aligned
    assert st == 1
    # decode needs T == 1
    st = lib.gqe_attn_decode(ctypes.byref(d), 16, 16, 16, 16, 100, 16, 16, 16, 16, 1 << 20, None)
    assert st == 1


def test_workspace_too_small_rejected():
    d = gq.make_dims(_cfg())
    lib = _lib.lib
    st = lib.gqe_routed_qproj(ctypes.byref(d), 16, 16, 16, 16, 16, 16, None, 16, 8, None)
    assert st == 3


def test_status_strings():
    assert gq.gqe_status_string(0) == "ok"
    assert "workspace" in gq.gqe_status_string(3)


def test_package_fails_loudly_without_library(tmp_path, monkeypatch):
    """The binding refuses to import when libgqe.so is absent (no CPU fallback)."""
    import importlib.util
    import sys
    src = os.path.join(os.path.dirname(gq.__file__), "_lib.py")
    spec = importlib.util.spec_from_file_location("gqe_lib_probe", src)
    mod = importlib.util.module_from_spec(spec)
    monkeypatch.setattr(os.path, "exists", lambda p: False if p.endswith("libgqe.so") else os.path.isfile(p))
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)
    sys.modules.pop("gqe_lib_probe", None)


# ---------------------------------------------------------------------------
# backward calls: sizes and argument checks (host side only)

def test_attention_backward_workspace_size():
    """LSE2 and Delta per padded query row (routed rows of each (b, g) padded to
    128, then the shared head's), 256-byte aligned, then the fp32 dQ accumulator."""
    for cfg in (_cfg(B=8, T=2048, D=1024, G=8, E=2, k=1), _cfg(B=2, T=300, D=256, G=3, E=4, k=3, d=128),
                _cfg(B=1, T=70, D=128, G=2, E=2, k=2)):
        for n_shared in (0, 1):
            d = gq.make_dims(cfg, n_shared=n_shared)
            rows_pad = -(-cfg.T * cfg.k // 128) * 128
            rows_pad_sh = -(-cfg.T // 128) * 128
            n = cfg.B * cfg.G * rows_pad + n_shared * cfg.B * rows_pad_sh
            a256 = lambda b: -(-b // 256) * 256
            assert gq.gqe_workspace_size(d, gq.GQE_OP_ATTN_BWD) == 2 * a256(4 * n) + 4 * n * cfg.d


def test_backward_pack_columns():
    """Kc = G*E*d (dq per expert) + n_shared*d + 2*G*d (dK, dV) + d logits padded to 64."""
    for cfg, n_shared in ((_cfg(B=8, T=2048, D=1024, G=8, E=2, k=1), 1), (_cfg(G=4, E=8, k=4, d=128), 1),
                          (_cfg(G=3, E=3, k=2), 0), (_cfg(G=8, E=8, k=1), 1)):
        d = gq.make_dims(cfg, n_shared=n_shared)
        GE = cfg.G * cfg.E
        want = GE * cfg.d + n_shared * cfg.d + 2 * cfg.G * cfg.d + 64 * (-(-GE // 64))
        assert gq.gqe_bwd_pack_cols(d) == want
    assert gq.gqe_bwd_pack_cols(gq.make_dims(_cfg(B=8, T=2048, D=1024, G=8, E=2, k=1))) == 2176


def test_backward_calls_reject_bad_arguments_before_launch():
    d = gq.make_dims(_cfg())
    lib = _lib.lib
    assert lib.gqe_attn_prefill_bwd(ctypes.byref(d), *([None] * 14), 0, None) == 1
    assert lib.gqe_combine_bwd(ctypes.byref(d), None, None, None, None, None, None, None, None) == 1
    assert lib.gqe_router_bwd(ctypes.byref(d), None, None, None, None, None, None, None) == 1
    assert lib.gqe_bwd_pack(ctypes.byref(d), None, None, None, None, None, None, None, None) == 1
    assert lib.gqe_bwd_pack_weights(ctypes.byref(d), None, None, None, None, None, None, None) == 1
    # a short attention-backward workspace
    assert lib.gqe_attn_prefill_bwd(ctypes.byref(d), *([256] * 13), 256, 16, None) == 3
    # transposes: empty or a destination narrower than the source's rows
    assert lib.gqe_transpose(0, 64, 16, 16, 64, None) == 1
    assert lib.gqe_transpose(100, 64, 16, 16, 64, None) == 1
    assert lib.gqe_transpose_f32(100, 64, 16, 16, 64, None) == 1


@pytest.mark.parametrize("fn", ["gqe_gemm", "gqe_gemm_acc"])
def test_gemm_argument_checks(fn):
    lib = _lib.lib
    call = (lambda M, N, K, A, ak, B, bk, C: lib.gqe_gemm(M, N, K, A, ak, B, bk, C, None)) if fn == "gqe_gemm" \
        else (lambda M, N, K, A, ak, B, bk, C: lib.gqe_gemm_acc(M, N, K, A, ak, B, bk, C, 0, None))
    assert call(0, 64, 64, 16, 0, 16, 0, 16) == 1          # empty
    assert call(64, 64, 64, None, 0, 16, 0, 16) == 1       # null operand
    assert call(64, 64, 64, 16, 2, 16, 0, 16) == 1         # layout flag not 0/1
    assert call(64, 96, 64, 16, 0, 16, 0, 16) == 2         # N not a multiple of 64
    assert call(64, 64, 70, 16, 0, 16, 0, 16) == 2         # contiguous K not a multiple of 8
    assert call(60, 64, 70, 16, 1, 16, 1, 16) == 2         # contiguous M not a multiple of 8
    assert call(64, 64, 64, 18, 0, 16, 0, 16) == 1         # misaligned A


def _fake_weights(**override):
    """Weight struct of made-up, 256-byte aligned addresses: only for calls
    that must return an argument error before touching them."""
    v = dict(Wr=0x10000, bias=None, Wq=0x20000, Wsh=0x30000, Wk=0x40000, Wv=0x50000, Wo=0x60000)
    v.update(override)
    return gq.gqe_layer_weights(**v)


def test_layer_forward_workspace_sizes():
    """The one-call forward's scratch holds every intermediate of the chained
    calls, and its host form adds two x and two y chunk buffers."""
    def up(n):
        return (n + 255) // 256 * 256
    for kw in (dict(B=8, T=2048, D=1024, G=8, E=2, k=1), dict(B=2, T=8192, D=4096, G=4, E=8, k=4, d=128),
               dict(B=1, T=128, D=256, G=2, E=2, k=1)):
        cfg = _cfg(**kw)
        d = gq.make_dims(cfg)
        N, G, k, dh, D = cfg.B * cfg.T, cfg.G, cfg.k, cfg.d, cfg.D
        parts = [N * G * k * 4, N * G * k * 4, N * G * k * dh * 2, N * dh * 2, N * G * dh * 2, N * G * dh * 2,
                 N * G * k * dh * 2, N * dh * 2, gq.gqe_workspace_size(d, gq.GQE_OP_ROUTED_QPROJ),
                 gq.gqe_workspace_size(d, gq.GQE_OP_COMBINE_OUT_PROJ)]
        whole = gq.gqe_workspace_size(d, gq.GQE_OP_LAYER_FORWARD)
        assert whole == sum(up(p) for p in parts)
        assert gq.gqe_workspace_size(d, gq.GQE_OP_LAYER_FORWARD_HOST) == whole + 4 * up(N * D * 2)


def test_layer_forward_bad_arguments_rejected_before_launch():
    lib = _lib.lib
    d = gq.make_dims(_cfg(B=4, T=128))
    w = _fake_weights()
    xh = (ctypes.c_uint16 * 16)()
    ws_ok = 1 << 30
    host = lambda **kw: lib.gqe_layer_forward_host(   # noqa: E731
        ctypes.byref(kw.get("d", d)), kw.get("w", ctypes.byref(w)), kw.get("x", ctypes.addressof(xh)),
        kw.get("y", ctypes.addressof(xh)), kw.get("chunk", 1), kw.get("ws", 0x1000000), kw.get("ws_bytes", ws_ok),
        None, None, None)
    assert host(chunk=0) == 1
    assert host(chunk=-2) == 1
    assert host(x=None) == 1
    assert host(w=None) == 1
    assert host(w=ctypes.byref(_fake_weights(Wq=None))) == 1
    assert host(w=ctypes.byref(_fake_weights(Wsh=None))) == 1      # the shared head needs Wsh
    assert host(w=ctypes.byref(_fake_weights(Wo=0x60008))) == 1    # misaligned
    assert host(ws=None) == 3
    assert host(ws_bytes=16) == 3
    assert host(d=gq.make_dims(_cfg(B=4, T=128, d=96))) == 2
    dev = lib.gqe_layer_forward
    assert dev(ctypes.byref(d), ctypes.byref(w), None, 0x1000000, 0x2000000, ws_ok, None) == 1
    assert dev(ctypes.byref(d), ctypes.byref(w), 0x1000008, 0x1000000, 0x2000000, ws_ok, None) == 1
    assert dev(ctypes.byref(d), ctypes.byref(w), 0x1000000, 0x1000000, 0x2000000, 100, None) == 3
