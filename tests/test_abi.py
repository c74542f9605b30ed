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


def test_library_is_built_for_sm100a():
    with open(gq.LIB_PATH, "rb") as f:
        blob = f.read()
    assert b"sm_100a" in blob


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
