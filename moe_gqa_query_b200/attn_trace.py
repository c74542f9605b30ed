"""Where the d = 64 prefill attention kernel spends its time, CTA by CTA.

Runs gqe_attn_prefill of one workload through the traced diagnostic build of
the library (libgqe_trace.so, include/gqe_trace.h) and prints, as JSON, the
per-CTA phases (set-up, first S tile, softmax loop, last P V, output stores),
the softmax loop time per key tile by CTA size, the share of SM time with 0, 1
or 2 resident CTAs, and when the last CTAs start and end.

  python moe_gqa_query_b200/build.py --trace
  GQE_LIB_PATH=moe_gqa_query_b200/libgqe_trace.so python -m moe_gqa_query_b200.attn_trace main_prefill

Inputs are random bf16 on the device (values do not change the timeline); the
L2 is flushed before the traced launch, as in the benchmark.
"""
from __future__ import annotations

import ctypes
import json
import os
import sys

import numpy as np
import torch

from . import _lib
from ._lib import gqe_attn_prefill, gqe_device_error, make_dims

FIELDS = 12


def _stats(x):
    x = np.asarray(x, dtype=np.float64)
    return {"mean": round(float(x.mean()), 3), "p10": round(float(np.percentile(x, 10)), 3),
            "p90": round(float(np.percentile(x, 90)), 3)}


def trace(dims, reps: int = 3, seed: int = 0) -> dict:
    if not hasattr(_lib.lib, "gqe_debug_attn_trace"):
        raise RuntimeError(f"{_lib.LIB_PATH} is not the traced build: set GQE_LIB_PATH to libgqe_trace.so")
    if dims.d != 64:
        raise ValueError("the trace covers the d_head = 64 kernel")
    read = _lib.lib.gqe_debug_attn_trace
    read.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    read.restype = ctypes.c_int
    B, G, T, k, d = dims.B, dims.G, dims.T, dims.k, dims.d
    gen = torch.Generator(device="cuda").manual_seed(seed)
    q = torch.randn((B, G, T, k, d), device="cuda", generator=gen).to(torch.bfloat16)
    qs = torch.randn((B, T, d), device="cuda", generator=gen).to(torch.bfloat16)
    K = torch.randn((B, G, T, d), device="cuda", generator=gen).to(torch.bfloat16)
    V = torch.randn((B, G, T, d), device="cuda", generator=gen).to(torch.bfloat16)
    o, os_ = torch.empty_like(q), torch.empty_like(qs)
    dc = make_dims(dims)
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    for _ in range(3):
        gqe_attn_prefill(dc, q, qs, K, V, o, os_, None)
    torch.cuda.synchronize()
    n_cta = ((T + 127) // 128) * (B * G * k + B * dims.n_shared)
    assert n_cta <= 16384
    for _ in range(reps):
        flush.zero_()
        torch.cuda._sleep(600_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        gqe_attn_prefill(dc, q, qs, K, V, o, os_, None)
        e1.record()
        torch.cuda.synchronize()
    buf = np.zeros(n_cta * FIELDS, dtype=np.uint64)
    assert read(buf.ctypes.data, buf.nbytes) == 0
    a = buf.reshape(n_cta, FIELDS).astype(np.int64)
    a = a[a[:, 1] > 0]                     # CTAs of q-tiles past the rows return at once, unrecorded
    sm = a[:, 0] & 0xFFFF
    nkv = (a[:, 0] >> 16) & 0x7FFF
    t0 = a[:, 1].min()
    us = lambda c1, c0: (a[:, c1] - a[:, c0]) / 1e3  # noqa: E731
    loop, tot = us(6, 4), us(9, 1)
    out = {"event_ms_last": e0.elapsed_time(e1), "span_us": (a[:, 9].max() - t0) / 1e3, "ctas": int(len(a)),
           "key_tiles": int(nkv.sum()), "key_tiles_per_sm": round(float(nkv.sum() / 148), 2)}
    out["per_cta_us"] = {
        "set-up (entry to dependent-launch wait done)": _stats(us(2, 1)),
        "Q arrival after set-up": _stats(us(3, 2)),
        "first S ready after set-up": _stats(us(4, 2)),
        "softmax of the first tile": _stats(us(5, 4)),
        "softmax loop, all tiles": _stats(loop),
        "waits for S after the first tile (summed)": _stats(a[:, 10] / 1e3),
        "waits for P V (summed)": _stats(a[:, 11] / 1e3),
        "last P V after the loop": _stats(us(7, 6)),
        "output stores": _stats(us(8, 7)),
        "teardown": _stats(us(9, 8)),
        "total": _stats(tot)}
    by = {}
    for n in sorted(set(nkv.tolist())):
        m = nkv == n
        by[int(n)] = {"ctas": int(m.sum()), "total_us": round(float(tot[m].mean()), 2),
                      "loop_per_tile_us": round(float((loop[m] / n).mean()), 3),
                      "outside_loop_us": round(float((tot[m] - loop[m]).mean()), 2)}
    out["by_key_tiles"] = by
    occ = np.zeros(3)
    t_end = a[:, 9].max()
    for s_ in np.unique(sm):
        m = sm == s_
        ev = sorted([(int(x), 1) for x in a[m, 1]] + [(int(x), -1) for x in a[m, 9]])
        cur, last = 0, t0
        for tt, dlt in ev:
            occ[min(cur, 2)] += tt - last
            cur += dlt
            last = tt
        occ[0] += t_end - last
    out["sm_time_share_with_0_1_2_ctas"] = [round(float(x), 3) for x in occ / occ.sum()]
    out["cta_start_us_p50_p90_max"] = [round(float(np.percentile(a[:, 1] - t0, q_)) / 1e3, 2) for q_ in (50, 90, 100)]
    out["cta_end_us_p50_p90_max"] = [round(float(np.percentile(a[:, 9] - t0, q_)) / 1e3, 2) for q_ in (50, 90, 100)]
    # slot-time budget: 2 CTA slots per SM over the span
    slot = 2 * 148 * out["span_us"]
    steady = float(np.median(loop[nkv == nkv.max()] / nkv.max()))
    out["slot_time_budget_share"] = {
        "softmax loops at the longest CTAs' per-tile rate": round(float(nkv.sum() * steady / slot), 3),
        "softmax loops above that rate": round(float((loop.sum() - nkv.sum() * steady) / slot), 3),
        "outside the loop (set-up, first S, last P V, stores)": round(float((tot - loop).sum() / slot), 3),
        "no CTA resident": round(float(1 - tot.sum() / slot), 3)}
    out["device_error"] = gqe_device_error()
    return out


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import gqe_inputs as gi
    wname = argv[0] if argv else "main_prefill"
    res = trace(gi.WORKLOADS[wname].dims)
    res = {"workload": wname, "library": os.path.basename(_lib.LIB_PATH), **res}
    print(json.dumps(res, indent=1))
    return 0


if __name__ == "__main__":
    sys.exit(main())
