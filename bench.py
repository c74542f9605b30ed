"""Benchmark of the GQE attention layer on B200.

A step is one prefill forward of the paper's main GQE layer (16 query experts /
8 KV heads, top-1 of 2 per group, one shared head, d_model 1024, d_head 64) over
one batch of 8 x 2048 synthetic tokens: router -> routed/shared query
projection -> K/V projection -> routed causal attention -> output construction
-> output projection, all in libgqe.so kernels.

Prints one JSON line: whole-job tokens/s (max over ranks of the summed
per-step CUDA-event time), the attention kernel's roofline against the
measured bf16 tensor peak, the end-to-end number through host buffers, the
fp64 oracle's CPU throughput on a bounded sample, a decode sub-measurement
(64 sequences x 32768-entry cache, % of HBM bandwidth), and the SM clocks
sampled during the timed region.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

For N > 1 it runs under torchrun, one independent replica per GPU (the layer's
path has no exchange step), and reports the aggregate.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gqe_inputs as gi  # noqa: E402

WORKLOAD = "main_prefill"
DECODE_WORKLOAD = "decode"
METRIC = "GQE prefill tokens/s per layer"
FALLBACK_PEAKS = dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0)
L2_FLUSH_BYTES = 256 << 20
E2E_CHUNK_SEQS = 2              # sequences per copy/compute chunk of the end-to-end leg
HOST_LEAD_CYCLES = 600_000      # ~0.3 ms at B200 clocks: longer than the host needs to enqueue a step


def profiled_traffic(kernel_label, workload=WORKLOAD):
    """DRAM bytes per launch of a kernel on a workload from the committed ncu
    summaries (profiles/traffic.json), or None when there is no capture for
    that kernel and workload or the kernel's source changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            caps = json.load(f)["captures"]
        entry = next((c for c in caps if c["kernel"] == kernel_label and c["workload"] == workload), None)
        if not entry:
            return None
        with open(os.path.join(ROOT, entry["source"]), "rb") as f:
            digest = hashlib.sha256(f.read()).hexdigest()[:16]
        if digest != entry["source_sha256_16"]:
            return None
        return int(entry["dram_read_bytes"]) + int(entry["dram_write_bytes"])
    except (OSError, ValueError, KeyError):
        return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16_tflops=float(p["bf16_tflops"]),
                    bf16_tflops_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(FALLBACK_PEAKS, source="fallback")


def attn_useful_flops(dims) -> float:
    """Causal useful FLOPs of the routed + shared attention: QK^T and PV over the
    kG+1 active query heads, keys 0..t only: 2 * 2 * d * T(T+1)/2 per head."""
    return 2.0 * dims.d * dims.T * (dims.T + 1) * dims.B * dims.h_active


def decode_attn_bytes(dims, L) -> float:
    """Algorithmic bytes of the decode attention: the K and V cache read once
    (bf16), plus the query rows and outputs."""
    cache = 2.0 * dims.B * dims.G * L * dims.d * 2
    q_o = 2.0 * dims.B * (dims.G * dims.k + dims.n_shared) * dims.d * 2
    return cache + q_o


# ----------------------------------------------------------------------------
# distributed plumbing (replicas; the only cross-rank steps are the barrier and
# the max over ranks of the measured time)

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world <= 1:
        return None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, dist, device=None) -> float:
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------
# clocks sampled during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.path or not os.path.exists(self.path):
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                p = [s.strip() for s in line.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    mx = float(p[2])
                except ValueError:
                    continue
                for n, v in zip(names, p[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample

def oracle_threads():
    """Threads the oracle's BLAS actually uses (os.cpu_count() when unknown)."""
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 0) for i in threadpool_info()] + [1])
    except Exception:
        return os.cpu_count()


def cpu_baseline(wname=WORKLOAD, seconds_budget=20.0):
    """The fp64 oracle's throughput on a bounded sample of a workload.

    Sequences of up to 8192 tokens: whole sequences of the workload through
    oracle.gqe_forward (up to 3, or until the budget is spent).  Longer
    sequences: oracle.gqe_forward over the sequence's first T/4 and first T/2
    tokens; the oracle's time for the whole sequence is extrapolated from
    those two runs as a T + b T^2 (projections linear in T, causal attention
    quadratic).
    """
    import oracle as orc
    cores = oracle_threads()
    w = gi.WORKLOADS[wname]
    dims = w.dims.replace(B=1)
    x = gi.layer_input(w.dims, rows=[0])
    Wt = gi.layer_weights(w.dims)
    bias = gi.router_bias(w)
    if dims.T <= 8192:
        n, t0 = 0, time.perf_counter()
        while True:
            orc.gqe_forward(x, Wt, dims, bias)
            n += 1
            if time.perf_counter() - t0 > seconds_budget or n >= 3:
                break
        dt = time.perf_counter() - t0
        return {"value": n * dims.N / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                "sample": f"{n} x one sequence (T={dims.T}) of the {wname} workload, fp64 numpy, {dt:.1f} s"}
    T1 = dims.T // 4
    times = []
    for Tp in (T1, 2 * T1):
        t0 = time.perf_counter()
        orc.gqe_forward(x[:, :Tp], Wt, dims.replace(T=Tp), bias)
        times.append(time.perf_counter() - t0)
    b = max((times[1] - 2 * times[0]) / (2.0 * T1 * T1), 0.0)
    a = (times[0] - b * T1 * T1) / T1
    est = a * dims.T + b * dims.T ** 2
    return {"value": dims.T / est, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{wname}: the first {T1} and {2 * T1} tokens of one sequence through the whole-layer "
                      f"oracle ({times[0]:.1f} s, {times[1]:.1f} s); time for its T={dims.T} extrapolated as "
                      f"a T + b T^2 = {est:.0f} s, fp64 numpy"}


# ----------------------------------------------------------------------------

def run_reference(args):
    """Reference arm: the fp64 oracle timed on the host cores (rank 0 only)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle as orc
    w = gi.WORKLOADS[WORKLOAD]
    dims = w.dims.replace(B=1)
    x = gi.layer_input(w.dims, rows=[0])
    Wt = gi.layer_weights(dims)
    bias = gi.router_bias(w)
    for _ in range(min(args.warmup, 1)):
        orc.gqe_forward(x, Wt, dims, bias)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.gqe_forward(x, Wt, dims, bias)
    dt = time.perf_counter() - t0
    value = args.steps * dims.N / dt
    cores = oracle_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": f"{WORKLOAD} (one sequence per step: bounded CPU sample)",
                                            "B": 1, "T": dims.T},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"one {dims.T}-token sequence of {WORKLOAD} per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_kernel(args):
    """One call of the path in isolation on its workload's inputs (for profiling)."""
    import torch
    import moe_gqa_query_b200 as gq
    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    if args.kernel == "decode_step":
        # the whole decode step of the layer (router, query projection, K/V
        # append, attention, output construction and projection)
        w = gi.WORKLOADS[DECODE_WORKLOAD]
        dd, Lc = w.dims, (args.decode_L or w.L)
        gen = torch.Generator(device=device).manual_seed(7)
        Kc = torch.empty((dd.B, dd.G, Lc, dd.d), dtype=torch.bfloat16, device=device).normal_(generator=gen)
        Vc = torch.empty_like(Kc).normal_(generator=gen)
        lay = gq.GQELayer(dd, {kk: torch.from_numpy(v.view(np.int16)) for kk, v in gi.layer_weights(dd).items()},
                          device=device)
        xn = torch.randn((dd.B, dd.D), device=device, generator=gen).to(torch.bfloat16)
        cl = torch.full((dd.B,), Lc, dtype=torch.int32, device=device)
        fn = lambda: lay.decode_step(xn, Kc, Vc, cl)  # noqa: E731
        work = dict(bytes=decode_attn_bytes(dd, Lc), tokens=float(dd.B))
    elif args.kernel == "decode":
        w = gi.WORKLOADS[DECODE_WORKLOAD]
        dd, Lc = w.dims, (args.decode_L or w.L)
        gen = torch.Generator(device=device).manual_seed(7)
        Kc = torch.empty((dd.B, dd.G, Lc, dd.d), dtype=torch.bfloat16, device=device).normal_(generator=gen)
        Vc = torch.empty_like(Kc).normal_(generator=gen)
        dc = gq.make_dims(dd, T=1)
        ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_DECODE, Lc),), dtype=torch.uint8, device=device)
        q = torch.randn((dd.B, dd.G, 1, dd.k, dd.d), device=device, generator=gen).to(torch.bfloat16)
        qs = torch.randn((dd.B, 1, dd.d), device=device, generator=gen).to(torch.bfloat16)
        o, os_ = torch.empty_like(q), torch.empty_like(qs)
        cl = torch.full((dd.B,), Lc, dtype=torch.int32, device=device)
        fn = lambda: gq.gqe_attn_decode(dc, q, qs, Kc, Vc, Lc, cl, o, os_, ws)  # noqa: E731
        work = dict(bytes=decode_attn_bytes(dd, Lc))
    else:
        w = gi.WORKLOADS[args.workload]
        dims = w.dims
        dc = gq.make_dims(dims)
        gen = torch.Generator(device=device).manual_seed(7)

        def rn(*shape, std=1.0):
            return (torch.randn(shape, device=device, generator=gen) * std).to(torch.bfloat16)
        B, T, G, E, k, d, D = dims.B, dims.T, dims.G, dims.E, dims.k, dims.d, dims.D
        if args.kernel == "attn":
            q, qs, K, V = rn(B, G, T, k, d), rn(B, T, d), rn(B, G, T, d), rn(B, G, T, d)
            o, os_ = torch.empty_like(q), torch.empty_like(qs)
            fn = lambda: gq.gqe_attn_prefill(dc, q, qs, K, V, o, os_, None)  # noqa: E731
            work = dict(flops=attn_useful_flops(dims))
        elif args.kernel == "attn_bwd":
            q, qs, K, V = rn(B, G, T, k, d), rn(B, T, d), rn(B, G, T, d), rn(B, G, T, d)
            o, os_ = torch.empty_like(q), torch.empty_like(qs)
            lse = torch.empty((B * G * T * k + B * T * dims.n_shared,), dtype=torch.float32, device=device)
            gq.gqe_attn_prefill(dc, q, qs, K, V, o, os_, lse)
            dO, dOs = rn(B, G, T, k, d), rn(B, T, d)
            dq, dqs, dK, dV = torch.empty_like(q), torch.empty_like(qs), torch.empty_like(K), torch.empty_like(V)
            ws = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_BWD),), dtype=torch.uint8, device=device)
            fn = lambda: gq.gqe_attn_prefill_bwd(dc, q, qs, K, V, o, os_, lse, dO, dOs, dq, dqs, dK, dV, ws)  # noqa
            # five products per (query tile, key tile) against the forward's two
            work = dict(flops=2.5 * attn_useful_flops(dims))
        elif args.kernel in ("layer_bwd", "train_step"):
            x = rn(B, T, D)
            Wt = gi.layer_weights(dims)
            lay = gq.GQELayer(dims, {kk: torch.from_numpy(v.view(np.int16)) for kk, v in Wt.items()},
                              gi.router_bias(w), device=device)
            dy = rn(B, T, D)
            _, saved = lay.forward(x, keep=True)
            if args.kernel == "layer_bwd":
                fn = lambda: lay.backward(x, dy, saved)  # noqa: E731
            else:
                def fn():
                    _, sv = lay.forward(x, keep=True)
                    lay.backward(x, dy, sv)
            work = dict(tokens=float(dims.N))
        elif args.kernel in ("router", "qproj", "kv", "linear", "combine", "combine_out"):
            x = rn(B, T, D)
            Wt = gi.layer_weights(dims)
            lay = gq.GQELayer(dims, {kk: torch.from_numpy(v.view(np.int16)) for kk, v in Wt.items()},
                              gi.router_bias(w), device=device)
            y, inter = lay.forward(x, keep=True)
            if args.kernel == "router":
                fn = lambda: gq.gqe_router_topk(dc, x, lay.Wr, lay.bias, inter["idx"], inter["w"], None)  # noqa
                work = dict(bytes=dims.N * D * 2.0)
            elif args.kernel == "qproj":
                ws = lay._bufs["ws_q"]
                fn = lambda: gq.gqe_routed_qproj(dc, x, lay.Wq, lay.Wsh, inter["idx"], inter["q"], inter["q_sh"], ws)  # noqa
                work = dict(flops=2.0 * dims.N * dims.h_active * d * D)
            elif args.kernel == "kv":
                fn = lambda: gq.gqe_kv_proj(dc, x, lay.Wk, lay.Wv, inter["K"], inter["V"])  # noqa
                work = dict(flops=2.0 * 2 * dims.N * G * d * D)
            elif args.kernel == "combine":
                fn = lambda: gq.gqe_combine(dc, inter["o"], inter["o_sh"], inter["w"], inter["h"])  # noqa
                work = dict(bytes=2.0 * dims.N * (G * k + 1) * d + 2.0 * dims.N * dims.slots * d)
            elif args.kernel == "combine_out":
                ws_o = lay._bufs["ws_o"]
                fn = lambda: gq.gqe_combine_out_proj(dc, inter["o"], inter["o_sh"], inter["w"], lay.Wo, y, ws_o)  # noqa
                work = dict(flops=2.0 * dims.N * dims.slots * d * D)
            else:
                fn = lambda: gq.gqe_linear(inter["h"], lay.Wo, y)  # noqa
                work = dict(flops=2.0 * dims.N * dims.slots * d * D)
        else:
            raise SystemExit(f"unknown kernel {args.kernel}")
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        flush.zero_()                            # L2 flushed before every timed call, outside the events
        torch.cuda._sleep(HOST_LEAD_CYCLES)      # host runs ahead: events time device work only
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    out = {"kernel": args.kernel, "workload": DECODE_WORKLOAD if args.kernel.startswith("decode") else args.workload,
           "ms": ms, "l2": "flushed before every call", "device_error": gq.gqe_device_error()}
    if "flops" in work:
        out["TFLOP/s"] = work["flops"] / ms / 1e9
    if "bytes" in work:
        out["GB/s"] = work["bytes"] / ms / 1e6
    if "tokens" in work:
        out["tokens/s"] = work["tokens"] / ms * 1e3
    print(json.dumps(out), flush=True)
    return 0


SWEEP_T = (2048, 4096, 8192, 16384, 32768, 65536, 131072)


def run_sweep_gqa(args):
    """GQE against dense GQA on the same layer shape (B=1, D=1024, 8 KV groups,
    E=2 query heads per group, d=64), prefill T from 2K to 128K tokens.  GQE:
    top-1 of 2 per group plus the shared head (9 active query heads).  Dense
    GQA: the same kernels with k = E and no shared head (all 16 heads, the
    weighted-sum slot kept).  Attention alone and the whole layer forward, each
    timed with CUDA events on device-generated inputs (the pages' prefill
    speedup claim, re-measured on this GPU)."""
    import torch
    import moe_gqa_query_b200 as gq
    device = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    gen = torch.Generator(device=device).manual_seed(3)
    ts = [int(t) for t in args.sweep_t.split(",")] if args.sweep_t else list(SWEEP_T)

    def rn(*shape, std=1.0):
        return (torch.randn(shape, device=device, generator=gen) * std).to(torch.bfloat16)

    def time_ms(fn, reps):
        for _ in range(2):
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in evs:
            torch.cuda._sleep(HOST_LEAD_CYCLES)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in evs)

    for T in ts:
        line = {"sweep": "gqe_vs_dense_gqa", "T": T, "B": 1}
        for name, k, n_sh in (("gqe", 1, 1), ("gqa", 2, 0)):
            dims = gi.GQEDims(B=1, T=T, D=1024, G=8, E=2, k=k, d=64, n_shared=n_sh)
            dc = gq.make_dims(dims)
            q = rn(1, 8, T, k, 64)
            qs = rn(1, T, 64)
            K, V = rn(1, 8, T, 64), rn(1, 8, T, 64)
            o, os_ = torch.empty_like(q), torch.empty_like(qs)
            reps = 3 if T >= 65536 else 5
            a_ms = time_ms(lambda: gq.gqe_attn_prefill(dc, q, qs if n_sh else None, K, V, o,
                                                      os_ if n_sh else None, None), reps)
            del q, qs, K, V, o, os_
            Wt = {"Wr": rn(1024, 16, std=0.02), "Wq": rn(8, 2, 64, 1024, std=0.02),
                  "Wk": rn(512, 1024, std=0.02), "Wv": rn(512, 1024, std=0.02),
                  "Wsh": rn(64, 1024, std=0.02), "Wo": rn(1024, dims.slots * 64, std=0.02)}
            if not n_sh:
                Wt["Wsh"] = rn(0, 1024)
            lay = gq.GQELayer(dims, Wt, None, device=device)
            x = rn(1, T, 1024)
            y = torch.empty_like(x)
            l_ms = time_ms(lambda: lay.forward(x, out=y), reps)
            del lay, x, y
            torch.cuda.empty_cache()
            line[name] = {"attn_ms": a_ms, "attn_tflops": attn_useful_flops(dims) / a_ms / 1e9,
                          "layer_ms": l_ms, "active_query_heads": dims.h_active}
        line["attn_speedup"] = line["gqa"]["attn_ms"] / line["gqe"]["attn_ms"]
        line["layer_speedup"] = line["gqa"]["layer_ms"] / line["gqe"]["layer_ms"]
        line["device_error"] = gq.gqe_device_error()
        print(json.dumps(line), flush=True)
    return 0


LAUNCHES_PER_STEP = 7   # router, permutation, routed GEMM, K/V GEMM, attention, combine, Wo GEMM (+ one memset)
CONFIG_WORKLOADS = ("tiny_prefill", "main_prefill", "long_prefill", "wide_skewed_prefill")
SEG_NAMES = ("router", "routed_qproj", "kv_proj", "attn_prefill", "combine_out_proj")


def router_near_ties(wname):
    """The workload's router near-ties ((token, group) pairs whose k-th and
    (k+1)-th logits differ by less than 1e-4, where either expert is a correct
    choice), as the oracle counted them in tests/golden/near_ties.json."""
    try:
        with open(os.path.join(ROOT, "tests", "golden", "near_ties.json")) as f:
            v = json.load(f)["workloads"][wname]
        return {"pairs": v["near_ties"], "of": v["pairs"], "source": "tests/golden/near_ties.json (fp64 oracle)"}
    except (OSError, ValueError, KeyError):
        return None


def attn_kernel_label(dims) -> str:
    return "attn_prefill_single_kernel (d=64)" if dims.d == 64 else f"attn_prefill_kernel<{dims.d}>"


def measure_prefill(gq, wname, device, dist, peaks, steps, warmup, flush, rank, world, keep_layer=False):
    """Times the prefill layer forward of one workload on this GPU.

    Timed steps: GQELayer.forward (the K/V projection on a side stream), one
    event pair around each step, the L2 flushed between steps outside the
    events.  Per-call split: separate steps with an event between every call.
    Returns tokens/s (all ranks), ms per step (max over ranks), the per-call
    split and the attention kernel's roofline against the measured peak.
    """
    import torch
    w = gi.WORKLOADS[wname]
    dims = w.dims
    Wt = gi.layer_weights(dims, seed=0)
    layer = gq.GQELayer(dims, {k: torch.from_numpy(v.view(np.int16)) for k, v in Wt.items()},
                        gi.router_bias(w), device=device)
    x_host = torch.from_numpy(gi.layer_input(dims, seed=rank).view(np.int16)).view(torch.bfloat16)
    x = x_host.to(device)
    stream = torch.cuda.current_stream(device)
    c = layer.cfg
    B, T, N = dims.B, dims.T, dims.N
    d_ = gq.make_dims(c, B=B, T=T)

    def step(evs):
        idx = layer._buf("idx", (N, c.G, c.k), torch.int32)
        wt = layer._buf("w", (N, c.G, c.k), torch.float32)
        q = layer._buf("q", (B, c.G, T, c.k, c.d))
        qs = layer._buf("qs", (B, T, c.d))
        K = layer._buf("K", (B, c.G, T, c.d))
        V = layer._buf("V", (B, c.G, T, c.d))
        o = layer._buf("o", (B, c.G, T, c.k, c.d))
        os_ = layer._buf("os", (B, T, c.d))
        y = layer._buf("y", (B, T, c.D))
        ws = layer._ws("ws_q", gq.gqe_workspace_size(d_, gq.GQE_OP_ROUTED_QPROJ))
        ws_o = layer._ws("ws_o", gq.gqe_workspace_size(d_, gq.GQE_OP_COMBINE_OUT_PROJ))
        evs[0].record(stream)
        gq.gqe_router_topk(d_, x, layer.Wr, layer.bias, idx, wt, None)
        evs[1].record(stream)
        gq.gqe_routed_qproj(d_, x, layer.Wq, layer.Wsh, idx, q, qs, ws)
        evs[2].record(stream)
        gq.gqe_kv_proj(d_, x, layer.Wk, layer.Wv, K, V)
        evs[3].record(stream)
        gq.gqe_attn_prefill(d_, q, qs, K, V, o, os_, None)
        evs[4].record(stream)
        gq.gqe_combine_out_proj(d_, o, os_, wt, layer.Wo, y, ws_o)
        evs[5].record(stream)

    y_step = torch.empty((B, T, dims.D), dtype=torch.bfloat16, device=device)
    warm_evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for _ in range(warmup):
        step(warm_evs)
        layer.forward(x, out=y_step)
        flush.zero_()
    torch.cuda.synchronize()
    assert gq.gqe_device_error() == 0
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    barrier(dist, device)
    torch.cuda.synchronize()
    for s_ in range(steps):
        flush.zero_()                       # L2 flushed between timed steps (outside the events)
        # a GPU-side pause (outside the events) lets the host enqueue the whole
        # step before the GPU reaches it, so the events time device work only
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        events[s_][0].record(stream)
        layer.forward(x, out=y_step)        # the layer's own call sequence (K/V on a side stream)
        events[s_][1].record(stream)
    torch.cuda.synchronize()
    barrier(dist, device)
    local_total_ms = float(sum(a.elapsed_time(b) for a, b in events))
    n_seg = min(steps, 10)
    seg_events = [[torch.cuda.Event(enable_timing=True) for _ in range(len(SEG_NAMES) + 1)] for _ in range(n_seg)]
    for s_ in range(n_seg):
        flush.zero_()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        step(seg_events[s_])
    torch.cuda.synchronize()
    seg_ms = np.array([[seg_events[s_][i].elapsed_time(seg_events[s_][i + 1]) for i in range(len(SEG_NAMES))]
                       for s_ in range(n_seg)])
    total_ms = max_over_ranks(local_total_ms, dist, device)
    attn_ms = float(seg_ms[:, 3].mean())
    flops = attn_useful_flops(dims)
    achieved_tf = flops / (attn_ms / 1e3) / 1e12
    label = attn_kernel_label(dims)
    out = {"workload": f"{wname}: {w.desc}", "B": B, "T": T, "d_model": dims.D, "G": dims.G, "E": dims.E,
           "k": dims.k, "d_head": dims.d, "n_shared": dims.n_shared, "steps": steps,
           "tokens_per_s": world * N * steps / (total_ms / 1e3), "ms_per_step": total_ms / steps,
           "segments_ms": {n: float(seg_ms[:, i].mean()) for i, n in enumerate(SEG_NAMES)},
           "roofline": {"bound": "tensor", "kernel": label, "achieved": achieved_tf, "peak": peaks["bf16_tflops"],
                        "unit": "TFLOP/s", "frac": achieved_tf / peaks["bf16_tflops"],
                        "peak_source": f"{peaks['source']} bf16 dense (burst)", "traffic": profiled_traffic(label, wname),
                        "algorithmic_flops_per_launch": flops, "avg_launch_ms": attn_ms},
           "gpu_launches": LAUNCHES_PER_STEP * steps, "router_near_ties": router_near_ties(wname),
           "device_error": gq.gqe_device_error()}
    if keep_layer:
        out.update(_layer=layer, _x=x, _x_host=x_host)
    else:
        del layer, x
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="gqe", choices=["gqe", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-train", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="measure the headline workload only")
    ap.add_argument("--kernel", default=None,
                    help="time one call alone: attn | attn_bwd | layer_bwd | train_step | decode | decode_step | router | qproj | kv | "
                         "combine | linear | combine_out")
    ap.add_argument("--decode-L", type=int, default=0,
                    help="cache length for --kernel decode / decode_step (default: the decode workload's 32768)")
    ap.add_argument("--workload", default=WORKLOAD, choices=[k for k, v in gi.WORKLOADS.items() if not v.decode])
    ap.add_argument("--sweep", default=None, choices=["gqa"],
                    help="gqa: GQE against dense GQA, prefill T from 2K to 128K (one JSON line per T)")
    ap.add_argument("--sweep-t", default=None, help="comma-separated T values for --sweep")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.kernel:
        return run_kernel(args)
    if args.sweep == "gqa":
        return run_sweep_gqa(args)
    args.warmup = max(args.warmup, 3)

    world, rank, local = dist_env()
    import torch
    import moe_gqa_query_b200 as gq

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    peaks = load_peaks()

    # ---------------- prefill: the headline workload, timed under the clock sampler
    w = gi.WORKLOADS[WORKLOAD]
    dims = w.dims
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    with ClockSampler(local) as clocks:
        head = measure_prefill(gq, WORKLOAD, device, dist, peaks, args.steps, args.warmup, flush, rank, world,
                               keep_layer=True)
    layer, x, x_host = head.pop("_layer"), head.pop("_x"), head.pop("_x_host")
    total_ms = head["ms_per_step"] * args.steps
    value = head["tokens_per_s"]
    roofline = head["roofline"]
    seg_ms_mean = head["segments_ms"]
    err_code = gq.gqe_device_error()
    launches_per_step = LAUNCHES_PER_STEP

    # ---------------- the other prefill workloads: same measurement, fewer steps
    configs = {WORKLOAD: {k_: v for k_, v in head.items()}}
    if not args.no_configs:
        for wn in CONFIG_WORKLOADS:
            if wn == WORKLOAD:
                continue
            configs[wn] = measure_prefill(gq, wn, device, dist, peaks, min(args.steps, 10), args.warmup, flush,
                                          rank, world)
            torch.cuda.empty_cache()

    # ---------------- end to end through host buffers (pinned), on the same step
    # one C-ABI call per step (gqe_layer_forward_host): the batch's input is
    # copied in and its output copied back one sequence at a time, the copies
    # overlapping each other and the compute on three streams; consecutive
    # steps chain on the same streams
    e2e = None
    x_pin = x_host.pin_memory()
    y_pins = [torch.empty((dims.B, dims.T, dims.D), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    n_e2e = max(3, min(args.steps, 20))
    for i in range(3):                                    # warm-up: streams, scratch, tensor maps
        layer.forward_host_c(x_pin, y_pins[i & 1], chunk_seqs=E2E_CHUNK_SEQS)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist, device)
    torch.cuda.synchronize()
    e0.record(stream)
    for i in range(n_e2e):
        done = layer.forward_host_c(x_pin, y_pins[i & 1], chunk_seqs=E2E_CHUNK_SEQS, join=False)
    stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
    e2e = {"value": world * dims.N * n_e2e / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": int(x_pin.numel() * 2), "d2h_bytes_per_step": int(y_pins[0].numel() * 2),
           "steps": n_e2e, "api": f"gqe_layer_forward_host via GQELayer.forward_host_c (pinned host batches, "
                                  f"{E2E_CHUNK_SEQS}-sequence chunks)"}

    # ---------------- decode sub-measurement (64 sequences x 32768-entry cache)
    decode = None
    if not args.no_decode:
        dw = gi.WORKLOADS[DECODE_WORKLOAD]
        dd, Lc = dw.dims, dw.L
        dlayer = gq.GQELayer(dd, {k: torch.from_numpy(v.view(np.int16)) for k, v in gi.layer_weights(dd).items()},
                             device=device)
        gen = torch.Generator(device=device).manual_seed(1234 + rank)
        Kc = torch.empty((dd.B, dd.G, Lc, dd.d), dtype=torch.bfloat16, device=device).normal_(generator=gen)
        Vc = torch.empty_like(Kc).normal_(generator=gen)
        xn = torch.from_numpy(gi.normal_bf16(rank, "xdec", (dd.B, dd.D)).view(np.int16)).view(torch.bfloat16).to(device)
        cl = torch.full((dd.B,), Lc, dtype=torch.int32, device=device)
        for _ in range(3):
            dlayer.decode_step(xn, Kc, Vc, cl)
        torch.cuda.synchronize()
        nd = max(3, min(args.steps, 20))
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(nd)]
        tot = []
        # attention-only timing: same call sequence, events around gqe_attn_decode
        dims_c = gq.make_dims(dd, T=1)
        ws = torch.empty((gq.gqe_workspace_size(dims_c, gq.GQE_OP_ATTN_DECODE, Lc),), dtype=torch.uint8, device=device)
        qd = torch.randn((dd.B, dd.G, 1, dd.k, dd.d), device=device).to(torch.bfloat16)
        qsd = torch.randn((dd.B, 1, dd.d), device=device).to(torch.bfloat16)
        od = torch.empty_like(qd)
        osd = torch.empty_like(qsd)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for i in range(nd):
            ev[i][0].record(stream)
            gq.gqe_attn_decode(dims_c, qd, qsd, Kc, Vc, Lc, cl, od, osd, ws)
            ev[i][1].record(stream)
        s0.record(stream)
        for i in range(nd):
            dlayer.decode_step(xn, Kc, Vc, cl)
        s1.record(stream)
        torch.cuda.synchronize()
        attn_dec_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
        step_dec_ms = s0.elapsed_time(s1) / nd
        bytes_ = decode_attn_bytes(dd, Lc)
        gbs = bytes_ / (attn_dec_ms / 1e3) / 1e9
        decode = {"workload": dw.desc, "tokens_per_s": world * dd.B / (max_over_ranks(step_dec_ms, dist, device) / 1e3),
                  "ms_per_step": step_dec_ms,
                  "roofline": {"bound": "hbm", "kernel": "decode_split_kernel<64> + merge", "achieved": gbs,
                               "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                               "peak_source": f"{peaks['source']} HBM copy",
                               "traffic": profiled_traffic("decode_split_kernel<64> + merge", DECODE_WORKLOAD),
                               "algorithmic_bytes_per_launch": bytes_, "avg_launch_ms": attn_dec_ms},
                  "data": "synthetic: cache ~N(0,1) from a seeded torch generator on the device"}
        del Kc, Vc
        torch.cuda.empty_cache()

    # ---------------- training sub-measurement: forward (keeping what the
    # backward reads) + backward of the same layer on the same batch
    training = None
    if not args.no_train:
        dy = torch.randn((dims.B, dims.T, dims.D), device=device).to(torch.bfloat16)
        _, saved = layer.forward(x, keep=True)
        for _ in range(3):
            layer.backward(x, dy, saved)
        torch.cuda.synchronize()
        nt = max(3, min(args.steps, 20))
        t0, t1, t2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        t0.record(stream)
        for _ in range(nt):
            layer.backward(x, dy, saved)
        t1.record(stream)
        for _ in range(nt):
            _, saved = layer.forward(x, keep=True)
            layer.backward(x, dy, saved)
        t2.record(stream)
        torch.cuda.synchronize()
        bwd_ms = max_over_ranks(t0.elapsed_time(t1) / nt, dist, device)
        step_ms = max_over_ranks(t1.elapsed_time(t2) / nt, dist, device)
        # the attention backward alone (five products per query/key tile pair)
        dc = gq.make_dims(dims)
        ws_a = torch.empty((gq.gqe_workspace_size(dc, gq.GQE_OP_ATTN_BWD),), dtype=torch.uint8, device=device)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        bufs = [torch.empty_like(saved[n]) for n in ("q", "q_sh", "K", "V")]
        call = lambda: gq.gqe_attn_prefill_bwd(dc, saved["q"], saved["q_sh"], saved["K"], saved["V"], saved["o"],  # noqa
                                               saved["o_sh"], saved["lse"], saved["o"], saved["o_sh"], *bufs, ws_a)
        call()
        torch.cuda.synchronize()
        a0.record(stream)
        for _ in range(nt):
            call()
        a1.record(stream)
        torch.cuda.synchronize()
        ab_ms = a0.elapsed_time(a1) / nt
        ab_tf = 2.5 * attn_useful_flops(dims) / ab_ms / 1e9
        training = {"workload": f"{WORKLOAD}: forward(keep) + backward of the layer, dy ~ N(0,1)",
                    "ms_per_step": step_ms, "backward_ms": bwd_ms,
                    "tokens_per_s": world * dims.N / (step_ms / 1e3),
                    "attn_bwd": {"ms": ab_ms, "tflops": ab_tf, "frac": ab_tf / peaks["bf16_tflops"],
                                 "flops_note": "2.5 x the forward's useful causal FLOPs (five products per tile pair)"}}
        del saved, bufs, ws_a
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(WORKLOAD)
        configs[WORKLOAD]["cpu_baseline"] = cpu
        for wn in configs:
            if wn != WORKLOAD:
                configs[wn]["cpu_baseline"] = cpu_baseline(wn)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{WORKLOAD}: {w.desc}", "B": dims.B, "T": dims.T, "d_model": dims.D,
                       "G": dims.G, "E": dims.E, "k": dims.k, "d_head": dims.d, "n_shared": dims.n_shared,
                       "parallelism": f"replicas x{world}", "l2": "flushed between steps (256 MB write)"},
            "segments_ms": seg_ms_mean,
            "segments_note": "per-call CUDA events in separate L2-flushed steps; their sum exceeds "
                             "ms_per_step by the overlap of each kernel's launch with its predecessor",
            "roofline": roofline, "e2e": e2e, "cpu_baseline": cpu, "decode": decode, "training": training,
            "clocks": clocks.summary(), "gpu_launches": launches_per_step * args.steps,
            "device_error": err_code,
            "configs": configs,
            "configs_note": "every prefill workload measured the same way as the headline (layer forward, "
                            "L2 flushed between steps, attention roofline from per-call events); the headline "
                            "is the main layer, the workload the metric is quoted on",
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
