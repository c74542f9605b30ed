"""Stream and event ordering of gqe_layer_forward_host, checked on the CPU.

The host-buffer layer forward (csrc/layer_fwd.cu) copies chunk i of the
batch in on one stream, runs the layer on a second and copies the result back
on a third, reusing two device buffers per direction and one set of
intermediates, and lets calls in a row chain on the same streams.  Whether
every reuse is ordered depends only on the CUDA events it records and waits
for, so it is checked here without a GPU: the file is compiled unchanged
against tests/fake_cuda_runtime.cpp, whose stand-ins for the CUDA calls and for
the per-step entry points log every copy, kernel step, event record and
stream wait with the byte ranges it reads and writes.  From that log:

  - the happens-before graph of CUDA's rules (work on one stream runs in
    issue order; a wait orders the stream's later work after the work
    captured by the event's latest record issued before the wait);
  - no race: any two accesses to overlapping bytes, one of them a write, are
    ordered by that graph;
  - data flow: executing the log in many random orders that respect the
    graph, each chunk's host output derives from that chunk's input (and the
    weights) alone;
  - the documented end state: the last work each call leaves on the compute
    stream (and on the copy-back stream) comes after every copy back;
  - calls in a row with batches of different sizes (one chunk_seqs) chain
    race-free; with another chunk_seqs on the same workspace they would not,
    which is why the header asks for a synchronisation there.

A planted mistake, one of the waits taken out of the log, must be caught.
Errors injected on the host into one step or one copy come back as the
call's status, and the call releases its events on that path too.
"""
import ctypes
import os
import random
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"

GQE_OP_LAYER_FORWARD_HOST = 6


class Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("d_model", ctypes.c_int),
                ("G", ctypes.c_int), ("E", ctypes.c_int), ("k", ctypes.c_int),
                ("d_head", ctypes.c_int), ("n_shared", ctypes.c_int),
                ("shared_kv_group", ctypes.c_int), ("renorm_scope", ctypes.c_int),
                ("scale", ctypes.c_float), ("output_mode", ctypes.c_int)]


class Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("Wr", "bias", "Wq", "Wsh", "Wk", "Wv", "Wo")]


@pytest.fixture(scope="module")
def fake(tmp_path_factory):
    gxx = shutil.which("g++")
    if not gxx or not os.path.exists(os.path.join(CUDA_INC, "cuda_runtime.h")):
        pytest.skip("needs g++ and the CUDA headers")
    out = str(tmp_path_factory.mktemp("fake") / "libfake_pipeline.so")
    # -Bsymbolic: the library's calls bind to its own stand-ins even when a
    # real CUDA runtime is already loaded into the process
    cmd = [gxx, "-std=c++17", "-O1", "-fPIC", "-shared", "-Wl,-Bsymbolic", "-x", "c++",
           os.path.join(ROOT, "moe_gqa_query_b200", "csrc", "layer_fwd.cu"),
           os.path.join(ROOT, "tests", "fake_cuda_runtime.cpp"), "-I", CUDA_INC, "-o", out]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    lib = ctypes.CDLL(out)
    lib.fake_log_line.restype = ctypes.c_char_p
    lib.fake_fail.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.gqe_workspace_size.argtypes = [ctypes.POINTER(Dims), ctypes.c_int, ctypes.c_int,
                                       ctypes.POINTER(ctypes.c_size_t)]
    lib.gqe_layer_forward_host.argtypes = [ctypes.POINTER(Dims), ctypes.POINTER(Weights), ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return lib


# made-up addresses: nothing is dereferenced
WS = 0x1000_0000_0000
X_HOST = 0x2000_0000_0000
Y_HOST = 0x3000_0000_0000
W_BASE = 0x4000_0000_0000
CALL_STRIDE = 1 << 36


def _dims(B, T, D):
    return Dims(B=B, T=T, d_model=D, G=2, E=3, k=2, d_head=64, n_shared=1, shared_kv_group=1,
                renorm_scope=0, scale=0.0, output_mode=0)


def _run(fake, Bs, chunks, streams=(0x11, 0x22, 0x33), T=4, D=128, expect=0):
    """Issues one host-buffer forward per entry of Bs (batch sizes) and chunks
    (chunk_seqs), in a row on the same streams and workspace, each on its own
    host x and y; returns the parsed log."""
    w = Weights(**{n: W_BASE + i * 0x10000 for i, n in enumerate(("Wr", "bias", "Wq", "Wsh", "Wk", "Wv", "Wo"))})
    w.bias = None
    need = 0
    for chunk in chunks:
        n = ctypes.c_size_t(0)
        assert fake.gqe_workspace_size(ctypes.byref(_dims(chunk, T, D)), GQE_OP_LAYER_FORWARD_HOST, 0,
                                       ctypes.byref(n)) == 0
        need = max(need, n.value)
    fake.fake_log_clear()
    for c, (B, chunk) in enumerate(zip(Bs, chunks)):
        st = fake.gqe_layer_forward_host(ctypes.byref(_dims(B, T, D)), ctypes.byref(w), X_HOST + c * CALL_STRIDE,
                                         Y_HOST + c * CALL_STRIDE, chunk, WS, need, *streams)
        assert st == expect
    lines = [fake.fake_log_line(i).decode() for i in range(fake.fake_log_size())]
    seq_bytes = T * D * 2
    return [_parse(s) for s in lines], seq_bytes


def _ranges(field):
    out = []
    for item in field.split("=", 1)[1].split(","):
        if item:
            p, n = item.split(":")
            out.append((int(p, 16), int(p, 16) + int(n)))
    return out


def _parse(line):
    f = line.split()
    kind = f[0]
    if kind in ("create", "destroy"):
        return dict(kind=kind, event=int(f[1], 16))
    if kind == "record":
        return dict(kind=kind, event=int(f[1], 16), stream=int(f[2], 16))
    if kind == "wait":
        return dict(kind=kind, stream=int(f[1], 16), event=int(f[2], 16))
    if kind == "copy":
        return dict(kind=kind, stream=int(f[1], 16), name=f[2], reads=_ranges(f[3]), writes=_ranges(f[4]))
    assert kind == "kernel", line
    return dict(kind=kind, stream=int(f[1], 16), name=f[2], reads=_ranges(f[3]), writes=_ranges(f[4]))


def _graph(ops):
    """Predecessors and ancestor bitsets of the stream operations (issue
    order is a topological order of CUDA's happens-before)."""
    nodes, preds = [], []
    last_on_stream, last_record = {}, {}
    for op in ops:
        if op["kind"] in ("create", "destroy"):
            continue
        i = len(nodes)
        p = []
        if op["stream"] in last_on_stream:
            p.append(last_on_stream[op["stream"]])
        if op["kind"] == "wait" and op["event"] in last_record:
            p.append(last_record[op["event"]])
        if op["kind"] == "record":
            last_record[op["event"]] = i
        last_on_stream[op["stream"]] = i
        nodes.append(op)
        preds.append(p)
    anc = []
    for i, p in enumerate(preds):
        a = 0
        for j in p:
            a |= anc[j] | (1 << j)
        anc.append(a)
    return nodes, preds, anc


def _races(nodes, anc):
    out = []
    acc = [(i, r, False) for i, n in enumerate(nodes) for r in n.get("reads", [])]
    acc += [(i, r, True) for i, n in enumerate(nodes) for r in n.get("writes", [])]
    for x in range(len(acc)):
        i, (a0, a1), wa = acc[x]
        for y in range(x + 1, len(acc)):
            j, (b0, b1), wb = acc[y]
            if i == j or not (wa or wb) or a1 <= b0 or b1 <= a0:
                continue
            lo, hi = min(i, j), max(i, j)
            if not (anc[hi] >> lo) & 1:
                out.append((nodes[lo].get("name", nodes[lo]["kind"]), nodes[hi].get("name", nodes[hi]["kind"])))
    return out


class _Memory:
    """Byte ranges -> the set of input labels their contents derive from."""

    def __init__(self):
        self.seg = []          # (start, end, labels)

    def write(self, a, b, labels):
        keep = []
        for s, e, lab in self.seg:
            if e <= a or b <= s:
                keep.append((s, e, lab))
                continue
            if s < a:
                keep.append((s, a, lab))
            if b < e:
                keep.append((b, e, lab))
        keep.append((a, b, labels))
        self.seg = keep

    def read(self, a, b):
        labels, covered = set(), 0
        for s, e, lab in self.seg:
            if e <= a or b <= s:
                continue
            labels |= lab
            covered += min(b, e) - max(a, s)
        if covered < b - a:
            labels.add("uninitialised")
        return labels


def _simulate(nodes, preds, rng, Bs, chunk, seq_bytes):
    """Runs the nodes in one random order that respects the graph; returns,
    per (call, sequence), the labels the host output derives from."""
    mem = _Memory()
    for c, B in enumerate(Bs):
        for b in range(B):
            base = X_HOST + c * CALL_STRIDE + b * seq_bytes
            mem.write(base, base + seq_bytes, frozenset({("x", c, b // chunk)}))
    mem.write(W_BASE, W_BASE + 0x100000, frozenset({"W"}))
    succ = [[] for _ in nodes]
    indeg = [len(p) for p in preds]
    for i, p in enumerate(preds):
        for j in p:
            succ[j].append(i)
    ready = [i for i, d in enumerate(indeg) if d == 0]
    done = 0
    while ready:
        i = ready.pop(rng.randrange(len(ready)))
        n = nodes[i]
        if "reads" in n:
            lab = set()
            for a, b in n["reads"]:
                lab |= mem.read(a, b)
            for a, b in n["writes"]:
                mem.write(a, b, frozenset(lab))
        done += 1
        for j in succ[i]:
            indeg[j] -= 1
            if indeg[j] == 0:
                ready.append(j)
    assert done == len(nodes)
    out = {}
    for c, B in enumerate(Bs):
        for b in range(B):
            base = Y_HOST + c * CALL_STRIDE + b * seq_bytes
            out[(c, b)] = mem.read(base, base + seq_bytes)
    return out


CASES = [  # (batch size of each call in the row, chunk_seqs)
    ((8, 8), 1), ((8, 8), 3), ((8, 8, 8), 8), ((5, 5, 5), 2), ((1, 1, 1), 1), ((6, 6), 4), ((7,), 7),
    ((8, 5, 3), 2),         # batches of different sizes chain on one layout
    ((2, 9, 1), 4),         # chunk_seqs above the batch: one chunk
]


@pytest.mark.parametrize("Bs,chunk", CASES)
@pytest.mark.parametrize("one_stream", [False, True])
def test_host_pipeline_is_race_free_and_keeps_chunks_apart(fake, Bs, chunk, one_stream):
    streams = (0x11, 0x11, 0x11) if one_stream else (0x11, 0x22, 0x33)
    ops, seq_bytes = _run(fake, Bs, [chunk] * len(Bs), streams)
    n_chunks = sum(-(-B // chunk) for B in Bs)
    assert sum(op["kind"] == "copy" for op in ops) == 2 * n_chunks
    assert sum(op["kind"] == "kernel" for op in ops) == 5 * n_chunks
    created = [op["event"] for op in ops if op["kind"] == "create"]
    destroyed = [op["event"] for op in ops if op["kind"] == "destroy"]
    assert sorted(created) == sorted(destroyed)         # every event released
    nodes, preds, anc = _graph(ops)
    assert _races(nodes, anc) == []
    rng = random.Random(1234 + sum(Bs) * 31 + chunk)
    for _ in range(20):
        got = _simulate(nodes, preds, rng, Bs, chunk, seq_bytes)
        for (c, b), labels in got.items():
            assert labels == {("x", c, b // chunk), "W"}, (c, b, labels)
    # y_host is complete once the compute stream's (or the copy-back
    # stream's) last work has run: every copy back precedes both
    d2h = [i for i, n in enumerate(nodes) if n["kind"] == "copy" and n["name"] == "d2h"]
    for s in set(streams[1:]):
        last = max(i for i, n in enumerate(nodes) if n["stream"] == s)
        assert all(i == last or (anc[last] >> i) & 1 for i in d2h)


@pytest.mark.parametrize("drop", ["x_slot_reuse", "y_slot_reuse", "next_call_inputs", "next_call_outputs"])
def test_a_missing_wait_is_caught(fake, drop):
    """Planted mistakes: taking any one of the pipeline's waits out of the log
    leaves a race that the check finds."""
    ops, _ = _run(fake, (8, 8), (1, 1))
    waits = [i for i, op in enumerate(ops) if op["kind"] == "wait"]
    s_in, s_cmp = 0x11, 0x22
    # the first call's waits, in issue order: on s_in for chunks >= 2 (x slot
    # reuse), on s_cmp after each copy in and, for chunks >= 2, for the y
    # slot; then the two at the call's end
    first_call_end = max(i for i, op in enumerate(ops[: len(ops) // 2 + 1]) if op["kind"] == "destroy")
    w1 = [i for i in waits if i < first_call_end]
    in_waits = [i for i in w1 if ops[i]["stream"] == s_in]
    cmp_waits = [i for i in w1 if ops[i]["stream"] == s_cmp]
    pick = {
        "x_slot_reuse": in_waits[0],
        "y_slot_reuse": cmp_waits[3],        # chunk 2: the copy-in wait is cmp_waits[2]
        "next_call_inputs": in_waits[-1],
        "next_call_outputs": cmp_waits[-1],
    }[drop]
    broken = ops[:pick] + ops[pick + 1:]
    nodes, _, anc = _graph(broken)
    assert _races(nodes, anc), f"dropping the {drop} wait went unnoticed"


def test_another_chunk_size_on_the_same_workspace_needs_a_synchronisation(fake):
    """Why the header asks callers to let stream_out's work complete before
    the workspace serves another chunk_seqs: the layout moves, and the next
    call's copy in can land on a buffer the previous call is still copying
    back from."""
    ops, _ = _run(fake, (8, 8), (1, 4))
    nodes, _, anc = _graph(ops)
    assert ("d2h", "h2d") in _races(nodes, anc)


@pytest.mark.parametrize("step,copy", [(0, -1), (3, -1), (7, -1), (19, -1), (-1, 0), (-1, 5), (-1, 7)])
def test_a_failing_step_or_copy_is_reported_and_releases_the_events(fake, step, copy):
    """An error from one of the steps (injected on the host, GQE_ERR_CUDA from
    the fifth step say) or from a copy comes back as the call's status, and
    every event the call created is released on that path too (8 sequences in
    chunks of 2: 20 steps, 8 copies)."""
    fake.fake_fail(step, 4, copy)
    try:
        ops, _ = _run(fake, (8,), (2,), expect=4)
    finally:
        fake.fake_fail(-1, 0, -1)
    created = sorted(op["event"] for op in ops if op["kind"] == "create")
    destroyed = sorted(op["event"] for op in ops if op["kind"] == "destroy")
    assert len(created) == 5 and created == destroyed
    n_steps = sum(op["kind"] == "kernel" for op in ops)
    if step >= 0:
        assert n_steps == step          # nothing launched after the failing step
