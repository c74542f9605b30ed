"""Seeded synthetic inputs for the GQE attention forward.

This module is shared by the fp64 oracle's tests, the CUDA parity tests and the
benchmark. It holds shapes, seeds and random draws only: none of the method's
arithmetic lives here (no projection, softmax, top-k or attention).

Recipe (every tensor):
  * generator: numpy PCG64 seeded with ``[seed, tensor_id, i]``, one stream per
    index ``i`` of the leading axis, so a slice along that axis can be
    regenerated alone;
  * values: float32 standard normals times ``std``, rounded to bfloat16 with
    round-to-nearest-even and kept as raw uint16 bit patterns.

Shapes follow the five workloads the GQE pages discuss (the tiny 2-group case,
the paper's 16-query / 8-KV-head layer at context 2048, a 32K-token long
context, a wide 8-expert group with skewed routing, and a decode step against a
32K-entry cache). x ~ N(0, 1); every weight ~ N(0, 0.02^2).
"""
from __future__ import annotations

import dataclasses
import numpy as np

# tensor ids for the seeded streams
TID = dict(x=1, Wr=2, Wq=3, Wk=4, Wv=5, Wsh=6, Wo=7, bias=8, Kc=9, Vc=10,
           route=11, q=12, K=13, V=14, qsh=15, o=16, osh=17, w=18, xdec=19,
           do=20, dosh=21, dy=22, dh=23, dw=24)

WEIGHT_STD = 0.02


@dataclasses.dataclass(frozen=True)
class GQEDims:
    """Shape of one GQE layer call.

    B sequences of T tokens, model width D, G KV groups of E query experts each,
    k experts routed per (token, group), head width d, n_shared always-on
    shared query heads (0 or 1) reading KV group ``sg``.  ``renorm_scope`` 0
    normalises the selected router probabilities over all k*G selections of a
    token, 1 within each group, 2 not at all.  ``scale`` 0 means 1/sqrt(d).
    ``output_mode`` 0 is GQE's output (hard slots, weighted-sum slot, shared
    head); 1 hard slots only (+ shared); 2 router-weighted hard slots (+ shared).
    """
    B: int
    T: int
    D: int
    G: int
    E: int
    k: int
    d: int
    n_shared: int = 1
    sg: int = 0
    renorm_scope: int = 0
    scale: float = 0.0
    output_mode: int = 0

    @property
    def N(self) -> int:
        return self.B * self.T

    @property
    def slots(self) -> int:
        """Output-projection input slots: k*G hard (+ 1 weighted sum in mode 0) + n_shared."""
        return self.k * self.G + (1 if self.output_mode == 0 else 0) + self.n_shared

    @property
    def h_active(self) -> int:
        """Query heads whose attention is computed per token: k*G + n_shared."""
        return self.k * self.G + self.n_shared

    def replace(self, **kw) -> "GQEDims":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    dims: GQEDims
    bias: str = "none"          # none | normal | expert0
    bias_beta: float = 0.0
    decode: bool = False
    L: int = 0                  # decode cache length
    desc: str = ""


WORKLOADS = {
    "tiny_prefill": Workload(
        "tiny_prefill", GQEDims(B=1, T=128, D=256, G=2, E=2, k=1, d=64),
        desc="B1 T128 D256, 2 KV groups x 2 experts, top-1, 1 shared head, d64"),
    "main_prefill": Workload(
        "main_prefill", GQEDims(B=8, T=2048, D=1024, G=8, E=2, k=1, d=64),
        desc="paper main layer: 16 query experts / 8 KV heads, top-1 of 2, +1 shared, "
             "B8 T2048 D1024 d64"),
    "long_prefill": Workload(
        "long_prefill", GQEDims(B=1, T=32768, D=1024, G=8, E=2, k=1, d=64),
        bias="normal",
        desc="main layer shape at B1 T32768, router bias ~N(0,1) per expert"),
    "wide_skewed_prefill": Workload(
        "wide_skewed_prefill", GQEDims(B=2, T=8192, D=4096, G=4, E=8, k=4, d=128),
        bias="expert0", bias_beta=3.0,
        desc="D4096, 32 experts / 4 KV heads (E8, top-4), +1 shared, d128, B2 T8192; "
             "router bias +3 on expert 0 of every group"),
    "decode": Workload(
        "decode", GQEDims(B=64, T=1, D=1024, G=8, E=2, k=1, d=64),
        decode=True, L=32768,
        desc="main layer shape, 64 sequences x 1 new token against a dense "
             "[64,8,32768,64] bf16 KV cache ~N(0,1)"),
}


# ----------------------------------------------------------------------------
# bfloat16 bit handling (storage format only)

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest, ties to even); uint16 bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(u, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _stream(seed: int, tid: int, i: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, tid, i]))


def normal_bf16(seed: int, name: str, shape, std: float = 1.0, rows=None) -> np.ndarray:
    """bf16 bits of N(0, std^2) draws; one stream per index of axis 0.

    ``rows`` (an iterable of axis-0 indices) regenerates only those slices.
    """
    shape = tuple(int(s) for s in shape)
    tid = TID[name]
    idx = range(shape[0]) if rows is None else list(rows)
    out = np.empty((len(idx),) + shape[1:], dtype=np.uint16)
    for j, i in enumerate(idx):
        v = _stream(seed, tid, i).standard_normal(shape[1:], dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out[j] = f32_to_bf16_bits(v)
    return out


def router_bias(w: Workload, seed: int = 0):
    """float32 router bias [G*E] of the workload, or None."""
    G, E = w.dims.G, w.dims.E
    if w.bias == "none":
        return None
    if w.bias == "normal":
        return _stream(seed, TID["bias"], 0).standard_normal(G * E, dtype=np.float32)
    if w.bias == "expert0":
        b = np.zeros((G, E), dtype=np.float32)
        b[:, 0] = np.float32(w.bias_beta)
        return b.reshape(-1)
    raise ValueError(w.bias)


def layer_weights(dims: GQEDims, seed: int = 0) -> dict:
    """bf16 weights of one layer (nn.Linear [out, in] layout except Wr).

    Wr [D, G*E]; Wq [G, E, d, D]; Wk, Wv [G*d, D]; Wsh [d, D];
    Wo [D, slots*d].
    """
    D, G, E, d = dims.D, dims.G, dims.E, dims.d
    s = WEIGHT_STD
    return dict(
        Wr=normal_bf16(seed, "Wr", (D, G * E), s),
        Wq=normal_bf16(seed, "Wq", (G, E, d, D), s),
        Wk=normal_bf16(seed, "Wk", (G * d, D), s),
        Wv=normal_bf16(seed, "Wv", (G * d, D), s),
        Wsh=normal_bf16(seed, "Wsh", (dims.n_shared * d, D), s),
        Wo=normal_bf16(seed, "Wo", (D, dims.slots * d), s),
    )


def layer_input(dims: GQEDims, seed: int = 0, rows=None) -> np.ndarray:
    """x [B, T, D] bf16 bits ~ N(0, 1) (``rows`` selects sequences)."""
    return normal_bf16(seed, "x", (dims.B, dims.T, dims.D), 1.0, rows=rows)


def random_routing(dims: GQEDims, seed: int = 0, skew0: float = 0.0) -> np.ndarray:
    """A valid routing decision, drawn directly: int32 [B*T, G, k].

    For every (token, group) a k-subset of the E experts, in ascending order.
    ``skew0`` > 0 puts expert 0 in the subset with that probability (load
    imbalance); the rest are uniform.  Used to drive the projection, attention
    and combine calls on their own, independent of any router.
    """
    N, G, E, k = dims.N, dims.G, dims.E, dims.k
    rng = _stream(seed, TID["route"], 0)
    keys = rng.random((N, G, E))
    if skew0 > 0:
        force = rng.random((N, G)) < skew0
        keys[..., 0] = np.where(force, -1.0, keys[..., 0])
    sel = np.argsort(keys, axis=-1, kind="stable")[..., :k]
    return np.sort(sel, axis=-1).astype(np.int32)


def random_weights_simplex(dims: GQEDims, seed: int = 0) -> np.ndarray:
    """float32 [B*T, G, k] positive weights summing to 1 over (G, k) per token."""
    rng = _stream(seed, TID["w"], 0)
    w = rng.random((dims.N, dims.G, dims.k)).astype(np.float64) + 0.05
    w /= w.sum(axis=(1, 2), keepdims=True)
    return w.astype(np.float32)
