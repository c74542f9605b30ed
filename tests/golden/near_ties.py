"""Writes tests/golden/near_ties.json: the router's near-ties in every workload.

A (token, group) pair is a near-tie when its k-th and (k+1)-th largest router
logits differ by less than 1e-4; both expert choices are then correct, so the
parity tests exempt such pairs from the exact TopK comparison and count them.
This script computes them with the fp64 oracle alone (oracle.router_topk) on
the seeded inputs the parity tests and the benchmark use (seed 0: x, Wr and
the workload's router bias; the decode workload's new-token rows come from the
``xdec`` stream).  It calls nothing of the CUDA library.

  python tests/golden/near_ties.py            # rewrite the file
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gqe_inputs as gi  # noqa: E402
import oracle as orc  # noqa: E402

NEAR_TIE = 1e-4
OUT = os.path.join(HERE, "near_ties.json")


def workload_router_input(w: gi.Workload, seed: int = 0) -> np.ndarray:
    """The router's input rows of a workload: x [N, D] (bf16 bits)."""
    dims = w.dims
    if w.decode:
        return gi.normal_bf16(seed, "xdec", (dims.B, dims.D))
    return gi.layer_input(dims, seed).reshape(dims.N, dims.D)


def near_ties(w: gi.Workload, seed: int = 0) -> dict:
    dims = w.dims
    x = workload_router_input(w, seed)
    Wr = gi.layer_weights(dims, seed)["Wr"]
    r = orc.router_topk(x, Wr, dims.G, dims.E, dims.k, gi.router_bias(w, seed), dims.renorm_scope)
    pairs = np.argwhere(r["margin"] < NEAR_TIE)
    counts, _ = orc.router_stats(r["probs"], r["idx"], dims.G, dims.E)
    return {"tokens": int(x.shape[0]), "groups": dims.G, "E": dims.E, "k": dims.k,
            "pairs": int(x.shape[0]) * dims.G, "near_ties": int(len(pairs)),
            "near_tie_pairs": [[int(t), int(g)] for t, g in pairs],
            "min_margin": float(r["margin"].min()) if np.isfinite(r["margin"]).any() else None,
            "expert_counts": [int(c) for c in counts]}


def compute(seed: int = 0) -> dict:
    return {
        "what": "router near-ties (k-th/(k+1)-th logit margin < 1e-4) per workload, from the fp64 oracle; "
                "expert_counts are the oracle's per-(group, expert) selection counts",
        "cite": "GQE study note §3-2 2) (router score, in-group softmax, TopK); the TopK of a near-tie pair "
                "is decided by rounding, so either expert is a correct choice",
        "seed": seed,
        "threshold": NEAR_TIE,
        "workloads": {name: near_ties(w, seed) for name, w in gi.WORKLOADS.items()},
    }


def main():
    data = compute()
    with open(OUT, "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")
    for name, v in data["workloads"].items():
        print(f"{name}: {v['near_ties']} near-ties of {v['pairs']} (token, group) pairs")


if __name__ == "__main__":
    main()
