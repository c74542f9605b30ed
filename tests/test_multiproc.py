"""Host logic of the benchmark, on CPU.

The GQE path does not shard across GPUs here: each rank runs its own replica.
The only cross-rank steps are the barrier around the timed region and the max
over ranks of the measured time; these run as world_size-2 gloo ranks.  Also:
the work counts behind the roofline, the reference arm's JSON line, the
traffic lookup that follows the captured kernel source, and the peak fallback.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    w, r, local = bench.dist_env()
    assert (w, r, local) == (world, rank, rank)
    dist = bench.init_dist(world, "gloo")
    bench.barrier(dist)
    local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
    total = bench.max_over_ranks(local_ms, dist)
    out[rank] = total
    bench.barrier(dist)
    dist.destroy_process_group()


def test_two_rank_max_over_ranks():
    world = 2
    port = _free_port()
    out = mp.Manager().dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == out[1] == 15.0


def test_single_rank_has_no_process_group():
    import bench
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(3.5, None) == 3.5


def test_work_counts():
    import bench
    import gqe_inputs as gi
    main = gi.WORKLOADS["main_prefill"].dims
    assert bench.attn_useful_flops(main) == pytest.approx(3.867e10, rel=1e-3)
    dec = gi.WORKLOADS["decode"]
    assert bench.decode_attn_bytes(dec.dims, dec.L) == pytest.approx(4.295e9, rel=1e-3)


def _bench(args, env_extra):
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, "bench.py", *args], cwd=root, env=env, capture_output=True,
                          text=True, timeout=600)


def test_reference_arm_json_line():
    """`bench.py --impl reference`: the oracle timed on the host cores, one JSON
    line with the main arm's metric, unit and direction, a cpu_baseline that
    describes the run and an e2e object with no host-device bytes."""
    r = _bench(["--impl", "reference", "--steps", "1", "--warmup", "0"], {})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    import bench
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["value"] > 0 and line["steps"] == 1 and line["n_gpus"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    """Under torchrun only rank 0 runs and prints the reference arm."""
    r = _bench(["--impl", "reference", "--steps", "1", "--warmup", "0", "--gpus", "2"],
               {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_roofline_traffic_follows_the_captured_source(tmp_path, monkeypatch):
    """The bench reports a kernel's ncu DRAM traffic only for the captured
    kernel and workload, and only while the kernel's source file still hashes
    to the captured version; anything else gives null."""
    import hashlib
    import shutil
    import bench
    label = "attn_prefill_single_kernel (d=64)"
    assert bench.profiled_traffic("no such kernel") is None
    src = tmp_path / "moe_gqa_query_b200" / "csrc" / "attn_prefill.cu"
    src.parent.mkdir(parents=True)
    shutil.copy(os.path.join(bench.ROOT, "moe_gqa_query_b200", "csrc", "attn_prefill.cu"), src)
    (tmp_path / "profiles").mkdir()
    entry = {"kernel": label, "workload": "main_prefill", "source": "moe_gqa_query_b200/csrc/attn_prefill.cu",
             "source_sha256_16": hashlib.sha256(src.read_bytes()).hexdigest()[:16],
             "dram_read_bytes": 1000, "dram_write_bytes": 24}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"captures": [entry]}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.profiled_traffic(label, "main_prefill") == 1024
    assert bench.profiled_traffic(label, "long_prefill") is None
    src.write_text(src.read_text() + "\n// edited\n")
    assert bench.profiled_traffic(label, "main_prefill") is None


def test_committed_traffic_entries_are_well_formed():
    import bench
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        caps = json.load(f)["captures"]
    for c in caps:
        assert os.path.exists(os.path.join(bench.ROOT, c["source"]))
        assert c["workload"] in bench.gi.WORKLOADS
        assert int(c["dram_read_bytes"]) > 0 and int(c["dram_write_bytes"]) >= 0


def test_peaks_fall_back_without_the_measured_file(tmp_path, monkeypatch):
    import bench
    p = bench.load_peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert p["source"] == "measured" and p["bf16_tflops"] > 0 and p["hbm_gbs"] > 0
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = bench.load_peaks()
    assert f["source"] == "fallback"
    assert (f["hbm_gbs"], f["bf16_tflops"]) == (6650.0, 1590.0)


def test_router_near_ties_come_from_the_oracle_file():
    # the bench line's per-workload near-tie counts are those the oracle wrote
    # into tests/golden/near_ties.json; an unknown workload reports none
    import bench
    with open(os.path.join(bench.ROOT, "tests", "golden", "near_ties.json")) as f:
        golden = json.load(f)["workloads"]
    for wname, v in golden.items():
        got = bench.router_near_ties(wname)
        assert got["pairs"] == v["near_ties"] and got["of"] == v["pairs"]
    assert bench.router_near_ties("no_such_workload") is None
