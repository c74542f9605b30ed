"""The stored expected values under tests/golden/ are current: each file
equals what its committed generator (which calls only the oracle) writes
today.  CPU only."""
import importlib.util
import json
import os

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    spec = importlib.util.spec_from_file_location(name, os.path.join(GOLDEN, name + ".py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_near_ties_file_is_current():
    mod = _load("near_ties")
    with open(mod.OUT) as f:
        stored = json.load(f)
    fresh = json.loads(json.dumps(mod.compute(stored["seed"])))
    assert stored == fresh
    # every near-tie pair is within the workload's (token, group) range
    for name, v in stored["workloads"].items():
        assert v["near_ties"] == len(v["near_tie_pairs"])
        for t, g in v["near_tie_pairs"]:
            assert 0 <= t < v["tokens"] and 0 <= g < v["groups"]
        assert sum(v["expert_counts"]) == v["tokens"] * v["groups"] * v["k"]
