"""The JSON contract of bench.py, checked on the CPU through its reference arm
(the oracle on host cores), plus the shape of the committed DRAM-traffic
records that bench.py reads for its roofline line."""
import glob
import json
import os
import re
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _bench(*args, env_extra=None, timeout=300):
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    return [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]


def test_reference_arm_prints_one_contract_line():
    lines = _bench("--impl", "reference", "--steps", "3", "--warmup", "3")
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference"
    for key, typ in (("metric", str), ("unit", str), ("value", float), ("ms_per_step", float), ("dtype", str),
                     ("data", str), ("scaling", str)):
        assert isinstance(d[key], typ), key
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["config"]["workload"] == "llama3.1-8b_q_proj_p10_M512_N4096_K4096"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert cb["host_cores"] >= cb["cores"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["unit"] == d["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_on_rank_zero_only():
    lines = _bench("--impl", "reference", "--steps", "3", "--warmup", "3",
                   env_extra={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert lines == []


@pytest.mark.parametrize("workload", ["llama3.1-8b_layer@M1", "llama3.1-8b_search_q_gate_D16"])
def test_workloads_without_a_reference_arm_say_so(workload):
    lines = _bench("--impl", "reference", "--workload", workload, "--steps", "3", "--warmup", "3")
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["unavailable"]


def test_traffic_records_are_well_formed():
    import bench
    csrc = os.path.join(ROOT, "mixed_precision_quantized_act_b200", "csrc")
    paths = sorted(glob.glob(os.path.join(ROOT, "profiles", "*_traffic.json")))
    assert paths
    for path in paths:
        with open(path) as f:
            rec = json.load(f)
        for e in rec.get("entries", [rec]):
            assert e["sources"] and all(os.path.exists(os.path.join(csrc, s)) for s in e["sources"]), path
            assert re.fullmatch(r"[0-9a-f]{16}", e["source_hash"])
            assert e["dram_bytes_per_launch"] == e["dram_bytes_read_per_launch"] + e["dram_bytes_write_per_launch"]
            assert e["algorithmic_bytes_per_launch"] > 0
            assert "--clock-control none" in e["command"] and "ncu" in e["command"]
            assert bench.layer_for(e["workload"]) is not None
            assert bench.source_hash(e["sources"]) == bench.source_hash(e["sources"])
