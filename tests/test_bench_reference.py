"""The bench's reference arm runs on the CPU (the oracle, as it stands): its JSON line carries
the contract's keys, and under a multi-rank launch only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra, extra=("--config", "2")):
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "3",
                        "--warmup", "3", *extra], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_arm_json_line():
    lines = _run({})
    assert len(lines) == 1
    j = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
              "cpu_baseline", "e2e"):
        assert k in j, k
    assert j["impl"] == "reference" and j["value"] > 0 and j["steps"] == 3 and j["warmup"] == 3
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert "workload" in j["config"]


def test_reference_arm_other_ranks_print_nothing():
    assert _run({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_both_arms_name_the_same_config():
    """The two arms build their config dicts with one helper: for the default multi-layer
    workload it names every layer, and a multi-rank run names the global batch."""
    sys.path.insert(0, ROOT)
    import bench
    for world in (1, 2):
        sp = bench._global_spec(3, world)
        c = bench._config(3, sp, world, 32)
        assert c["layers"] == 32 and c["global_batch"] == 256 * world and c["config_id"] == 3
        assert "layers 32 of 32" in c["workload"]
    c1 = bench._config(1, bench._global_spec(1, 1), 1, 1)
    assert "layers" not in c1 and "flushed" in c1["l2"]
