"""bench.py's reference arm on the CPU: `--impl reference` times the f64
oracle on a bounded sample of the workload and prints one JSON line with
the keys the driver reads; under torchrun only rank 0 prints."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.strip()]


def test_reference_arm_prints_one_json_line():
    lines = _run({"WORLD_SIZE": "1", "RANK": "0"})
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"].startswith("prefill q-rows/s")
    assert d["unit"] == "q-rows/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "q-rows/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["decode"]["unit"] == "tok/s" and d["decode"]["value"] > 0


def test_reference_arm_is_silent_on_other_ranks():
    assert _run({"WORLD_SIZE": "2", "RANK": "1"}) == []


def test_e2e_copy_groups_cover_the_prompt_in_order():
    """The end-to-end leg's copy groups: E2E_FIRST chunks, then E2E_GROUP at
    a time, every chunk exactly once and in prompt order."""
    sys.path.insert(0, ROOT)
    import bench
    chunks = [(768 * i, 768) for i in range(21)] + [(16128, 256)]
    groups = bench.e2e_groups(chunks)
    assert [c for g in groups for c in g] == chunks
    assert len(groups[0]) == bench.E2E_FIRST
    assert all(len(g) == bench.E2E_GROUP for g in groups[1:-1]) and 0 < len(groups[-1]) <= bench.E2E_GROUP
    for first, size in ((0, 4), (1, 1), (4, 4), (30, 4), (2, 50)):
        got = bench.e2e_groups(chunks, first, size)
        assert [c for g in got for c in g] == chunks and all(got)
