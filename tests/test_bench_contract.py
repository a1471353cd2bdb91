"""The benchmark's JSON-line contract, checked on its CPU arm (no GPU needed).

``bench.py --impl reference`` times the FP64 oracle on the host cores; its line
must carry the same keys as the CUDA arm's, for the workload it was asked for,
and only rank 0 of a multi-process launch prints it.
"""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ARGS = ["--impl", "reference", "--steps", "2", "--warmup", "0", "--workload", "tiny", "--reference-rows", "8"]


def _run(env_extra=None):
    env = dict(os.environ, **(env_extra or {}))
    r = subprocess.run([sys.executable, "bench.py", *ARGS], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return [ln for ln in r.stdout.splitlines() if ln.startswith("{")]


def test_reference_line_has_the_contract_keys():
    lines = _run()
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 0 and d["n_gpus"] == 1
    assert d["unit"] == "pairs/s" and d["higher_is_better"] is True and d["value"] > 0
    assert d["config"]["workload"].startswith("tiny: T=256")
    assert d["config"]["T"] == 256 and d["config"]["H"] == 12
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] >= 1 and "8 random" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "pairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_only_rank_zero_prints():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}) == []


def test_pass_ms_sums_the_stages():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    stages = {n: float(i + 1) for i, n in enumerate(bench.FWD_STAGES + bench.BWD_STAGES)}
    got = bench.pass_ms(stages)
    assert got == {"forward": 3.0, "backward": 3.0 + 4 + 5 + 6 + 7, "total": 28.0}
    assert bench.pass_ms({}) == {"forward": 0.0, "backward": 0.0, "total": 0.0}
