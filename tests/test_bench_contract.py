"""bench.py's reference arm (the fp64 oracle on the host cores) prints one JSON line
with the fields the benchmark contract asks for; ranks other than 0 print nothing.
CPU only (one oracle step, ~10 s)."""
import json
import os
import subprocess
import sys

ROOT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "..")


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                           "--warmup", "0"], capture_output=True, text=True, env=env, timeout=600)


def test_reference_arm_prints_the_contract_line():
    r = _run({})
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["higher_is_better"] is True and line["steps"] == 1 and line["warmup"] == 0
    assert "workload" in line["config"]
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_runs_on_rank_zero_only():
    r = _run({"RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_plan_timing_on_the_benchmark_layout():
    """The host plan that the bench line reports under "plan" builds the long-context layout
    (cp=16, T=131072) on the CPU and closes every plan it timed."""
    sys.path.insert(0, ROOT)
    import bench
    import context_packed_sequence_cp_b200 as thd
    from context_packed_sequence_cp_b200 import synthetic as syn
    cu = syn.cu_seqlens_of(syn.doc_lengths(bench.WORKLOAD, 0))
    ms = bench.time_plan(thd, cu, syn.WORKLOADS[bench.WORKLOAD].cp, reps=2)
    assert 0 < ms < 10_000
