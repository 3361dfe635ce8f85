"""The bench's reference arm (the float64 oracle on the host cores) keeps the
one-JSON-line contract, and under a multi-rank launch only rank 0 works."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CMD = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "single",
       "--steps", "1", "--warmup", "0"]


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run(CMD, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["ms_per_step"] == 1e3 / d["value"] or abs(d["ms_per_step"] * d["value"] - 1e3) < 1e-6
    assert d["config"]["workload"]
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run(CMD, capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_oracle_sample_plans_cover_one_layer_or_one_of_each_shape():
    sys.path.insert(0, ROOT)
    import bench
    import workloads as WL
    for wl, layers in ((WL.llama_3p8b_aurora(), 28), (WL.llama_3p8b_plain(), 28), (WL.gpt2_124m_plain(), 12)):
        idx, w = bench.sample_plan(wl)
        assert idx == [0, 1, 2, 3, 4, 5] and w == [layers] * 6      # q, k, v, o, fc, proj of layer 0
        assert sum(w) == wl.n
    wl = WL.llama_3p8b_aurora()
    assert {wl.shapes[i] for i in range(6)} == {(3072, 3072), (1024, 3072), (12288, 3072), (3072, 12288)}
    sw = WL.aurora_shape_sweep()
    idx, w = bench.sample_plan(sw)
    assert [sw.shapes[i] for i in idx] == [(1024, 4096), (4096, 1024), (2048, 2048), (768, 3072)]
    assert w == [32] * 4 and sum(w) == sw.n
    single = WL.single_aurora_256x128()
    assert bench.sample_plan(single) == ([0], [1])


def test_reference_arm_rotates_the_sample_over_steps():
    cmd = CMD[:4] + ["--workload", "single", "--steps", "3", "--warmup", "1"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads(r.stdout.strip().splitlines()[-1])
    cb = d["cpu_baseline"]
    assert d["extrapolated"] is False and cb["timed_matrices"] == 1 and cb["scale"] == 1
    assert cb["sample_wall_s"] > 0 and "in turn" in cb["sample"]
