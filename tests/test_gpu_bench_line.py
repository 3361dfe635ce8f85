"""bench.py prints one JSON line with the fields the measurement contract
names: the metric and its unit, the timing of the steps, the roofline of the
dominant kernel, the end-to-end figure with its copied bytes, the count of
the library's launches and the sampled clocks.  A small case (one layer of
the 3.8B set), run as a child process, in both GEMM modes."""
import json
import os
import subprocess
import sys

import pytest

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def bench_line(*args):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--layers", "1", "--steps", "2", "--warmup", "3",
           "--no-cpu-baseline", *args]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("gemm,bound,kernel", [("bf16", "tensor", "k_gemm_tc"), ("fp32", "alu", "k_gemm_simt")])
def test_bench_line_carries_the_contract_fields(gemm, bound, kernel):
    d = bench_line("--gemm", gemm)
    assert d["unit"] == "steps/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] >= 3
    assert d["value"] > 0 and abs(d["value"] - 1e3 / d["ms_per_step"]) <= 1e-6 * d["value"]
    assert d["config"]["workload"].startswith("llama_3p8b") and d["config"]["matrices"] == 6
    assert d["dtype"] == ("bf16" if gemm == "bf16" else "f32")
    r = d["roofline"]
    assert r["bound"] == bound and r["kernel"] == kernel and r["unit"] == "TFLOP/s"
    assert 0 < r["achieved"] and 0 < r["peak"] and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    # per-launch algorithmic work and launch time, and the launch count of the
    # timed region (every kernel of the library, counted by its tracing)
    assert r["flops_per_launch"] > 0 and r["ms_per_launch"] > 0
    assert d["gpu_launches"] > 0 and d["gpu_launches"] % d["steps"] == 0
    e = d["e2e"]
    assert e["unit"] == "steps/s" and 0 < e["value"]
    # one layer: grads in (bf16) and params out (bf16), 6 matrices
    elems = d["config"]["elements"]
    assert e["h2d_bytes_per_step"] == 2 * elems and e["d2h_bytes_per_step"] == 2 * elems
    c = d["clocks"]
    assert c is not None and c["samples"] >= 1 and c["sm_max_mhz"] >= c["sm_mhz"] > 0
    assert {"ns_gemm_tc" if gemm == "bf16" else "ns_gemm_simt", "prologue", "epilogue"} <= set(d["stages"])
