"""The benchmark's JSON line on a GPU: one short run per kind of workload
(tensor-core products, thin factors, the single-launch cluster kernel, the
sharded mode) and the reference arm, each checked for the keys and the
sanity of the values the line promises."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")]

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=600):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         cwd=ROOT, capture_output=True, text=True, timeout=timeout)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


@pytest.mark.parametrize("workload,bound", [("square1024", "tensor"), ("lora_r8", "hbm"),
                                            ("lora_r32", "hbm"), ("toy", "hbm")])
def test_bench_line(workload, bound):
    d = run_bench("--workload", workload, "--steps", "3", "--warmup", "3", "--no-cpu-baseline")
    assert d["metric"] and d["unit"] == "matrices/s" and d["higher_is_better"] is True
    assert d["n_gpus"] == 1 and d["steps"] == 3 and d["warmup"] == 3
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"]
    r = d["roofline"]
    assert r["bound"] == bound and r["achieved"] > 0 and r["peak"] > 0
    assert 0 < r["frac"] < 2 and r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] == 4
    assert d["gpu_launches"] >= 3
    assert d["clocks"]["sm_max_mhz"] > 0


def test_sharded_line_on_one_rank():
    d = run_bench("--sharded", "--workload", "gpt2_small", "--steps", "3", "--warmup", "3",
                  "--no-cpu-baseline")
    assert d["mode"] == "sharded" and d["scaling"] == "strong" and d["n_gpus"] == 1
    assert d["value"] > 0 and d["exchange_bytes_per_step"] == 0


def test_reference_line():
    d = run_bench("--impl", "reference", "--workload", "toy", "--steps", "3", "--warmup", "3")
    assert d["impl"] == "reference" and d["value"] > 0 and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["value"] == d["value"]
