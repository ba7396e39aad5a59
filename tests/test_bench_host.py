"""Host logic of bench.py (no GPU): the algorithmic flop count against the
figures the workload definitions quote, the workload table, the clock-log
summary that accepts or rejects a timed run, and the reference arm's JSON
line (the fp64 oracle timed on the host cores)."""
import importlib.util
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


bench = _bench()


@pytest.mark.parametrize("name,total", [
    # five-iteration algorithmic totals quoted for the workloads (3 m^2 n + m^3
    # per matrix per iteration, symmetric products counted once)
    ("square1024", 2.15e10),
    ("gpt2_small", 1.14e12),
    ("large_batch", 4.26e13),
])
def test_ns_flops_matches_quoted_totals(name, total):
    shapes = bench.workload_spec(name)["shapes"]
    assert 5 * bench.ns_flops(shapes) == pytest.approx(total, rel=5e-3)


def test_ns_flops_uses_the_short_side():
    assert bench.ns_flops([(4096, 14336)]) == bench.ns_flops([(14336, 4096)])
    # a square matrix: 3 m^3 + m^3
    assert bench.ns_flops([(64, 64)]) == 4 * 64 ** 3


@pytest.mark.parametrize("name,count", [
    ("large_batch", 16), ("large_batch_dimuon", 16), ("large_batch_quarter", 4),
    ("gpt2_small", 72), ("square1024", 1), ("square4096", 1), ("lora_r2", 448), ("lora_r8", 448),
    ("lora_r32", 448), ("vec_w1", 64), ("vec_w32", 64), ("vec_w128", 64), ("toy", 1)])
def test_workload_table(name, count):
    spec = bench.workload_spec(name)
    assert len(spec["shapes"]) == count
    assert spec["desc"]
    assert spec["mdt"] in ("bf16", "fp32")


def test_unknown_workload_exits():
    with pytest.raises(SystemExit):
        bench.workload_spec("no_such_workload")


def _row(sm, util, pcap="Not Active", hw="Not Active", hwt="Not Active", swt="Not Active"):
    return f"2026/12/02 10:00:00.000, {sm}, 1965, 900.0, {util}, 0x0, {hw}, {hwt}, {swt}, {pcap}"


def test_clock_log_busy_samples_only():
    text = "\n".join([_row(1965, 0), _row(1300, 100, pcap="Active"), _row(1310, 99, pcap="Active"),
                      _row(1290, 98), _row(1965, 3)])
    out = bench.parse_clock_log(text)
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1300.0
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_log_reports_slowdowns():
    text = "\n".join([_row(900, 100, hw="Active"), _row(950, 100, hwt="Active", swt="Active")])
    out = bench.parse_clock_log(text)
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_log_without_samples():
    assert bench.parse_clock_log("garbage\n\n")["reasons"] == ["no samples"]
    # all idle: the summary falls back to every sample
    assert bench.parse_clock_log(_row(1965, 0))["samples"] == 1


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "3", "--workload", "square1024"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC
    assert d["unit"] == "matrices/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["value"] == d["cpu_baseline"]["value"] == d["e2e"]["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    # the same workload description, steps and warm-ups as the GPU arm prints
    assert d["config"] == bench.config_of(bench.workload_spec("square1024"), 1)
    assert d["steps"] == 2 and d["warmup"] == 3
    assert d["ms_per_step"] > 0


def test_interleaved_order_samples_every_class():
    shapes = bench.workload_spec("large_batch")["shapes"]
    order = bench.interleaved_order(shapes)
    assert sorted(order) == list(range(len(shapes)))
    first = [shapes[i] for i in order[:3]]
    assert sorted(first) == sorted({(4096, 4096), (4096, 14336), (14336, 4096)})


def test_reference_sample_is_bounded():
    # about 2e12 algorithmic flops per reference step, at least one matrix
    assert bench.reference_budget(bench.workload_spec("large_batch")) == 1
    lora = bench.workload_spec("lora_r8")
    k = bench.reference_budget(lora)
    assert k >= len(lora["shapes"])


def test_l2_policy():
    # small workloads are timed with L2 flushed between steps
    assert bench.l2_flushed(bench.workload_spec("square1024"))
    assert bench.l2_flushed(bench.workload_spec("lora_r2"))
    assert not bench.l2_flushed(bench.workload_spec("large_batch"))
    assert "no flush" in bench.config_of(bench.workload_spec("large_batch"), 1)["l2"]


def test_sharded_line_shape():
    """The --sharded mode's JSON line: strong scaling, the workload's matrices
    per second over the step time, the exchange time beside it."""
    spec = bench.workload_spec("gpt2_small")
    d = bench.sharded_line(spec, 4, 10, 5, 2e-3, 3e-4, [1.0, 1.0, 1.1, 0.9],
                           {"sm_mhz": 1900.0}, 170, slice_elems=1000)
    assert d["exchange_bytes_per_step"] == 2 * 3 * 1000 * 2
    assert d["scaling"] == "strong" and d["mode"] == "sharded"
    assert d["value"] == pytest.approx(72 / 2e-3)
    assert d["ms_per_step"] == pytest.approx(2.0)
    assert d["exchange_ms_per_step"] == pytest.approx(0.3)
    assert d["n_gpus"] == 4 and d["steps"] == 10 and d["warmup"] == 5
    assert "reduce-scatter" in d["config"]["parallelism"]
    assert d["config"]["workload"] == spec["desc"]
    json.dumps(d)


def test_thin_fp64_flops():
    """Per column of a rank-r factor: S_1 and S_2 (conditioned) upper
    triangles and O = T b, two flops per multiply-add; matrices with a short
    side above 32 are not thin."""
    spec = {"shapes": [(8, 100), (100, 8), (64, 64)], "cond": True}
    per_col = 2 * (36 * 2 + 64)
    assert bench.thin_fp64_flops(spec) == 2 * 100 * per_col
    spec["cond"] = False
    assert bench.thin_fp64_flops(spec) == 2 * 100 * 2 * (36 + 64)
    # the LoRA rank-32 batch is bound by fp64 arithmetic in fp32 mode, rank 8 by
    # HBM; in bf16 mode the rank-32 sums run on bf16 tensor cores (no fp64)
    r32, r8 = bench.workload_spec("lora_r32"), bench.workload_spec("lora_r8")
    f64 = 148 * bench.FP64_FMA_PER_SM_CLK * 2 * 1965e6
    assert bench.thin_fp64_flops(r32) / f64 > bench.step_bytes(r32) / 6.5e12
    assert bench.thin_fp64_flops(r8) / f64 < bench.step_bytes(r8) / 6.5e12
    assert bench.thin_fp64_flops(r32, split_r32=True) == 0.0
    assert bench.thin_fp64_flops(r8, split_r32=True) == bench.thin_fp64_flops(r8)
