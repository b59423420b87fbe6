"""The bench's JSON line keeps its contract: every key the harness reads, with
values derived from the timings as documented (CPU; synthetic timings)."""
import argparse
import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


class _Clocks:
    def summary(self):
        return {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 10}


def _line(capsys, world=1, ms=0.5, e2e=12.0, dec=0.085):
    args = argparse.Namespace(steps=20, warmup=5, no_cpu_baseline=True, cpu_budget=1.0)
    bench.report(args, world, 0, ms, e2e, 604_000_000, 71_000_000, dec, _Clocks())
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    return json.loads(out[0])


def test_keys_and_types(capsys):
    d = _line(capsys)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "e2e", "roofline", "gpu_launches", "clocks",
              "cpu_baseline", "decode", "long_ragged", "backward"):
        assert k in d, k
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["steps"] == 20 and d["warmup"] == 5 and d["n_gpus"] == 1 and d["gpu_launches"] == 20
    assert "workload" in d["config"]
    for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert k in d["e2e"], k
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in d["roofline"], k
    assert d["roofline"]["bound"] == "hbm" and d["roofline"]["unit"] == "GB/s"
    assert d["clocks"]["sm_mhz"] == 1965.0


def test_values_follow_the_timings(capsys):
    d = _line(capsys, ms=0.5, e2e=12.0)
    P = bench.PREFILL
    tokens = P["B"] * P["T"]
    assert d["value"] == pytest.approx(tokens / 0.5e-3)
    assert d["e2e"]["value"] == pytest.approx(tokens / 12.0e-3)
    algo = bench.prefill_bytes(P["B"], P["T"], P["H"], P["dk"], P["dv"])
    assert algo == 675_282_944                     # 2,560 B per token-head + the FP32 final state
    r = d["roofline"]
    assert r["achieved"] == pytest.approx(algo / 0.5e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])


def test_job_value_scales_with_ranks(capsys):
    one = _line(capsys, world=1, ms=0.5)
    four = _line(capsys, world=4, ms=0.5)
    assert four["value"] == pytest.approx(4 * one["value"])
    assert four["n_gpus"] == 4 and four["config"]["global_batch"] == 4 * bench.PREFILL["B"]


def test_tensor_issued_tf32(capsys):
    d = _line(capsys, ms=0.5)
    t = d["tensor_issued_tf32"]
    # 72 TF32 MMAs of M128 N64 K8 = 4.72 M MACs per CTA and chunk; 128 CTAs x 64 chunks
    assert t["flops_per_launch"] == 2 * 4_718_592 * 64 * 128
    assert t["achieved"] == pytest.approx(t["flops_per_launch"] / 0.5e-3 / 1e12)
    assert t["frac"] == pytest.approx(t["achieved"] / t["peak"])


def test_tensor_algorithmic_against_bf16_peak(capsys):
    """Tensor-pipe utilisation: the method's own FLOPs (each triangle counted once) over
    the launch time, against the dense BF16 peak."""
    d = _line(capsys, ms=0.5)
    t = d["tensor"]
    C, dk, dv = 64, 128, 128
    per_chunk_macs = C * C * dk + 2 * C * dk * dv + C * (C + 1) * dv + C * dk * dv + C ** 3 / 6
    assert per_chunk_macs == pytest.approx(4_246_186.67, rel=1e-9)
    P = bench.PREFILL
    assert t["flops_per_launch"] == pytest.approx(2 * per_chunk_macs * (P["T"] / C) * P["B"] * P["H"])
    assert 3.4e10 < t["flops_per_launch"] < 3.6e10
    assert t["achieved"] == pytest.approx(t["flops_per_launch"] / 0.5e-3 / 1e12)
    assert t["frac"] == pytest.approx(t["achieved"] / t["peak"])
    assert "bf16" in t["peak_source"]


def test_reference_arm_prints_the_same_config():
    assert bench.bench_config(1)["workload"] == bench.bench_config(2)["workload"]
    assert set(bench.bench_config(1)) >= {"workload", "global_batch", "seq_len", "heads", "d_k", "d_v", "dtypes"}


def test_backward_entry(capsys):
    args = argparse.Namespace(steps=20, warmup=5, no_cpu_baseline=True, cpu_budget=1.0)
    bench.report(args, 1, 0, 0.5, 12.0, 1, 1, 0.085, _Clocks(), (float("nan"), float("nan"), 1), 2.0)
    d = json.loads(capsys.readouterr().out.strip())
    bw = d["backward"]
    P = bench.PREFILL
    assert bw["value"] == pytest.approx(P["B"] * P["T"] / 2.0e-3)
    # 4,864 B per token-head (q,k,v,dO bf16 + alpha,b,w fp32 in; dq,dk,dv bf16 + dalpha,db,dw fp32 out)
    assert bench.backward_bytes(1, 1, 1, 128, 128) == 4864 + 128 * 128 * 4
    assert bw["roofline"]["achieved"] == pytest.approx(bench.backward_bytes(4, 4096, 16, 128, 128) / 2.0e-3 / 1e9)
    assert bw["launches_per_call"] == 5


def test_long_ragged_entry(capsys):
    """The long workload reports the segmented call (with its segment count) and the sequential one."""
    args = argparse.Namespace(steps=20, warmup=5, no_cpu_baseline=True, cpu_budget=1.0)
    bench.report(args, 1, 0, 0.5, 12.0, 1, 1, 0.085, _Clocks(), (7.3, 4.9, 3))
    lr = json.loads(capsys.readouterr().out.strip())["long_ragged"]
    assert lr["ms_per_call"] == pytest.approx(4.9) and lr["ms_per_call_sequential"] == pytest.approx(7.3)
    assert lr["segments"] == 3
    assert lr["tokens_per_s"] == pytest.approx(bench.LONG["T"] / 4.9e-3)


def test_logits_entry(capsys):
    args = argparse.Namespace(steps=20, warmup=5, no_cpu_baseline=True, cpu_budget=1.0)
    bench.report(args, 1, 0, 0.5, 12.0, 1, 1, 0.085, _Clocks(), (float("nan"), float("nan"), 1), float("nan"), 0.4)
    d = json.loads(capsys.readouterr().out.strip())
    lg = d["prefill_logits"]
    # six BF16 logit tensors in, BF16 o out: 1,792 B per token-head at d = 128
    assert bench.logits_bytes(1, 1, 1, 128, 128) == 1792 + 128 * 128 * 4
    assert lg["roofline"]["achieved"] == pytest.approx(bench.logits_bytes(4, 4096, 16, 128, 128) / 0.4e-3 / 1e9)
    assert d["backward"]["value"] is None


def test_output_gate_entry(capsys):
    args = argparse.Namespace(steps=20, warmup=5, no_cpu_baseline=True, cpu_budget=1.0)
    bench.report(args, 1, 0, 0.5, 12.0, 1, 1, 0.085, _Clocks(), (float("nan"), float("nan"), 1), float("nan"), float("nan"), 0.04)
    d = json.loads(capsys.readouterr().out.strip())
    og = d["output_gate"]
    # o and g read, y written, BF16: 768 B per token-head at d_v = 128
    assert bench.output_gate_bytes(1, 1, 1, 128) == 768 + 512
    assert og["roofline"]["achieved"] == pytest.approx(bench.output_gate_bytes(4, 4096, 16, 128) / 0.04e-3 / 1e9)
