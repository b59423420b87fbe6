"""Benchmark of the Gated DeltaNet-2 recurrence on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Headline: chunkwise prefill tokens/s on the
4K-token workload B=4, T=4096, H=16, d_k=d_v=128 (BF16 q/k/v, FP32 gates, FP32
state, S0 = 0).  One timed step = one gdn2_chunk_fwd call on that batch (one
kernel launch).  The decode step (batch 256, H=16, d=128, FP32 state, 64
consecutive in-place steps) is timed in the same run and reported under
"decode" as state GB/s; the chunkwise backward (gdn2_chunk_bwd: gradients of
every input of the prefill workload) under "backward" as tokens/s, and the
prefill from BF16 pre-activation logits (gdn2_chunk_fwd_logits) under
"prefill_logits", and the output epilogue (gdn2_output_gate) under
"output_gate".

* value      device time, inputs resident in HBM, CUDA events on the launching
             stream, max over ranks; inputs (675 MB) exceed the 126 MB L2.
* e2e        the same call from pinned HOST buffers: H2D of every input and D2H
             of o and S_T inside the timed region, through the public API.
* roofline   algorithmic bytes per launch / measured launch time, against the
             measured HBM copy bandwidth (MEASURED_PEAKS.json).
* cpu_baseline  the FP64 oracle on this host's cores, on a bounded sample.
* --impl reference  times the oracle alone (the CPU reference arm).

Multi-GPU (torchrun): every rank runs its own replica of the workload (the
(batch, head) recurrences are independent; no data-path collective), so
scaling is weak and value = tokens of all ranks / max time over ranks.
"""
from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import gdn2_inputs as gi  # noqa: E402

PREFILL = gi.PREFILL_4K
DECODE = gi.DECODE_B256
LONG = gi.LONG_RAGGED
BYTES_PER_TOKEN_HEAD = 2560        # q,k,v bf16 (768) + alpha,b,w fp32 (1536) + o bf16 (256)
METRIC = "GDN-2 chunk fwd tokens/s @H16 d128 T4K"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0


def prefill_bytes(B, T, H, dk, dv):
    tok = B * T * H
    return tok * (2 * dk * 2 + dv * 2 + 2 * dk * 4 + dv * 4 + dv * 2) + B * H * dk * dv * 4  # + S_T


def prefill_mma_flops(B, T, H, dk=128, dv=128, C=64):
    """Tensor-core FLOPs one tensor-core prefill launch issues (TF32 MMAs, M = 128, N = 64,
    as issued per CTA = (batch, head, d_v/2 columns) and chunk: Gram [Etil;Qtil]Ktil^T
    2C x C x dk, [Etil;Qtil]S 2C x dv/2 x dk, U = [T;P](R_hi + R_lo) 2 x 2C x dv/2 x C,
    state update Ktil^T(U_hi + U_lo) 2 x dk x dv/2 x C, output [T;P] U_hi 2C x dv/2 x C)."""
    n = dv // 2
    macs = 2 * C * C * dk + 2 * C * n * dk + 2 * (2 * C * n * C) + 2 * (dk * n * C) + 2 * C * n * C
    chunks = -(-T // C)
    return 2 * macs * chunks * 2 * B * H


def prefill_algorithmic_flops(B, T, H, dk=128, dv=128, C=64):
    """FLOPs of the chunkwise method itself, counting each triangle once: per chunk of C
    tokens and head, A and P (C^2 dk together), [Etil;Qtil] S (2 C dk dv), T R and P U
    (C(C+1)/2 dv each), Ktil^T U (C dk dv) and the triangular inversion (C^3 / 6) --
    about 1.33e5 FLOP per token and head at d = 128, 3.5e10 per launch of the 4K workload."""
    macs = C * C * dk + 2 * C * dk * dv + C * (C + 1) * dv + C * dk * dv + C ** 3 / 6
    return 2 * macs * (T / C) * B * H


TF32_PER_BF16 = 1.1 / 2.25       # nominal dense TF32 / BF16 tensor rates on B200


def measured_bf16_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured bf16 dense burst (cuBLAS)"
    return 1590.0, "fallback bf16 dense burst"


def measured_tensor_peak():
    bf, src = measured_bf16_peak()
    return bf * TF32_PER_BF16, src + " x nominal tf32/bf16"


def backward_bytes(B, T, H, dk, dv):
    """Algorithmic HBM bytes of one backward call: q,k,v,dO bf16 and alpha,b,w fp32 read;
    dq,dk,dv bf16 and dalpha,db,dw fp32 written (4,864 B per token-head); the FP32 dS0
    written.  The workspace (chunk-boundary states, T, P, U, dR) is not counted."""
    per = 2 * (2 * dk + dv) + 4 * (2 * dk + dv) + 2 * dv + 2 * (2 * dk + dv) + 4 * (2 * dk + dv)
    return B * T * H * per + B * H * dk * dv * 4


def logits_bytes(B, T, H, dk, dv):
    """Algorithmic HBM bytes of one logits prefill: six BF16 logit tensors read and BF16 o
    written (1,792 B per token-head at d = 128), plus the FP32 final state."""
    return B * T * H * (2 * (4 * dk + 2 * dv) + 2 * dv) + B * H * dk * dv * 4


def output_gate_bytes(B, T, H, dv, es=2):
    """Algorithmic bytes of the output epilogue: o and g read, y written (768 B per
    token-head in BF16 at d_v = 128) and the weight vector."""
    return B * T * H * dv * es * 3 + dv * 4


def decode_bytes(B, H, dk, dv):
    bh = B * H
    return bh * (2 * dk * dv * 4 + (2 * dk + dv) * 2 + (2 * dk + dv) * 4 + dv * 2)


def state_bytes(B, H, dk, dv):
    return 2 * B * H * dk * dv * 4


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x, torch, dist, world, device):
    """The largest of every rank's ``x`` (one all-reduce; every rank calls it
    in the same order).  With one rank, ``x`` itself."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sync_ranks(torch, dist, world):
    """Device idle, then all ranks meet (brackets every timed region)."""
    if torch.cuda.is_available():
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()


def job_tokens_per_s(B, T, world, ms):
    """Whole-job throughput: every rank runs one B x T replica per step, so the
    job processes B*T*world tokens in the slowest rank's time."""
    return B * T * world / (ms / 1e3)


# ----------------------------------------------------------------------------- CPU oracle

def oracle_tokens_per_s(budget_s=12.0, max_heads=None):
    """Time the FP64 oracle on a bounded sample of the prefill workload.

    Sample: every (batch, head) chain of the workload (up to ``max_heads``) over
    the first T_s tokens, T_s chosen from a short calibration so that the timed
    run takes about ``budget_s`` seconds on all host cores.  Returns
    (tokens/s in the workload's unit, threads, description)."""
    import oracle
    B, T, H, dk, dv = PREFILL["B"], PREFILL["T"], PREFILL["H"], PREFILL["dk"], PREFILL["dv"]
    threads = oracle.num_threads()
    heads = B * H if max_heads is None else min(B * H, max_heads)
    calib = gi.chunk_inputs(1, 64, min(heads, threads), dk, dv, dtype="bf16", seed=1)
    t0 = time.perf_counter()
    oracle.gdn2(calib["q"], calib["k"], calib["v"], calib["alpha"], calib["b"], calib["w"])
    per_tok = (time.perf_counter() - t0) / 64           # seconds per token for min(heads, threads) heads in parallel
    waves = -(-heads // threads)
    Ts = int(max(64, min(T, budget_s / max(per_tok * waves, 1e-9))))
    x = gi.chunk_inputs(1, Ts, heads, dk, dv, dtype="bf16", seed=0)
    reps, dt = 0, 0.0
    t0 = time.perf_counter()
    while reps == 0 or dt < budget_s:                # repeat a short sample to fill the budget
        oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"])
        reps += 1
        dt = time.perf_counter() - t0
    token_heads = heads * Ts * reps
    value = token_heads / H / dt                       # tokens of H heads each, per second
    desc = (f"oracle FP64 on {heads} heads x {Ts} tokens (d=128) of the prefill workload"
            f"{f', repeated {reps}x' if reps > 1 else ''}, {dt:.1f} s")
    return value, threads, desc, dt


def oracle_decode_state_gbs(budget_s=4.0):
    """The FP64 oracle's decode step on a bounded sample of the decode workload: as many
    of its (batch, head) states as fill ``budget_s`` of repeated steps, reported in the
    decode metric's unit (GB of FP32 state read and written per second)."""
    import oracle
    D = DECODE
    threads = oracle.num_threads()
    heads = max(threads, 16)
    x = gi.decode_inputs(1, 1, heads, D["dk"], D["dv"], dtype="bf16", seed=3, s0_std=0.02)
    S = x["S0"].astype(np.float64)
    args = [x[n][0] for n in ("q", "k", "v", "alpha", "b", "w")]
    reps, dt = 0, 0.0
    t0 = time.perf_counter()
    while reps == 0 or dt < budget_s:
        _, S = oracle.gdn2_step(*args, S)
        reps += 1
        dt = time.perf_counter() - t0
    gbs = state_bytes(1, heads, D["dk"], D["dv"]) * reps / dt / 1e9
    return gbs, threads, f"oracle FP64 decode step on {heads} heads (d=128), {reps} steps, {dt:.1f} s"


def oracle_long_tokens_per_s(budget_s=4.0):
    """The FP64 oracle on a bounded sample of the long ragged workload (its 16 heads over
    the first tokens, with S0), in tokens of H heads per second."""
    import oracle
    L = LONG
    threads = oracle.num_threads()
    Ts = 256
    x = gi.chunk_inputs(1, Ts, L["H"], L["dk"], L["dv"], dtype="bf16", seed=0, s0_std=0.02)
    reps, dt = 0, 0.0
    t0 = time.perf_counter()
    while reps == 0 or dt < budget_s:
        oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
        reps += 1
        dt = time.perf_counter() - t0
    return Ts * reps / dt, threads, f"oracle FP64 on the 16 heads x {Ts} tokens, {reps}x, {dt:.1f} s"


def oracle_backward_tokens_per_s(budget_s=4.0, Ts=256):
    """The FP64 oracle gradient on a bounded sample of the prefill workload (its 16 heads
    over the first ``Ts`` tokens, with upstream gradients dO and dST), in tokens of H heads
    per second."""
    import oracle
    P = PREFILL
    threads = oracle.num_threads()
    x = gi.chunk_inputs(1, Ts, P["H"], P["dk"], P["dv"], dtype="bf16", seed=0)
    rng = np.random.default_rng(1)
    dO = gi.round_to_bf16(rng.standard_normal((1, Ts, P["H"], P["dv"])).astype(np.float32))
    reps, dt = 0, 0.0
    t0 = time.perf_counter()
    while reps == 0 or dt < budget_s:
        oracle.gdn2_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], None, dO)
        reps += 1
        dt = time.perf_counter() - t0
    return Ts * reps / dt, threads, f"oracle FP64 gradient on the 16 heads x {Ts} tokens, {reps}x, {dt:.1f} s"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is None:
            self.out = ""
            return
        self.proc.terminate()
        try:
            self.out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.out, _ = self.proc.communicate()

    def summary(self):
        rows = [r for r in csv.reader(io.StringIO(getattr(self, "out", ""))) if len(r) >= 9]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}

        def num(s):
            try:
                return float(s.strip().split()[0])
            except (ValueError, IndexError):
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- GPU arm

def device_inputs(torch, x, dev):
    out = {}
    for n in ("q", "k", "v", "alpha", "b", "w"):
        t = torch.from_numpy(np.ascontiguousarray(x[n]))
        out[n] = t.to(dev).to(torch.bfloat16 if n in ("q", "k", "v") else torch.float32)
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist
    import gated_delta_rule_111_b200 as g

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", device_id=dev, timeout=timedelta(seconds=300))
    g.load_library(rebuild_if_stale=(world == 1))
    stream = torch.cuda.current_stream(dev)

    B, T, H, dk, dv = (PREFILL[n] for n in ("B", "T", "H", "dk", "dv"))
    ms_step = e2e_ms = dec_ms = float("nan")
    h2d = d2h = 0
    clk = None
    if args.workload in ("all", "prefill"):
        ms_step, e2e_ms, h2d, d2h, clk = run_prefill(args, torch, dist, g, world, rank, dev, stream)
    if args.workload in ("all", "decode"):
        dec_ms = run_decode(args, torch, dist, g, world, rank, dev, stream)
    long_ms = long_seg_ms = float("nan")
    long_segments = 1
    if args.workload in ("all", "long"):
        long_ms, long_seg_ms, long_segments = run_long(args, torch, dist, g, world, rank, dev, stream)
    bwd_ms = float("nan")
    if args.workload in ("all", "backward"):
        bwd_ms = run_backward(args, torch, dist, g, world, rank, dev, stream)
    lg_ms = float("nan")
    if args.workload in ("all", "logits"):
        lg_ms = run_prefill_logits(args, torch, dist, g, world, rank, dev, stream)
    og_ms = float("nan")
    if args.workload in ("all", "output_gate"):
        og_ms = run_output_gate(args, torch, dist, g, world, rank, dev, stream)
    report(args, world, rank, ms_step, e2e_ms, h2d, d2h, dec_ms, clk, (long_ms, long_seg_ms, long_segments), bwd_ms,
           lg_ms, og_ms)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_prefill(args, torch, dist, g, world, rank, dev, stream):
    """Device-timed prefill steps and the end-to-end variant; returns timings."""
    B, T, H, dk, dv = (PREFILL[n] for n in ("B", "T", "H", "dk", "dv"))
    x = gi.chunk_inputs(**PREFILL, seed=rank)
    d = device_inputs(torch, x, dev)
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)

    def step():
        g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], None, o=o, S_T=ST, stream=stream)

    for _ in range(args.warmup):
        step()
    sync_ranks(torch, dist, world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # nvidia-smi samples every 100 ms: keep the GPU busy with the same step for
    # about a second before the timed region so the samples see it under load.
    t_est = time.perf_counter()
    step()
    torch.cuda.synchronize()
    per = max(time.perf_counter() - t_est, 1e-5)
    with ClockSampler(dev.index) as clk:
        for _ in range(int(min(4000, 1.2 / per))):
            step()
        sync_ranks(torch, dist, world)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        sync_ranks(torch, dist, world)
    ms_total = max_over_ranks(ev0.elapsed_time(ev1), torch, dist, world, dev)
    ms_step = ms_total / args.steps

    # ---- e2e: pinned host buffers, copies inside the timed region
    host = {n: d[n].cpu().pin_memory() for n in d}
    o_h = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    S_h = torch.empty(ST.shape, dtype=ST.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_h.numel() * o_h.element_size() + S_h.numel() * S_h.element_size()

    work = dict(d, o=o, S_T=ST)

    def e2e_step():     # inputs streamed in per sequence, each sequence's outputs streamed back
        g.gdn2_chunk_fwd_from_host(*(host[n] for n in ("q", "k", "v", "alpha", "b", "w")), None, device=dev,
                                   work=work, o=o_h, S_T=S_h, stream=stream)

    for _ in range(2):
        e2e_step()
    sync_ranks(torch, dist, world)
    e2e_steps = max(2, min(args.steps, 5))
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    sync_ranks(torch, dist, world)
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1) / e2e_steps, torch, dist, world, dev)
    del host, o_h, S_h, d, o, ST
    torch.cuda.empty_cache()
    return ms_step, e2e_ms, h2d, d2h, clk


def run_decode(args, torch, dist, g, world, rank, dev, stream):
    """64 consecutive in-place decode steps timed as one region; returns ms per step."""
    dv = DECODE["dv"]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    xd = gi.decode_inputs(**DECODE, seed=rank)
    steps_d = DECODE["steps"]
    Bd, Hd = DECODE["B"], DECODE["H"]
    dd = device_inputs(torch, xd, dev)
    S0d = torch.from_numpy(xd["S0"]).to(dev)
    Sd = S0d.clone()
    od = torch.empty((Bd, Hd, dv), dtype=torch.bfloat16, device=dev)
    views = [[dd[n][s] for n in ("q", "k", "v", "alpha", "b", "w")] for s in range(steps_d)]

    def decode_run():
        for s in range(steps_d):
            g.gdn2_recurrent_step(*views[s], Sd, o=od, stream=stream)

    for _ in range(max(args.warmup, 1)):
        decode_run()
    sync_ranks(torch, dist, world)
    reps = 3
    ev0.record(stream)
    for _ in range(reps):
        decode_run()
    ev1.record(stream)
    sync_ranks(torch, dist, world)
    dec_ms = max_over_ranks(ev0.elapsed_time(ev1) / (reps * steps_d), torch, dist, world, dev)
    del dd, S0d, Sd, od, views
    torch.cuda.empty_cache()
    return dec_ms


def run_long(args, torch, dist, g, world, rank, dev, stream):
    """The long ragged workload (B=1, T=65,573, H=16, S0 != 0): one sequential prefill call
    (32 CTAs walk 1,025 chunks each) and one segment-parallel call with the automatic segment
    count.  Returns (ms per sequential call, ms per segmented call, segments)."""
    x = gi.chunk_inputs(**LONG, seed=rank)
    d = device_inputs(torch, x, dev)
    S0 = torch.from_numpy(x["S0"]).to(dev)
    del x
    B, T, H, dv = LONG["B"], LONG["T"], LONG["H"], LONG["dv"]
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    ST = torch.empty_like(S0)

    segments = g.gdn2_chunk_fwd_segments(B, T, H, LONG["dk"], dv, 0)
    ws = torch.empty((max(g.gdn2_chunk_fwd_segmented_workspace_size(B, T, H, LONG["dk"], dv, 0), 1),),
                     dtype=torch.uint8, device=dev)

    def call():
        g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S0, o=o, S_T=ST, stream=stream)

    def call_seg():
        g.gdn2_chunk_fwd_segmented(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S0, segments=0,
                                   workspace=ws, o=o, S_T=ST, stream=stream)

    out = []
    for fn in (call, call_seg):
        fn()
        sync_ranks(torch, dist, world)
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 3
        ev0.record(stream)
        for _ in range(reps):
            fn()
        ev1.record(stream)
        sync_ranks(torch, dist, world)
        out.append(max_over_ranks(ev0.elapsed_time(ev1) / reps, torch, dist, world, dev))
    del d, S0, o, ST, ws
    torch.cuda.empty_cache()
    return out[0], out[1], segments


def run_backward(args, torch, dist, g, world, rank, dev, stream):
    """The chunkwise backward (gdn2_chunk_bwd) on the prefill workload with a BF16 upstream
    gradient dO and dST = 0, workspace preallocated; returns ms per call (three launches)."""
    B, T, H, dk, dv = (PREFILL[n] for n in ("B", "T", "H", "dk", "dv"))
    x = gi.chunk_inputs(**PREFILL, seed=rank)
    d = device_inputs(torch, x, dev)
    del x
    gen = torch.Generator(device=dev)
    gen.manual_seed(100 + rank)
    dO = torch.randn((B, T, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    ws = torch.empty(g.gdn2_chunk_bwd_workspace_size(B, T, H, dk, dv), dtype=torch.uint8, device=dev)
    out = {"dq": torch.empty_like(d["q"]), "dk": torch.empty_like(d["k"]), "dv": torch.empty_like(d["v"]),
           "dalpha": torch.empty_like(d["alpha"]), "db": torch.empty_like(d["b"]), "dw": torch.empty_like(d["w"]),
           "dS0": torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)}

    def call():
        g.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], None, dO, None, workspace=ws,
                         out=out, stream=stream)

    for _ in range(max(args.warmup, 3)):
        call()
    sync_ranks(torch, dist, world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(3, min(args.steps, 10))
    ev0.record(stream)
    for _ in range(reps):
        call()
    ev1.record(stream)
    sync_ranks(torch, dist, world)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / reps, torch, dist, world, dev)
    del d, dO, ws, out
    torch.cuda.empty_cache()
    return ms


def run_prefill_logits(args, torch, dist, g, world, rank, dev, stream):
    """gdn2_chunk_fwd_logits on the prefill workload (BF16 logits, activations and gates
    inside the kernel); returns ms per call."""
    B, T, H, dk, dv = (PREFILL[n] for n in ("B", "T", "H", "dk", "dv"))
    x = gi.logit_inputs(B, T, H, dk, dv, seed=rank)
    d = {n: torch.from_numpy(x[n]).to(dev).to(torch.bfloat16) for n in ("xq", "xk", "xv", "xa", "xb", "xw")}
    del x
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    ST = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)

    def call():
        g.gdn2_chunk_fwd_logits(d["xq"], d["xk"], d["xv"], d["xa"], d["xb"], d["xw"], None, o=o, S_T=ST,
                                stream=stream)

    for _ in range(max(args.warmup, 3)):
        call()
    sync_ranks(torch, dist, world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(3, args.steps)
    ev0.record(stream)
    for _ in range(reps):
        call()
    ev1.record(stream)
    sync_ranks(torch, dist, world)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / reps, torch, dist, world, dev)
    del d, o, ST
    torch.cuda.empty_cache()
    return ms


def run_output_gate(args, torch, dist, g, world, rank, dev, stream):
    """gdn2_output_gate on the prefill workload's output shape (BF16 o and gate logits);
    returns ms per call."""
    B, T, H, dv = (PREFILL[n] for n in ("B", "T", "H", "dv"))
    gen = torch.Generator(device=dev)
    gen.manual_seed(200 + rank)
    o = torch.randn((B, T, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    gl = torch.randn((B, T, H, dv), generator=gen, device=dev).to(torch.bfloat16)
    w = torch.rand((dv,), generator=gen, device=dev) + 0.5
    y = torch.empty_like(o)

    def call():
        g.gdn2_output_gate(o, gl, w, 1e-6, y=y, stream=stream)

    for _ in range(max(args.warmup, 3)):
        call()
    sync_ranks(torch, dist, world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = max(10, args.steps)
    ev0.record(stream)
    for _ in range(reps):
        call()
    ev1.record(stream)
    sync_ranks(torch, dist, world)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / reps, torch, dist, world, dev)
    del o, gl, w, y
    torch.cuda.empty_cache()
    return ms


def bench_config(world):
    """The workload description both arms print (the reference arm times the same workload)."""
    B, T, H, dk, dv = (PREFILL[n] for n in ("B", "T", "H", "dk", "dv"))
    return {"workload": "GDN-2 chunkwise prefill B=4 T=4096 H=16 d_k=d_v=128 chunk=64, S0=0",
            "global_batch": B * world, "seq_len": T, "heads": H, "d_k": dk, "d_v": dv,
            "dtypes": "q/k/v/o bf16, alpha/b/w fp32, state fp32, fp32 accumulation",
            "l2": "inputs (675 MB per call) larger than the 126 MB L2; no flush",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


def _num(x):
    return None if x != x else x      # NaN (workload not run) -> null


def report(args, world, rank, ms_step, e2e_ms, h2d, d2h, dec_ms, clk, long=(float("nan"), float("nan"), 1),
           bwd_ms=float("nan"), lg_ms=float("nan"), og_ms=float("nan")):
    """long: (ms per sequential call, ms per segmented call, segments) of the long ragged workload."""
    long_ms, long_seg_ms, long_segments = long
    B, T, H, dk, dv = (PREFILL[n] for n in ("B", "T", "H", "dk", "dv"))
    Bd, Hd = DECODE["B"], DECODE["H"]
    steps_d = DECODE["steps"]
    reps = 3
    value = job_tokens_per_s(B, T, world, ms_step)
    hbm, hbm_src = measured_peaks()
    pre_bytes = prefill_bytes(B, T, H, dk, dv)
    pre_gbs = pre_bytes / (ms_step / 1e3) / 1e9
    dec_bytes = decode_bytes(Bd, Hd, dk, dv)
    dec_gbs = dec_bytes / (dec_ms / 1e3) / 1e9
    st_gbs = state_bytes(Bd, Hd, dk, dv) / (dec_ms / 1e3) / 1e9
    traffic = load_traffic()
    tflops = prefill_mma_flops(B, T, H, dk, dv) / (ms_step / 1e3) / 1e12
    tpeak, tsrc = measured_tensor_peak()
    algo_flops = prefill_algorithmic_flops(B, T, H, dk, dv)
    atflops = algo_flops / (ms_step / 1e3) / 1e12
    bpeak, bsrc = measured_bf16_peak()

    og_bytes = output_gate_bytes(B, T, H, dv)
    og_gbs = og_bytes / (og_ms / 1e3) / 1e9
    lg_bytes = logits_bytes(B, T, H, dk, dv)
    lg_gbs = lg_bytes / (lg_ms / 1e3) / 1e9
    bwd_bytes = backward_bytes(B, T, H, dk, dv)
    bwd_gbs = bwd_bytes / (bwd_ms / 1e3) / 1e9
    cpu = dec_cpu = long_cpu = bwd_cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, desc, _ = oracle_tokens_per_s(budget_s=args.cpu_budget)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
        v, cores, desc = oracle_decode_state_gbs()
        dec_cpu = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc}
        v, cores, desc = oracle_long_tokens_per_s()
        long_cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
        if bwd_ms == bwd_ms:
            v, cores, desc = oracle_backward_tokens_per_s()
            bwd_cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": _num(value), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": _num(ms_step), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; recipe in gdn2_inputs.py)",
            "config": bench_config(world),
            "e2e": {"value": _num(job_tokens_per_s(B, T, world, e2e_ms)), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": _num(e2e_ms),
                    "api": "gdn2_chunk_fwd_from_host: pinned host inputs streamed in per sequence, each "
                           "sequence's prefill as its inputs arrive, outputs streamed back"},
            "roofline": {"bound": "hbm", "achieved": _num(pre_gbs), "peak": hbm, "unit": "GB/s",
                         "frac": _num(pre_gbs / hbm), "traffic": traffic.get("gdn2_chunk"),
                         "kernel": "gdn2 chunkwise prefill", "algorithmic_bytes_per_launch": pre_bytes,
                         "peak_source": f"{hbm_src} HBM copy bandwidth", "frac_of_8TBps": _num(pre_gbs / 8000.0)},
            "tensor": {"achieved": _num(atflops), "peak": bpeak, "unit": "TFLOP/s", "frac": _num(atflops / bpeak),
                       "flops_per_launch": algo_flops, "peak_source": bsrc,
                       "note": "algorithmic FLOPs of the chunkwise method over the measured launch time, "
                               "against the dense BF16 peak"},
            "tensor_issued_tf32": {"achieved": _num(tflops), "peak": tpeak, "unit": "TFLOP/s",
                                   "frac": _num(tflops / tpeak), "flops_per_launch": prefill_mma_flops(B, T, H, dk, dv),
                                   "peak_source": tsrc,
                                   "note": "TF32 MMA FLOPs as issued (split operands and the per-CTA key side counted)"},
            "decode": {"metric": "GDN-2 decode state GB/s @B256 H16 d128", "value": _num(st_gbs), "unit": "GB/s",
                       "us_per_step": _num(dec_ms * 1e3), "steps": steps_d * reps,
                       "roofline": {"bound": "hbm", "achieved": _num(dec_gbs), "peak": hbm, "unit": "GB/s",
                                    "frac": _num(dec_gbs / hbm), "traffic": traffic.get("gdn2_decode"),
                                    "algorithmic_bytes_per_launch": dec_bytes,
                                    "frac_of_8TBps": _num(dec_gbs / 8000.0)},
                       "cpu_baseline": dec_cpu},
            "long_ragged": {"workload": "B=1 T=65573 H=16 d_k=d_v=128, S0 != 0 (ragged last chunk)",
                            "ms_per_call": _num(long_seg_ms),
                            "tokens_per_s": _num(LONG["B"] * LONG["T"] * world / (long_seg_ms / 1e3)),
                            "segments": long_segments,
                            "ms_per_call_sequential": _num(long_ms),
                            "note": "gdn2_chunk_fwd_segmented with the automatic segment count (three passes "
                                    "over 4 (P-1) + 2 P CTAs per head); the sequential call has 32 CTAs walk "
                                    "1,025 chunks each; reported, no target",
                            "cpu_baseline": long_cpu},
            "backward": {"metric": "GDN-2 chunk bwd tokens/s @H16 d128 T4K", "unit": "tokens/s",
                         "value": _num(job_tokens_per_s(B, T, world, bwd_ms)), "ms_per_call": _num(bwd_ms),
                         "workload": "gradients of every input of the prefill workload (BF16 dO, dST = 0)",
                         "launches_per_call": 5,
                         "roofline": {"bound": "hbm", "achieved": _num(bwd_gbs), "peak": hbm, "unit": "GB/s",
                                      "frac": _num(bwd_gbs / hbm), "traffic": traffic.get("gdn2_chunk_bwd"),
                                      "algorithmic_bytes_per_launch": bwd_bytes,
                                      "note": "whole call (prep + state + grad launches) against the "
                                              "algorithmic bytes; workspace traffic not counted"},
                         "cpu_baseline": bwd_cpu},
            "prefill_logits": {"metric": "GDN-2 chunk fwd from BF16 logits tokens/s @H16 d128 T4K",
                               "unit": "tokens/s", "value": _num(job_tokens_per_s(B, T, world, lg_ms)),
                               "ms_per_call": _num(lg_ms),
                               "workload": "the prefill workload from BF16 pre-activation logits (SiLU, L2 norm, "
                                           "sigmoid gates and the decay inside the kernel)",
                               "roofline": {"bound": "hbm", "achieved": _num(lg_gbs), "peak": hbm, "unit": "GB/s",
                                            "frac": _num(lg_gbs / hbm), "traffic": traffic.get("gdn2_chunk_logits"),
                                            "algorithmic_bytes_per_launch": lg_bytes}},
            "output_gate": {"metric": "GDN-2 output epilogue (RMS norm + sigmoid gate) tokens/s @H16 d128",
                            "unit": "tokens/s", "value": _num(job_tokens_per_s(B, T, world, og_ms)),
                            "us_per_call": _num(og_ms * 1e3),
                            "roofline": {"bound": "hbm", "achieved": _num(og_gbs), "peak": hbm, "unit": "GB/s",
                                         "frac": _num(og_gbs / hbm), "traffic": traffic.get("gdn2_output_gate"),
                                         "algorithmic_bytes_per_launch": og_bytes}},
            "gpu_launches": args.steps,
            "clocks": clk.summary() if clk is not None else None,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)


def load_traffic():
    """Per-launch DRAM traffic from the committed ncu summary (profiles/traffic.json),
    or None for a kernel whose sources changed since that capture."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return {}
    try:
        with open(path) as f:
            data = json.load(f)
        out = {}
        for name, rec in data.items():
            m = hashlib.sha256()
            for src in rec["sources"]:
                with open(os.path.join(ROOT, src), "rb") as f:
                    m.update(f.read())
            out[name] = rec["bytes_per_launch"] if m.hexdigest()[:16] == rec["sources_sha256_16"] else None
        return out
    except (OSError, KeyError, ValueError):
        return {}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    budget = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_tokens_per_s(budget_s=budget / 4)
    vals, descs, secs = [], [], []
    for _ in range(args.steps):
        v, cores, desc, dt = oracle_tokens_per_s(budget_s=budget)
        vals.append(v)
        descs.append(desc)
        secs.append(dt)
    value = statistics.median(vals)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": statistics.median(secs) * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": bench_config(world),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": descs[-1]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["all", "prefill", "decode", "long", "backward", "logits", "output_gate"], default="all",
                    help="run only one workload's measurement (for profiling one kernel)")
    args = ap.parse_args()
    if args.impl == "ours":
        args.warmup = max(3, args.warmup)       # at least 3 untimed warm-up steps
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
