"""Run one prefill, decode, backward or logits-prefill case a few times on seeded inputs, for profilers.

    python -m gated_delta_rule_111_b200.profile_case prefill --B 2 --T 4096 --H 16 --calls 3
    python -m gated_delta_rule_111_b200.profile_case decode --B 64 --H 16 --calls 3
    python -m gated_delta_rule_111_b200.profile_case backward --B 1 --T 4096 --H 16 --calls 2
    python -m gated_delta_rule_111_b200.profile_case logits --B 2 --T 4096 --H 16 --calls 3

Inputs come from ``gdn2_inputs`` (same recipe as the tests and ``bench.py``), are moved to the GPU
once, and every call goes through the C ABI.  Nothing is checked or timed here: this exists so that
``ncu`` can capture a chosen number of launches of a smaller case of the same kernels.
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import gdn2_inputs as gi  # noqa: E402

from . import (gdn2_chunk_bwd, gdn2_chunk_bwd_workspace_size, gdn2_chunk_fwd, gdn2_chunk_fwd_logits,  # noqa: E402
               gdn2_recurrent_step)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("mode", choices=["prefill", "decode", "backward", "logits"])
    ap.add_argument("--B", type=int, default=2)
    ap.add_argument("--T", type=int, default=4096)
    ap.add_argument("--H", type=int, default=16)
    ap.add_argument("--d", type=int, default=128)
    ap.add_argument("--dtype", choices=["bf16", "fp32"], default="bf16")
    ap.add_argument("--calls", type=int, default=3)
    a = ap.parse_args(argv)
    tdt = torch.bfloat16 if a.dtype == "bf16" else torch.float32
    dev = torch.device("cuda:0")
    if a.mode == "logits":
        x = gi.logit_inputs(a.B, a.T, a.H, a.d, a.d, seed=0)
        lg = {n: torch.from_numpy(x[n]).to(dev).to(torch.bfloat16) for n in ("xq", "xk", "xv", "xa", "xb", "xw")}
        o = torch.empty(a.B, a.T, a.H, a.d, dtype=torch.bfloat16, device=dev)
        S_T = torch.empty(a.B, a.H, a.d, a.d, dtype=torch.float32, device=dev)
        for _ in range(a.calls):
            gdn2_chunk_fwd_logits(lg["xq"], lg["xk"], lg["xv"], lg["xa"], lg["xb"], lg["xw"], o=o, S_T=S_T)
        torch.cuda.synchronize()
        print(f"logits B={a.B} T={a.T} H={a.H} d={a.d}: {a.calls} calls done")
        return
    if a.mode in ("prefill", "backward"):
        x = gi.chunk_inputs(a.B, a.T, a.H, a.d, a.d, dtype=a.dtype, seed=0)
    else:
        x = gi.decode_inputs(1, a.B, a.H, a.d, a.d, dtype=a.dtype, seed=0)
    g = {n: torch.from_numpy(x[n]).to(dev) for n in ("q", "k", "v", "alpha", "b", "w")}
    for n in ("q", "k", "v"):
        g[n] = g[n].to(tdt)
    if a.mode == "prefill":
        o = torch.empty(a.B, a.T, a.H, a.d, dtype=tdt, device=dev)
        S_T = torch.empty(a.B, a.H, a.d, a.d, dtype=torch.float32, device=dev)
        for _ in range(a.calls):
            gdn2_chunk_fwd(g["q"], g["k"], g["v"], g["alpha"], g["b"], g["w"], o=o, S_T=S_T)
    elif a.mode == "backward":
        gen = torch.Generator(device=dev)
        gen.manual_seed(1)
        dO = torch.randn(a.B, a.T, a.H, a.d, generator=gen, device=dev).to(tdt)
        ws = torch.empty(gdn2_chunk_bwd_workspace_size(a.B, a.T, a.H, a.d, a.d), dtype=torch.uint8, device=dev)
        for _ in range(a.calls):
            gdn2_chunk_bwd(g["q"], g["k"], g["v"], g["alpha"], g["b"], g["w"], None, dO, None, workspace=ws)
    else:
        S = torch.from_numpy(x["S0"]).to(dev)
        q, k, v, al, b, w = (g[n][0] for n in ("q", "k", "v", "alpha", "b", "w"))
        o = torch.empty(a.B, a.H, a.d, dtype=tdt, device=dev)
        for _ in range(a.calls):
            gdn2_recurrent_step(q, k, v, al, b, w, S, o=o)
    torch.cuda.synchronize()
    print(f"{a.mode} B={a.B} T={a.T} H={a.H} d={a.d} {a.dtype}: {a.calls} calls done")


if __name__ == "__main__":
    main()
