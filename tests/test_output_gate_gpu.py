"""Parity of gdn2_output_gate (through the C ABI) with the FP64 oracle epilogue:
y = o / sqrt(mean(o^2) + eps) * weight * sigmoid(g) per (token, head) row.
BF16: 2e-2 beyond the output's own BF16 rounding (max |delta| / RMS) and 1e-2
normwise; FP32: 1e-4 (as for the prefill's outputs).
"""
import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import oracle
from conftest import record_margin
from test_parity_gpu import rel, rel_bf16, rel_rms

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_111_b200 as mod
    mod.load_library()
    return mod


def draw(B, T, H, dv, dtype, seed):
    rng = np.random.default_rng(seed)
    o = (rng.standard_normal((B, T, H, dv)) * rng.uniform(0.05, 3.0, (B, T, H, 1))).astype(np.float32)
    gl = (rng.standard_normal((B, T, H, dv)) * 2.0).astype(np.float32)
    w = rng.uniform(0.5, 1.5, dv).astype(np.float32)
    if dtype == "bf16":
        o, gl = gi.round_to_bf16(o), gi.round_to_bf16(gl)
    return o, gl, w


def run(g, o, gl, w, dtype, eps, inplace=False):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    ot = torch.from_numpy(o).cuda().to(tdt)
    gt = torch.from_numpy(gl).cuda().to(tdt)
    wt = torch.from_numpy(w).cuda()
    y = g.gdn2_output_gate(ot, gt, wt, eps, y=ot if inplace else None)
    torch.cuda.synchronize()
    return y.float().cpu().numpy()


def check(name, y, ref, dtype):
    if dtype == "fp32":
        e = rel(y, ref)
        record_margin(name, "y", e, 1e-4)
        assert e <= 1e-4, f"y error {e:.3e}"
    else:
        e, en = rel_bf16(y, ref), rel_rms(y, ref)
        record_margin(name, "y", e, 2e-2)
        assert e <= 2e-2 and en <= 1e-2, f"y error {e:.3e} (normwise {en:.3e})"


@pytest.mark.parametrize("dtype,dv", [("bf16", 128), ("fp32", 128), ("bf16", 64), ("fp32", 64)])
def test_output_gate_matches_oracle(g, dtype, dv):
    o, gl, w = draw(2, 37, 3, dv, dtype, seed=dv)
    y = run(g, o, gl, w, dtype, 1e-6)
    check(f"output gate {dtype} d{dv}", y, oracle.output_gate(o, gl, w, 1e-6), dtype)


def test_output_gate_zero_rows_and_in_place(g):
    o, gl, w = draw(1, 20, 2, 128, "bf16", seed=5)
    o[0, 3] = 0.0                                  # zero rows: y = 0 (eps > 0)
    y = run(g, o, gl, w, "bf16", 1e-5, inplace=True)
    assert np.all(y[0, 3] == 0.0)
    check("output gate zero rows in place", y, oracle.output_gate(o, gl, w, 1e-5), "bf16")


def test_output_gate_full_size(g):
    """The prefill workload's output shape (B 4, T 4096, H 16, d_v 128), every element."""
    o, gl, w = draw(4, 4096, 16, 128, "bf16", seed=9)
    y = run(g, o, gl, w, "bf16", 1e-6)
    check("output gate 4x4096x16", y, oracle.output_gate(o, gl, w, 1e-6), "bf16")
