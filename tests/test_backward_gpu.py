"""Parity of the chunkwise backward (gdn2_chunk_bwd, through the C ABI) with the
FP64 oracle gradient (reverse mode through the token loop, itself pinned by
finite differences in test_oracle_grad.py).

Every gradient tensor is compared element by element.  Error metric as in
test_parity_gpu.py: max |x - ref| / RMS(ref).  Tolerances: FP32 inputs 1e-4 on
every gradient; BF16 q/k/v (gradients dq, dk, dv returned in BF16) 2e-2 beyond
the BF16 rounding of the result and 1e-2 normwise; the FP32 gradients (dalpha,
db, dw, dS0) of BF16 runs 1e-2.

Decay gradient under strong decay.  The chunkwise gradient with respect to a
channel's decay at token j, alpha_j * dL/dalpha_j = dL/d(ln alpha_j), is the sum
over the chunk's tokens t >= j of per-token terms that cancel down to a value of
order alpha_j (every path that crosses token j carries the factor alpha_j).  In
FP32 that sum keeps an absolute error of order eps times the terms, so dalpha_j
itself carries a relative error of order eps / alpha_j -- about 1e-4 relative to
RMS(dalpha) once alpha_j is near 1e-3 -- whereas dL/d(ln alpha) stays accurate to
FP32 rounding.  With alpha down to 1e-3 the test therefore compares
alpha * dalpha (the gradient with respect to ln alpha, which is what a gate
parameterised in log space consumes) at the FP32 tolerance.
"""
import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import oracle
from conftest import record_margin
from test_parity_gpu import rel, rel_bf16, rel_rms, sel_heads

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-4
TOL_BF16 = 2e-2
TOL_BF16_RMS = 1e-2
TOL_BF16_F32 = 1e-2
NAMES = ("dq", "dk", "dv", "dalpha", "db", "dw", "dS0")


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_111_b200 as mod
    mod.load_library()
    return mod


def upstream(x, seed, dst=True):
    """Seeded upstream gradients dO (in the run's dtype) and dST."""
    rng = np.random.default_rng(seed)
    B, T, H, dv, dk = x["B"], x["T"], x["H"], x["dv"], x["dk"]
    dO = rng.standard_normal((B, T, H, dv)).astype(np.float32)
    if x["dtype"] == "bf16":
        dO = gi.round_to_bf16(dO)
    dST = (rng.standard_normal((B, H, dk, dv)) * 0.5).astype(np.float32) if dst else None
    return dO, dST


def run_bwd(g, x, dO, dST, **kw):
    dt = torch.bfloat16 if x["dtype"] == "bf16" else torch.float32
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda().to(dt if n in "qkv" else torch.float32)
         for n in ("q", "k", "v", "alpha", "b", "w")}
    S0 = None if x.get("S0") is None else torch.from_numpy(x["S0"]).cuda()
    dOt = None if dO is None else torch.from_numpy(dO).cuda().to(dt)
    dSTt = None if dST is None else torch.from_numpy(dST).cuda()
    out = g.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S0, dOt, dSTt, **kw)
    torch.cuda.synchronize()
    return {n: out[n].float().cpu().numpy() for n in NAMES}


def check(name, got, ref, dtype, alpha=None):
    """alpha given: dalpha is compared as alpha * dalpha (the gradient with respect to ln alpha)."""
    for n in NAMES:
        a, r = got[n], ref[n]
        if n == "dalpha" and alpha is not None:
            a, r = a * alpha, r * alpha
        if dtype == "fp32":
            e = rel(a, r)
            record_margin(name, n, e, TOL_FP32)
            assert e <= TOL_FP32, f"{n}: error {e:.3e} > {TOL_FP32}"
        elif n in ("dq", "dk", "dv"):
            e, en = rel_bf16(a, r), rel_rms(a, r)
            record_margin(name, n, e, TOL_BF16)
            assert e <= TOL_BF16, f"{n}: error beyond BF16 rounding {e:.3e} > {TOL_BF16}"
            assert en <= TOL_BF16_RMS, f"{n}: normwise error {en:.3e} > {TOL_BF16_RMS}"
        else:
            e = rel(a, r)
            record_margin(name, n, e, TOL_BF16_F32)
            assert e <= TOL_BF16_F32, f"{n}: error {e:.3e} > {TOL_BF16_F32}"


CASES = [
    # dtype, B, T, H, dk, dv, s0
    ("fp32", 2, 150, 2, 64, 64, 0.05),
    ("fp32", 1, 130, 2, 128, 64, 0.05),
    ("fp32", 1, 64, 1, 64, 128, None),
    ("bf16", 2, 200, 2, 128, 128, 0.05),
    ("bf16", 1, 1, 3, 128, 128, 0.05),
    ("bf16", 1, 257, 1, 64, 128, None),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-B{c[1]}T{c[2]}H{c[3]}-d{c[4]}x{c[5]}")
def test_backward_matches_oracle_gradient(g, case):
    dtype, B, T, H, dk, dv, s0 = case
    x = gi.chunk_inputs(B, T, H, dk, dv, dtype=dtype, seed=11 + T, s0_std=s0)
    dO, dST = upstream(x, seed=5 + T)
    got = run_bwd(g, x, dO, dST)
    ref = oracle.gdn2_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], dO, dST)
    check(f"bwd {dtype} B{B}T{T}H{H} d{dk}x{dv}", got, ref, dtype)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_backward_strong_decay(g, dtype):
    """alpha down to 1e-3 in a fifth of the channels: many chunks decay far below 2^-64."""
    x = gi.chunk_inputs(1, 190, 2, 128, 128, dtype=dtype, seed=3, s0_std=0.05)
    rng = np.random.default_rng(4)
    mask = rng.random(x["alpha"].shape) < 0.2
    x["alpha"] = np.where(mask, rng.uniform(1e-3, 0.05, x["alpha"].shape), x["alpha"]).astype(np.float32)
    dO, dST = upstream(x, seed=6)
    got = run_bwd(g, x, dO, dST)
    ref = oracle.gdn2_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], dO, dST)
    check(f"bwd strong decay {dtype}", got, ref, dtype, alpha=x["alpha"].astype(np.float64))


def test_backward_only_final_state_gradient(g):
    """dO = 0 (None): the whole gradient flows from dST back through every chunk."""
    x = gi.chunk_inputs(1, 140, 2, 64, 64, dtype="fp32", seed=8, s0_std=0.05)
    _, dST = upstream(x, seed=9)
    got = run_bwd(g, x, None, dST)
    ref = oracle.gdn2_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], None, dST)
    check("bwd dST only", got, ref, "fp32")


def test_backward_no_tokens(g):
    """T = 0: every token gradient is empty and dS0 = dST."""
    x = gi.chunk_inputs(2, 0, 2, 64, 64, dtype="fp32", seed=1, s0_std=0.05)
    _, dST = upstream(x, seed=2)
    got = run_bwd(g, x, np.zeros((2, 0, 2, 64), np.float32), dST)
    assert got["dq"].shape == (2, 0, 2, 64)
    np.testing.assert_array_equal(got["dS0"], dST)


def test_backward_workspace_reuse_is_bit_identical(g):
    """The workspace's previous contents do not leak into the result."""
    x = gi.chunk_inputs(1, 100, 2, 128, 128, dtype="bf16", seed=12, s0_std=0.05)
    dO, dST = upstream(x, seed=13)
    need = g.gdn2_chunk_bwd_workspace_size(1, 100, 2, 128, 128)
    ws = torch.full((need,), 0x7f, dtype=torch.uint8, device="cuda")
    a = run_bwd(g, x, dO, dST, workspace=ws)
    ws.fill_(0xff)
    b = run_bwd(g, x, dO, dST, workspace=ws)
    for n in NAMES:
        np.testing.assert_array_equal(a[n], b[n])


def test_backward_rejects_small_workspace(g):
    x = gi.chunk_inputs(1, 70, 1, 64, 64, dtype="fp32", seed=0)
    need = g.gdn2_chunk_bwd_workspace_size(1, 70, 1, 64, 64)
    ws = torch.empty((need - 16,), dtype=torch.uint8, device="cuda")
    dO, dST = upstream(x, seed=1)
    with pytest.raises(g.Gdn2Error, match="workspace"):
        run_bwd(g, x, dO, dST, workspace=ws)


def test_backward_full_size_sampled_heads(g):
    """B 4, T 4096, H 16, d 128 BF16 (the prefill workload), one launch over the whole
    batch; two sampled (sequence, head) pairs are recomputed by the oracle in full
    (every token, every gradient of that head)."""
    B, T, H = 4, 4096, 16
    x = gi.chunk_inputs(B, T, H, 128, 128, dtype="bf16", seed=21, s0_std=0.02)
    dO, dST = upstream(x, seed=22)
    got = run_bwd(g, x, dO, dST)
    for n in NAMES:
        assert np.all(np.isfinite(got[n])), n
    for b, h in ((0, 0), (3, 11)):
        s = sel_heads(x, [(b, h)])
        ref = oracle.gdn2_bwd(s["q"], s["k"], s["v"], s["alpha"], s["b"], s["w"], s["S0"],
                              dO[b:b + 1, :, h:h + 1], dST[b:b + 1, h:h + 1])
        part = {n: (got[n][b:b + 1, h:h + 1] if n == "dS0" else got[n][b:b + 1, :, h:h + 1]) for n in NAMES}
        check(f"bwd 4x4096x16 head ({b},{h})", part, ref, "bf16")
