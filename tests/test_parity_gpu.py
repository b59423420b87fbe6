"""Parity of the CUDA library (through its C ABI) with the FP64 oracle.

Error metric: max |x_gpu - x_ref| / RMS(x_ref) over the compared tensor.
Tolerances: FP32 inputs 1e-4 (o and S_T); BF16 q/k/v with FP32 gates and
accumulation: o 2e-2, S_T 1e-2.

A BF16 output o cannot be closer to the exact value than its own rounding:
half a BF16 ulp is up to 2^-8 of |o|, and on these workloads max|o| reaches
15-20 x RMS(o), so rounding the exact FP64 result to BF16 alone gives
max|delta|/RMS of 0.035-0.048.  For BF16 outputs the 2e-2 bound therefore
applies to the error beyond that rounding: each element's |delta| is reduced by
half a BF16 ulp at its magnitude before the max is taken (``rel_bf16``).  The
normwise error RMS(delta)/RMS(ref) is checked as well (<= 1e-2).

At full workload sizes the oracle recomputes a sample of (batch, head) pairs --
every head is an independent recurrence, so a sampled head is compared element
by element over all tokens.
"""
import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import oracle
from conftest import record_margin

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-4
TOL_BF16_O = 2e-2
TOL_BF16_S = 1e-2


def rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.max(np.abs(x - ref)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30))


def half_ulp_bf16(a):
    """Half a BF16 ulp at magnitude |a| (8-bit significand): 2^(floor(log2|a|) - 8)."""
    a = np.abs(a)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8.0), 0.0)


def rel_bf16(x, ref, roundings=1):
    """max(|x - ref| - half BF16 ulp, 0) / RMS(ref): error beyond the output's own rounding.

    ``roundings=2`` when both sides are BF16 results (each carries its own rounding)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    slack = roundings * half_ulp_bf16(np.maximum(np.abs(ref), np.abs(x)))
    excess = np.maximum(np.abs(x - ref) - slack, 0.0)
    return float(np.max(excess) / max(np.sqrt(np.mean(ref ** 2)), 1e-30))


def rel_rms(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.sqrt(np.mean((x - ref) ** 2)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30))


TOL_BF16_O_RMS = 1e-2


def _test_name():
    import os
    return os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0].split("::")[-1]


def check_o(x, ref, dtype):
    if dtype == "fp32":
        e = rel(x, ref)
        record_margin(_test_name(), "o", e, TOL_FP32)
        assert e <= TOL_FP32, f"o error {e:.3e} > {TOL_FP32}"
    else:
        e, en = rel_bf16(x, ref), rel_rms(x, ref)
        record_margin(_test_name(), "o", e, TOL_BF16_O)
        record_margin(_test_name(), "o (rms)", en, TOL_BF16_O_RMS)
        assert e <= TOL_BF16_O, f"o error beyond BF16 rounding {e:.3e} > {TOL_BF16_O}"
        assert en <= TOL_BF16_O_RMS, f"o normwise error {en:.3e} > {TOL_BF16_O_RMS}"
    return e


def check_s(x, ref, tol):
    e = rel(x, ref)
    record_margin(_test_name(), "S_T", e, tol)
    assert e <= tol, f"S_T error {e:.3e} > {tol}"
    return e


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_111_b200 as mod
    mod.load_library()
    return mod


def to_dev(x, keys=("q", "k", "v", "alpha", "b", "w")):
    dt = torch.bfloat16 if x["dtype"] == "bf16" else torch.float32
    out = {}
    for n in keys:
        t = torch.from_numpy(np.ascontiguousarray(x[n]))
        out[n] = t.to("cuda").to(dt if n in ("q", "k", "v") else torch.float32)
    out["S0"] = None if x.get("S0") is None else torch.from_numpy(x["S0"]).cuda()
    return out


def run_chunk(g, x, **kw):
    d = to_dev(x)
    o, ST = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], d["S0"], **kw)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), (None if ST is None else ST.cpu().numpy())


def sel_heads(x, pairs):
    """Inputs restricted to the (b, h) pairs, as a batch of len(pairs) single-head sequences."""
    out = {}
    for n in ("q", "k", "v", "alpha", "b", "w"):
        out[n] = np.stack([x[n][b, :, h] for b, h in pairs])[:, :, None, :]
    out["S0"] = None if x["S0"] is None else np.stack([x["S0"][b, h] for b, h in pairs])[:, None]
    return out


def check_sampled(x, o, ST, pairs, tol_s, ref="gdn2"):
    s = sel_heads(x, pairs)
    if ref == "gdn2":
        o_ref, S_ref = oracle.gdn2(s["q"], s["k"], s["v"], s["alpha"], s["b"], s["w"], s["S0"])
    elif ref == "kda":
        beta = np.stack([x["beta"][b, :, h] for b, h in pairs])[:, :, None]
        o_ref, S_ref = oracle.kda(s["q"], s["k"], s["v"], s["alpha"], beta, s["S0"])
    else:
        beta = np.stack([x["beta"][b, :, h] for b, h in pairs])[:, :, None]
        a1 = np.stack([x["alpha_scalar"][b, :, h] for b, h in pairs])[:, :, None]
        o_ref, S_ref = oracle.gdn(s["q"], s["k"], s["v"], a1, beta, s["S0"])
    og = np.stack([o[b, :, h] for b, h in pairs])[:, :, None]
    eo = check_o(og, o_ref, x["dtype"])
    if ST is not None:
        Sg = np.stack([ST[b, h] for b, h in pairs])[:, None]
        check_s(Sg, S_ref, tol_s)
    return eo


# ---------------------------------------------------------------- small, full comparison

def test_tiny_fp32_full(g):
    """B=1, T=256, H=2, d=64, FP32 throughout, S0 = 0: every output checked."""
    x = gi.chunk_inputs(**gi.TINY_FP32, seed=0)
    o, ST = run_chunk(g, x)
    o_ref, S_ref = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], None)
    assert rel(o, o_ref) <= TOL_FP32
    check_s(ST, S_ref, TOL_FP32)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 129, 200])
@pytest.mark.parametrize("d", [64, 128])
def test_small_full(g, dtype, T, d):
    """Several chunks and a ragged tail, nonzero S0; every output checked."""
    x = gi.chunk_inputs(2, T, 3, d, d, dtype=dtype, seed=T + d, s0_std=0.05)
    o, ST = run_chunk(g, x)
    o_ref, S_ref = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
    check_o(o, o_ref, dtype)
    check_s(ST, S_ref, TOL_FP32 if dtype == "fp32" else TOL_BF16_S)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("dk,dv", [(128, 64), (64, 128)])
def test_prefill_unequal_head_sizes(g, dtype, dk, dv):
    """d_k != d_v (the FP32 CUDA-core prefill): several chunks, ragged tail, S0."""
    x = gi.chunk_inputs(2, 129, 2, dk, dv, dtype=dtype, seed=dk + 3 * dv, s0_std=0.05)
    o, ST = run_chunk(g, x)
    o_ref, S_ref = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
    check_o(o, o_ref, dtype)
    check_s(ST, S_ref, TOL_FP32 if dtype == "fp32" else TOL_BF16_S)


def _gate_case(case, seed):
    """B=1, T=500, H=4, d=128, BF16, S0 != 0, with the gates pushed to an edge of their range."""
    x = gi.chunk_inputs(1, 500, 4, 128, 128, dtype="bf16", seed=seed, s0_std=0.05)
    rng = np.random.default_rng(seed + 1000)
    if case == "strong_decay":
        # -ln(alpha) in [1.0, 1.2]: about 70 nats per 64 tokens, past the 2^-64 floor of one
        # chunk's decay, so the tensor-core path cuts every chunk about two thirds of the way.
        x["alpha"] = np.exp(-rng.uniform(1.0, 1.2, x["alpha"].shape)).astype(np.float32)
    elif case == "decay_to_1e-3":
        # per-channel alpha log-uniform in [1e-3, 1]: about 220 nats per 64 tokens in every
        # channel (chunks of a dozen or so tokens)
        x["alpha"] = np.exp(-rng.uniform(0.0, 6.9, x["alpha"].shape)).astype(np.float32)
    elif case == "extreme_decay":
        # 2% of the (token, channel) decays at 1e-30 and 1% exactly 0 (a state row wiped in
        # one token): most tokens start a new chunk; alpha below 2^-64 is computed as 2^-64
        a = x["alpha"].copy()
        u = rng.random(a.shape)
        a[u < 0.02] = np.float32(1e-30)
        a[(u >= 0.02) & (u < 0.03)] = np.float32(0.0)
        x["alpha"] = a
    elif case == "no_decay":
        x["alpha"] = np.ones_like(x["alpha"])
    elif case == "erase_to_2":
        # erase gate over [0, 2], the range of the pages' gate ablation
        x["b"] = (2.0 * x["b"]).astype(np.float32)
    return x


@pytest.mark.parametrize("case", ["strong_decay", "decay_to_1e-3", "extreme_decay", "no_decay", "erase_to_2"])
def test_gate_edges(g, case):
    """Every output and the final state, against the oracle, at the edges of the gate ranges
    (the BF16 d=128 tensor-core path): alpha anywhere in [0, 1] ("Independent decisions on
    two axes": a channel-wise decay gate) and an erase gate up to 2."""
    x = _gate_case(case, seed={"strong_decay": 31, "no_decay": 32, "erase_to_2": 33, "decay_to_1e-3": 34,
                               "extreme_decay": 35}[case])
    o, ST = run_chunk(g, x)
    o_ref, S_ref = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
    check_o(o, o_ref, "bf16")
    check_s(ST, S_ref, TOL_BF16_S)


def test_multi_wave_grid(g):
    """More CTAs than SMs (B=12, H=16: 384 column-half CTAs on 148 SMs, about three
    waves), ragged tail, nonzero S0: every output of every head checked, so each SM
    runs several CTAs one after another through the same Tensor Memory."""
    x = gi.chunk_inputs(12, 130, 16, 128, 128, dtype="bf16", seed=77, s0_std=0.05)
    o, ST = run_chunk(g, x)
    o_ref, S_ref = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
    check_o(o, o_ref, "bf16")
    check_s(ST, S_ref, TOL_BF16_S)


def test_delta_identity_fp32(g):
    """b = 1, w = 1, unit keys, q = k: every output equals v (the delta rule writes the error)."""
    x = gi.chunk_inputs(1, 130, 2, 128, 128, dtype="fp32", seed=9, s0_std=0.1)
    kk = x["k"]
    d = to_dev(x)
    kd = torch.from_numpy(kk).cuda()
    ones = torch.ones_like(d["b"])
    o, _ = g.gdn2_chunk_fwd(kd, kd, d["v"], d["alpha"], ones, torch.ones_like(d["w"]), d["S0"])
    torch.cuda.synchronize()
    assert rel(o.cpu().numpy(), x["v"]) <= TOL_FP32


def test_no_erase_matches_closed_form(g):
    """b = 0: the output is the decayed causal linear-attention sum (explicit O(T^2) oracle)."""
    x = gi.chunk_inputs(1, 96, 2, 64, 64, dtype="fp32", seed=4, s0_std=0.1)
    x["b"] = np.zeros_like(x["b"])
    o, _ = run_chunk(g, x)
    o_ref = oracle.b0_sum(x["q"], x["k"], x["v"], x["alpha"], x["w"], x["S0"])
    assert rel(o, o_ref) <= TOL_FP32


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 128)])
def test_no_erase_closed_form_both_paths(g, dtype, d):
    """b = 0 on the tensor-core path (BF16, d = 128) and the FP32 path: every output equals the
    decayed causal linear-attention sum computed by the explicit O(T^2) oracle."""
    x = gi.chunk_inputs(2, 200, 2, d, d, dtype=dtype, seed=44, s0_std=0.05)
    x["b"] = np.zeros_like(x["b"])
    o, _ = run_chunk(g, x)
    o_ref = oracle.b0_sum(x["q"], x["k"], x["v"], x["alpha"], x["w"], x["S0"])
    check_o(o, o_ref, dtype)


def test_state_inplace_and_optional_outputs(g):
    x = gi.chunk_inputs(1, 100, 2, 128, 128, dtype="bf16", seed=3, s0_std=0.05)
    d = to_dev(x)
    ref_o, ref_S = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], d["S0"])
    S = d["S0"].clone()
    o2, S2 = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S, S_T=S)
    assert S2.data_ptr() == S.data_ptr()
    o3, S3 = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], d["S0"], output_final_state=False)
    torch.cuda.synchronize()
    assert S3 is None
    assert torch.equal(o2, ref_o) and torch.equal(S, ref_S) and torch.equal(o3, ref_o)


def test_zero_length_and_empty(g):
    x = gi.chunk_inputs(2, 1, 2, 64, 64, dtype="bf16", seed=1, s0_std=0.1)
    d = to_dev(x)
    z = {n: t[:, :0].contiguous() for n, t in d.items() if n != "S0"}
    o, ST = g.gdn2_chunk_fwd(z["q"], z["k"], z["v"], z["alpha"], z["b"], z["w"], d["S0"])
    o0, ST0 = g.gdn2_chunk_fwd(z["q"], z["k"], z["v"], z["alpha"], z["b"], z["w"], None)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(ST, d["S0"]) and torch.count_nonzero(ST0) == 0
    e = {n: t[:0].contiguous() for n, t in d.items() if n != "S0"}
    o, ST = g.gdn2_chunk_fwd(e["q"], e["k"], e["v"], e["alpha"], e["b"], e["w"], None)
    assert o.numel() == 0 and ST.numel() == 0


def test_deterministic(g):
    x = gi.chunk_inputs(2, 300, 4, 128, 128, dtype="bf16", seed=8, s0_std=0.05)
    a = run_chunk(g, x)
    b = run_chunk(g, x)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_repeated_calls_bitwise_identical(g):
    """50 back-to-back calls on a ragged grid of about three waves give bit-identical o and
    S_T: the kernel's arithmetic order is fixed, so any hand-over race between its warp
    roles would show up as a difference."""
    x = gi.chunk_inputs(12, 1000, 16, 128, 128, dtype="bf16", seed=5, s0_std=0.05)
    d = to_dev(x)
    S0 = d["S0"]
    o0, S_T0 = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S0)
    o0, S_T0 = o0.clone(), S_T0.clone()
    same = 0
    for _ in range(50):
        o, S_T = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S0)
        same += int(torch.equal(o, o0) and torch.equal(S_T, S_T0))
    assert same == 50
    assert g.gdn2_device_error(clear=False) == 0


# ---------------------------------------------------------------- full workload sizes

@pytest.fixture(scope="module")
def prefill_4k():
    return gi.chunk_inputs(**gi.PREFILL_4K, seed=0)


def test_prefill_4k_sampled(g, prefill_4k):
    """B=4, T=4096, H=16, d=128, BF16 q/k/v, FP32 gates, S0 = 0 (the prefill workload)."""
    o, ST = run_chunk(g, prefill_4k)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(ST))
    check_sampled(prefill_4k, o, ST, [(0, 0), (1, 7), (2, 11), (3, 15)], TOL_BF16_S)


def test_prefill_4k_every_head(g, prefill_4k):
    """The prefill workload (B=4, T=4096, H=16, d=128), every head of o and S_T against the
    oracle element by element (the same launch the bench times)."""
    x = prefill_4k
    o, ST = run_chunk(g, x)
    o_ref, S_ref = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], None)
    check_o(o, o_ref, "bf16")
    check_s(ST, S_ref, TOL_BF16_S)


@pytest.mark.parametrize("variant", ["kda", "gdn"])
def test_reductions_at_prefill_shape(g, variant):
    """b = w = beta per (token, head): matches the separately coded KDA recurrence; with scalar
    alpha as well, the Gated DeltaNet recurrence ("Independent decisions on two axes")."""
    x = gi.chunk_inputs(**gi.PREFILL_4K, seed=0, gates=variant)
    o, ST = run_chunk(g, x)
    check_sampled(x, o, ST, [(1, 3), (3, 12)], TOL_BF16_S, ref=variant)


@pytest.fixture(scope="module")
def long_ragged():
    return gi.chunk_inputs(**gi.LONG_RAGGED, seed=0)


def test_long_ragged_sampled(g, long_ragged):
    """B=1, T=65573 (not a multiple of 64), H=16, d=128, S0 ~ N(0, 0.02^2)."""
    o, ST = run_chunk(g, long_ragged)
    check_sampled(long_ragged, o, ST, [(0, 2), (0, 9)], TOL_BF16_S)


def test_long_ragged_split_chaining(g, long_ragged):
    """Splitting at T1 = floor(T/2) and chaining S_T into the second call equals one call."""
    x = long_ragged
    T = x["T"]
    T1 = T // 2
    d = to_dev(x)
    o_full, S_full = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], d["S0"])
    parts = [{n: d[n][:, sl].contiguous() for n in ("q", "k", "v", "alpha", "b", "w")}
             for sl in (slice(0, T1), slice(T1, T))]
    oa, Sa = g.gdn2_chunk_fwd(*(parts[0][n] for n in ("q", "k", "v", "alpha", "b", "w")), d["S0"])
    ob, Sb = g.gdn2_chunk_fwd(*(parts[1][n] for n in ("q", "k", "v", "alpha", "b", "w")), Sa)
    torch.cuda.synchronize()
    o_split = torch.cat([oa, ob], 1).float().cpu().numpy()
    # both are BF16 results with different chunk boundaries: allow each its own rounding
    assert rel_bf16(o_split, o_full.float().cpu().numpy(), roundings=2) <= TOL_BF16_O
    assert rel(Sb.cpu().numpy(), S_full.cpu().numpy()) <= TOL_BF16_S
    check_sampled(x, o_split, Sb.cpu().numpy(), [(0, 5)], TOL_BF16_S)


# ---------------------------------------------------------------- decode step

def run_decode(g, x, steps):
    dt = torch.bfloat16 if x["dtype"] == "bf16" else torch.float32
    dev = {n: torch.from_numpy(x[n]).cuda().to(dt if n in ("q", "k", "v") else torch.float32)
           for n in ("q", "k", "v", "alpha", "b", "w")}
    S = torch.from_numpy(x["S0"]).cuda()
    outs = []
    for s in range(steps):
        outs.append(g.gdn2_recurrent_step(*(dev[n][s] for n in ("q", "k", "v", "alpha", "b", "w")), S))
    torch.cuda.synchronize()
    return torch.stack(outs).float().cpu().numpy(), S.cpu().numpy()


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 64), (64, 128)])
def test_decode_small(g, dtype, dk, dv):
    x = gi.decode_inputs(5, 3, 4, dk, dv, dtype=dtype, seed=dk + dv, s0_std=0.1)
    o, S = run_decode(g, x, 5)
    S_ref = x["S0"].astype(np.float64)
    tol_s = TOL_FP32 if dtype == "fp32" else TOL_BF16_S
    for s in range(5):
        o_ref, S_ref = oracle.gdn2_step(*(x[n][s] for n in ("q", "k", "v", "alpha", "b", "w")), S_ref)
        check_o(o[s], o_ref, dtype)
    assert rel(S, S_ref) <= tol_s


@pytest.mark.parametrize("case", ["strong_decay", "no_decay", "erase_to_2"])
def test_decode_gate_edges(g, case):
    """Decode steps at the edges of the gate ranges (as test_gate_edges), every output."""
    x = gi.decode_inputs(8, 3, 4, 128, 128, dtype="bf16", seed=41, s0_std=0.1)
    rng = np.random.default_rng(42)
    if case == "strong_decay":
        x["alpha"] = np.exp(-rng.uniform(1.0, 1.2, x["alpha"].shape)).astype(np.float32)
    elif case == "no_decay":
        x["alpha"] = np.ones_like(x["alpha"])
    else:
        x["b"] = (2.0 * x["b"]).astype(np.float32)
    o, S = run_decode(g, x, 8)
    S_ref = x["S0"].astype(np.float64)
    for s in range(8):
        o_ref, S_ref = oracle.gdn2_step(*(x[n][s] for n in ("q", "k", "v", "alpha", "b", "w")), S_ref)
        check_o(o[s], o_ref, "bf16")
    assert rel(S, S_ref) <= TOL_BF16_S


def test_decode_b256_64_steps_sampled(g):
    """Batch 256, H=16, d=128, FP32 state N(0, 0.02^2), 64 consecutive in-place steps."""
    x = gi.decode_inputs(**gi.DECODE_B256, seed=0)
    o, S = run_decode(g, x, 64)
    pairs = [(0, 0), (17, 5), (128, 9), (255, 15), (200, 3), (64, 12)]
    Sr = np.stack([x["S0"][b, h] for b, h in pairs])[:, None].astype(np.float64)
    for s in range(64):
        args = [np.stack([x[n][s, b, h] for b, h in pairs])[:, None] for n in ("q", "k", "v", "alpha", "b", "w")]
        o_ref, Sr = oracle.gdn2_step(*args, Sr)
        og = np.stack([o[s, b, h] for b, h in pairs])[:, None]
        check_o(og, o_ref, "bf16")
    Sg = np.stack([S[b, h] for b, h in pairs])[:, None]
    assert rel(Sg, Sr) <= TOL_BF16_S
    assert np.all(np.isfinite(S))


def test_decode_equals_chunk_of_one_token(g):
    """The two modes compute the same mathematics: T = 1 prefill equals one decode step."""
    x = gi.chunk_inputs(4, 1, 3, 128, 128, dtype="fp32", seed=21, s0_std=0.1)
    d = to_dev(x)
    o_c, S_c = g.gdn2_chunk_fwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], d["S0"])
    S = d["S0"].clone()
    o_d = g.gdn2_recurrent_step(*(d[n][:, 0].contiguous() for n in ("q", "k", "v", "alpha", "b", "w")), S)
    torch.cuda.synchronize()
    assert rel(o_d.cpu().numpy(), o_c[:, 0].cpu().numpy()) <= TOL_FP32
    assert rel(S.cpu().numpy(), S_c.cpu().numpy()) <= TOL_FP32


def test_zz_no_device_error_flag(g):
    """No bounded wait inside any kernel gave up during the parity runs above."""
    assert g.gdn2_device_error(clear=True) == 0


def test_zzz_wait_limit_gives_up_cleanly(g):
    """The kernels' failure handling, exercised without faulting the GPU: with every
    internal wait limited to a few thousand cycles the prefill gives up, raises the
    device-side flag, releases its resources and returns; with the default limit back, the
    next call is bit-identical to a clean run (the context is unharmed)."""
    x = gi.chunk_inputs(2, 300, 4, 128, 128, dtype="bf16", seed=12, s0_std=0.05)
    d = to_dev(x)
    args = [d[n] for n in ("q", "k", "v", "alpha", "b", "w")]
    o_ref, S_ref = g.gdn2_chunk_fwd(*args, d["S0"])
    torch.cuda.synchronize()
    assert g.gdn2_device_error(clear=True) == 0
    try:
        g.gdn2_set_wait_limit(2000)
        g.gdn2_chunk_fwd(*args, d["S0"])
        torch.cuda.synchronize()
    finally:
        g.gdn2_set_wait_limit(0)
    assert g.gdn2_device_error(clear=True) != 0
    o2, S2 = g.gdn2_chunk_fwd(*args, d["S0"])
    torch.cuda.synchronize()
    assert g.gdn2_device_error(clear=True) == 0
    assert torch.equal(o2, o_ref) and torch.equal(S2, S_ref)
