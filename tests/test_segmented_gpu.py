"""Segment-parallel prefill (gdn2_chunk_fwd_segmented, through the C ABI) against the
FP64 oracle on the whole sequences, at the tolerances of the prefill parity tests.

Cases span a ragged last segment, more segments requested than chunks (capped),
strong decay (chunks cut inside segments), S0 = None, B > 1, the automatic choice
(one segment on the 4K shape: bit-identical to gdn2_chunk_fwd) and the long ragged
workload (B=1, T=65573, H=16), where the automatic choice splits each sequence."""
import numpy as np
import pytest
import torch

import gdn2_inputs as gi
from test_parity_gpu import TOL_BF16_O, TOL_BF16_S, check_o, check_s, check_sampled, rel, rel_bf16, to_dev
import oracle

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "alpha", "b", "w")


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_111_b200 as mod
    mod.load_library()
    return mod


def run_seg(g, x, segments, **kw):
    d = to_dev(x)
    o, ST = g.gdn2_chunk_fwd_segmented(*(d[n] for n in NAMES), d["S0"], segments=segments, **kw)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), ST.cpu().numpy()


CASES = [
    # B, T, H, segments, s0
    (2, 700, 2, 3, 0.05),      # segments of 256 tokens, the last 188
    (1, 1000, 1, 5, 0.05),     # 4 chunks per segment, last ragged
    (3, 130, 2, 8, 0.05),      # 3 chunks: capped at 3 segments of 64, 64, 2 tokens
    (1, 256, 2, 4, None),      # four whole chunks, zero start state
    (1, 640, 3, 2, 0.3),       # two segments, larger start state
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c[0]}T{c[1]}H{c[2]}-P{c[3]}")
def test_segmented_matches_oracle(g, case):
    B, T, H, P, s0 = case
    assert g.gdn2_chunk_fwd_segments(B, T, H, 128, 128, P) > 1
    x = gi.chunk_inputs(B, T, H, 128, 128, dtype="bf16", seed=100 + T, s0_std=s0)
    o, ST = run_seg(g, x, P)
    o_ref, S_ref = oracle.gdn2(*(x[n] for n in NAMES), x["S0"])
    check_o(o, o_ref, "bf16")
    check_s(ST, S_ref, TOL_BF16_S)


def test_segmented_strong_decay(g):
    """alpha log-uniform down to 1e-3: chunks are cut inside every segment."""
    x = gi.chunk_inputs(1, 900, 2, 128, 128, dtype="bf16", seed=7, s0_std=0.05)
    rng = np.random.default_rng(8)
    x["alpha"] = np.exp(-rng.uniform(0.0, 6.9, x["alpha"].shape)).astype(np.float32)
    o, ST = run_seg(g, x, 4)
    o_ref, S_ref = oracle.gdn2(*(x[n] for n in NAMES), x["S0"])
    check_o(o, o_ref, "bf16")
    check_s(ST, S_ref, TOL_BF16_S)


def test_state_inplace_and_workspace_reuse(g):
    """S_T may alias S0; a reused workspace holding garbage gives identical bits."""
    x = gi.chunk_inputs(1, 500, 2, 128, 128, dtype="bf16", seed=21, s0_std=0.05)
    d = to_dev(x)
    need = g.gdn2_chunk_fwd_segmented_workspace_size(1, 500, 2, 128, 128, 3)
    ws = torch.full((need,), 0x7f, dtype=torch.uint8, device="cuda")
    o1, S1 = g.gdn2_chunk_fwd_segmented(*(d[n] for n in NAMES), d["S0"], segments=3, workspace=ws)
    ws.fill_(0xff)
    S_in = d["S0"].clone()
    o2, S2 = g.gdn2_chunk_fwd_segmented(*(d[n] for n in NAMES), S_in, segments=3, workspace=ws, S_T=S_in)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2) and S2.data_ptr() == S_in.data_ptr()


def test_rejects_small_workspace(g):
    x = gi.chunk_inputs(1, 300, 1, 128, 128, dtype="bf16", seed=2)
    d = to_dev(x)
    need = g.gdn2_chunk_fwd_segmented_workspace_size(1, 300, 1, 128, 128, 3)
    ws = torch.empty((need - 256,), dtype=torch.uint8, device="cuda")
    with pytest.raises(g.Gdn2Error, match="workspace"):
        g.gdn2_chunk_fwd_segmented(*(d[n] for n in NAMES), None, segments=3, workspace=ws)


def test_auto_on_the_4k_shape_is_the_plain_call(g):
    """On B=4 T=4096 H=16 the automatic choice is one segment: the plain kernel, same bits."""
    assert g.gdn2_chunk_fwd_segments(4, 4096, 16, 128, 128, 0) == 1
    x = gi.chunk_inputs(4, 4096, 16, 128, 128, dtype="bf16", seed=3)
    d = to_dev(x)
    o1, S1 = g.gdn2_chunk_fwd(*(d[n] for n in NAMES), None)
    o2, S2 = g.gdn2_chunk_fwd_segmented(*(d[n] for n in NAMES), None, segments=0)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


@pytest.fixture(scope="module")
def long_ragged():
    return gi.chunk_inputs(**gi.LONG_RAGGED, seed=0)


def test_long_ragged_segmented(g, long_ragged):
    """B=1, T=65573, H=16, S0 != 0 with the automatic segment count (more than one on a B200):
    two heads against the oracle over every token, every head against the sequential kernel."""
    x = long_ragged
    P = g.gdn2_chunk_fwd_segments(1, x["T"], 16, 128, 128, 0)
    assert P > 1
    d = to_dev(x)
    o, ST = g.gdn2_chunk_fwd_segmented(*(d[n] for n in NAMES), d["S0"], segments=0)
    o_seq, S_seq = g.gdn2_chunk_fwd(*(d[n] for n in NAMES), d["S0"])
    torch.cuda.synchronize()
    o, ST = o.float().cpu().numpy(), ST.cpu().numpy()
    check_sampled(x, o, ST, [(0, 4), (0, 13)], TOL_BF16_S)
    # both are BF16 results of different roundings of the same recurrence
    assert rel_bf16(o, o_seq.float().cpu().numpy(), roundings=2) <= TOL_BF16_O
    assert rel(ST, S_seq.cpu().numpy()) <= TOL_BF16_S
