"""The segment composition gdn2_chunk_fwd_segmented relies on, checked in FP64 on
the token-by-token oracle (CPU only).

"Independent decisions on two axes" (Gated DeltaNet-2 analysis): per token
Sbar = diag(alpha) S, r = Sbar^T e, S' = Sbar + k (z - r)^T, i.e.
S' = (I - k e^T) diag(alpha) S + k z^T, an affine map of S.  Over a token range
therefore S_end = M S_start + C with C = the end state from S_start = 0 and
M = the end state from S_start = I with z = w * v = 0.  A sequence cut into
segments is recovered by S_start(s + 1) = M_s S_start(s) + C_s, and every
segment's outputs equal the full run's when it starts from S_start(s).

Nothing here reuses the kernels' code: M and C come from the oracle itself, run
on the pieces; the checks compare against the oracle on the whole sequence.
"""
import numpy as np

import gdn2_inputs as gi
import oracle

NAMES = ("q", "k", "v", "alpha", "b", "w")


def _piece(x, a, e):
    return {n: x[n][:, a:e] for n in NAMES}


def _transition_and_offset(p, H, d):
    """M and C of a token range, both from the oracle: C from a zero start, M from the identity
    with the written values zeroed (w = 0 makes z = w * v = 0)."""
    _, C = oracle.gdn2(p["q"], p["k"], p["v"], p["alpha"], p["b"], p["w"], None)
    eye = np.broadcast_to(np.eye(d), (1, H, d, d)).copy()
    _, M = oracle.gdn2(p["q"], p["k"], p["v"], p["alpha"], p["b"], np.zeros_like(p["w"]), eye)
    return M, C


def test_affine_in_the_start_state():
    """S_T(S0) = M S0 + C for random S0, to FP64 rounding; o is affine in S0 as well."""
    H, d = 2, 8
    x = gi.chunk_inputs(1, 37, H, d, d, dtype="fp32", seed=5, s0_std=0.3)
    M, C = _transition_and_offset(_piece(x, 0, 37), H, d)
    o_full, S_full = oracle.gdn2(*(x[n] for n in NAMES), x["S0"])
    assert np.max(np.abs(M @ x["S0"] + C - S_full)) < 1e-12
    # the identity start with z = 0 alone is the transition: M S0 is the run with w = 0 from S0
    _, S_w0 = oracle.gdn2(*(x[n] for n in NAMES[:5]), np.zeros_like(x["w"]), x["S0"])
    assert np.max(np.abs(M @ x["S0"] - S_w0)) < 1e-12
    o0, _ = oracle.gdn2(*(x[n] for n in NAMES), None)
    o_w0, _ = oracle.gdn2(*(x[n] for n in NAMES[:5]), np.zeros_like(x["w"]), x["S0"])
    assert np.max(np.abs(o0 + o_w0 - o_full)) < 1e-12


def test_segments_chain_to_the_full_run():
    """Three segments (64, 64, 29 tokens): chaining M_s, C_s gives every segment's start state
    and the final state; each segment run from its start state gives the full run's outputs."""
    H, d, T = 2, 8, 157
    bounds = [0, 64, 128, T]
    x = gi.chunk_inputs(1, T, H, d, d, dtype="fp32", seed=9, s0_std=0.2)
    o_full, S_full = oracle.gdn2(*(x[n] for n in NAMES), x["S0"])
    S = x["S0"].astype(np.float64)
    for s in range(3):
        p = _piece(x, bounds[s], bounds[s + 1])
        o_seg, S_seg = oracle.gdn2(*(p[n] for n in NAMES), S)
        assert np.max(np.abs(o_seg - o_full[:, bounds[s]:bounds[s + 1]])) < 1e-12
        if s < 2:
            M, C = _transition_and_offset(p, H, d)
            S_next = M @ S + C
            assert np.max(np.abs(S_next - S_seg)) < 1e-12
            S = S_next
        else:
            assert np.max(np.abs(S_seg - S_full)) < 1e-12


def test_strong_decay_transition_is_small_not_singular_in_use():
    """With strong per-channel decay the transition shrinks the start state; the composition
    still holds to rounding (the same FP64 check under alpha down to 1e-3)."""
    H, d = 1, 8
    x = gi.chunk_inputs(1, 50, H, d, d, dtype="fp32", seed=13, s0_std=0.5)
    rng = np.random.default_rng(14)
    x["alpha"] = np.exp(-rng.uniform(0.0, 6.9, x["alpha"].shape))
    M, C = _transition_and_offset(_piece(x, 0, 50), H, d)
    _, S_full = oracle.gdn2(*(x[n] for n in NAMES), x["S0"])
    assert np.max(np.abs(M @ x["S0"] + C - S_full)) < 1e-12
    assert np.max(np.abs(M)) < 1.0
