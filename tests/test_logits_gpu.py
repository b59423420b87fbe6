"""Parity of gdn2_chunk_fwd_logits (input preparation fused into the tensor-core
prefill, through the C ABI) with the FP64 oracle: oracle_gdn2_prep on the same
BF16 logits, then the recurrence.  Tolerances as for the BF16 prefill: o 2e-2
beyond its own BF16 rounding and 1e-2 normwise, S_T 1e-2 (max |delta| / RMS).
"""
import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import oracle
from test_parity_gpu import check_o, check_s

pytestmark = pytest.mark.gpu
TOL_S = 1e-2
NAMES = ("xq", "xk", "xv", "xa", "xb", "xw")


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_111_b200 as mod
    mod.load_library()
    return mod


def run(g, x):
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n])).cuda().to(torch.bfloat16) for n in NAMES}
    S0 = None if x["S0"] is None else torch.from_numpy(x["S0"]).cuda()
    o, ST = g.gdn2_chunk_fwd_logits(*(d[n] for n in NAMES), S0)
    torch.cuda.synchronize()
    return o.float().cpu().numpy(), ST.cpu().numpy()


def reference(x):
    return oracle.gdn2_from_logits(*(x[n] for n in NAMES), x["S0"])


@pytest.mark.parametrize("B,T,H,s0", [(2, 150, 2, 0.05), (1, 64, 3, None), (1, 1, 2, 0.05), (3, 257, 1, 0.02)])
def test_logits_prefill_matches_oracle(g, B, T, H, s0):
    x = gi.logit_inputs(B, T, H, 128, 128, seed=40 + T, s0_std=s0)
    o, ST = run(g, x)
    o_ref, S_ref = reference(x)
    check_o(o, o_ref, "bf16")
    check_s(ST, S_ref, TOL_S)


def test_logits_strong_decay_and_zero_rows(g):
    """Decay logits up to +30 (alpha down to 1e-13: chunks cut early) and all-zero q/k rows."""
    x = gi.logit_inputs(1, 300, 2, 128, 128, seed=7, s0_std=0.05)
    rng = np.random.default_rng(8)
    mask = rng.random(x["xa"].shape) < 0.1
    x["xa"] = gi.round_to_bf16(np.where(mask, rng.uniform(5.0, 30.0, x["xa"].shape), x["xa"]).astype(np.float32))
    x["xq"][0, 10, 0] = 0.0
    x["xk"][0, 70:73, 1] = 0.0
    o, ST = run(g, x)
    o_ref, S_ref = reference(x)
    check_o(o, o_ref, "bf16")
    check_s(ST, S_ref, TOL_S)


def test_logits_full_size_sampled_heads(g):
    """B 4, T 4096, H 16 (the prefill workload) in one launch; two (sequence, head)
    pairs recomputed by the oracle over every token."""
    B, T, H = 4, 4096, 16
    x = gi.logit_inputs(B, T, H, 128, 128, seed=50)
    o, ST = run(g, x)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(ST))
    for b, h in ((0, 3), (3, 15)):
        sub = {n: x[n][b:b + 1, :, h:h + 1] for n in NAMES}
        o_ref, S_ref = oracle.gdn2_from_logits(*(sub[n] for n in NAMES))
        check_o(o[b:b + 1, :, h:h + 1], o_ref, "bf16")
        check_s(ST[b:b + 1, h:h + 1], S_ref, TOL_S)
