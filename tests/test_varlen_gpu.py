"""Packed variable-length prefill (gdn2_chunk_fwd_varlen) on the GPU: every sequence
of the pack against the FP64 oracle run on that sequence alone, and bit for bit
against a separate gdn2_chunk_fwd call on it (chunking restarts at every sequence
start in both, so the arithmetic is the same).  Both kernels: the tensor-core path
(BF16, d = 128) and the FP32 CUDA-core path."""
import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import oracle
from test_parity_gpu import TOL_BF16_S, TOL_FP32, check_o, check_s

pytestmark = pytest.mark.gpu

LENGTHS = [1, 63, 0, 64, 130, 300, 65]


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_111_b200 as mod
    mod.load_library()
    return mod


def _packed(dtype, d, seed, alpha=None):
    total = sum(LENGTHS)
    x = gi.chunk_inputs(1, total, 3, d, d, dtype=dtype, seed=seed)
    rng = np.random.default_rng(seed + 7)
    S0 = (rng.standard_normal((len(LENGTHS), 3, d, d)) * 0.05).astype(np.float32)
    if alpha is not None:
        x["alpha"] = alpha(rng, x["alpha"].shape)
    cu = np.concatenate([[0], np.cumsum(LENGTHS)]).astype(np.int32)
    return x, S0, cu


def _run(g, x, S0, cu):
    tdt = torch.bfloat16 if x["dtype"] == "bf16" else torch.float32
    d = {n: torch.from_numpy(np.ascontiguousarray(x[n][0])).cuda().to(tdt if n in "qkv" else torch.float32)
         for n in ("q", "k", "v", "alpha", "b", "w")}
    S0d = torch.from_numpy(S0).cuda()
    cud = torch.from_numpy(cu).cuda()
    o, ST = g.gdn2_chunk_fwd_varlen(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], cud, S0d)
    torch.cuda.synchronize()
    return d, S0d, o, ST


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("fp32", 64), ("bf16", 64)])
def test_varlen_matches_oracle_and_separate_calls(g, dtype, d):
    x, S0, cu = _packed(dtype, d, seed=60 + d)
    dd, S0d, o, ST = _run(g, x, S0, cu)
    tol_s = TOL_FP32 if dtype == "fp32" else TOL_BF16_S
    for n, L in enumerate(LENGTHS):
        a, e = cu[n], cu[n + 1]
        if L == 0:
            assert torch.equal(ST[n], S0d[n])
            continue
        seg = {m: x[m][:, a:e] for m in ("q", "k", "v", "alpha", "b", "w")}
        o_ref, S_ref = oracle.gdn2(seg["q"], seg["k"], seg["v"], seg["alpha"], seg["b"], seg["w"], S0[n:n + 1])
        check_o(o[a:e].float().cpu().numpy()[None], o_ref, dtype)
        check_s(ST[n].cpu().numpy()[None], S_ref, tol_s)
        # one gdn2_chunk_fwd call on the sequence alone: identical bits
        one = {m: dd[m][a:e].unsqueeze(0).contiguous() for m in ("q", "k", "v", "alpha", "b", "w")}
        o1, S1 = g.gdn2_chunk_fwd(*(one[m] for m in ("q", "k", "v", "alpha", "b", "w")), S0d[n:n + 1].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(o1[0], o[a:e]) and torch.equal(S1[0], ST[n])


def test_varlen_with_cut_chunks(g):
    """Strong per-channel decay (alpha log-uniform down to 1e-3): the tensor-core path cuts
    chunks inside every sequence of the pack; still the oracle's result per sequence."""
    x, S0, cu = _packed("bf16", 128, seed=71,
                        alpha=lambda rng, shape: np.exp(-rng.uniform(0.0, 6.9, shape)).astype(np.float32))
    _, _, o, ST = _run(g, x, S0, cu)
    for n, L in enumerate(LENGTHS):
        if L == 0:
            continue
        a, e = cu[n], cu[n + 1]
        seg = {m: x[m][:, a:e] for m in ("q", "k", "v", "alpha", "b", "w")}
        o_ref, S_ref = oracle.gdn2(seg["q"], seg["k"], seg["v"], seg["alpha"], seg["b"], seg["w"], S0[n:n + 1])
        check_o(o[a:e].float().cpu().numpy()[None], o_ref, "bf16")
        check_s(ST[n].cpu().numpy()[None], S_ref, TOL_BF16_S)
