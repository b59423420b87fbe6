"""gdn2_chunk_bwd_noalloc: the backward with the library's fixed device workspace.

Called through the C ABI (ctypes) on preallocated buffers, two calls in a row,
each compared with gdn2_chunk_bwd (caller workspace) on the same inputs, at the
tolerances of the backward parity tests.  This file is collected last on
purpose: it must hold both in a fresh process (where its first call looks up
the scratch array) and after every other test has used the library.
"""
import ctypes

import numpy as np
import pytest
import torch

import gdn2_inputs as gi
import gated_delta_rule_111_b200 as g

NAMES = ("dq", "dk", "dv", "dalpha", "db", "dw", "dS0")
TOL_BF16 = 2e-2          # BF16 gradients dq, dk, dv: max |delta| / RMS(ref)
TOL_F32 = 1e-4           # FP32 gradients


def _rel(a, ref):
    a, ref = a.double(), ref.double()
    return float((a - ref).abs().max() / ref.pow(2).mean().sqrt().clamp_min(1e-30))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_rejects_sizes_beyond_its_fixed_workspace():
    """Host-side check, before any CUDA call."""
    lib = g.load_library()
    need = lib.gdn2_chunk_bwd_workspace_size(4, 4096, 16, 128, 128)
    assert need > 32 << 20
    A = 0x10000
    st = lib.gdn2_chunk_bwd_noalloc(*([A] * 8), None, *([A * 64] * 6), None, 4, 4096, 16, 128, 128, 0, None)
    assert st == g.GDN2_ERR_INVALID_ARG
    msg = lib.gdn2_last_error().decode()
    assert "gdn2_chunk_bwd_noalloc" in msg and "more than its fixed" in msg


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_twice():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = g.load_library()
    dev = torch.device("cuda", 0)
    B, T, H, dk, dv = 2, 200, 2, 128, 128
    assert lib.gdn2_chunk_bwd_workspace_size(B, T, H, dk, dv) <= 32 << 20
    x = gi.chunk_inputs(B, T, H, dk, dv, dtype="bf16", seed=31, s0_std=0.05)
    d = {n: torch.from_numpy(x[n]).to(dev).to(torch.bfloat16 if n in "qkv" else torch.float32)
         for n in ("q", "k", "v", "alpha", "b", "w")}
    S0 = torch.from_numpy(x["S0"]).to(dev)
    rng = np.random.default_rng(32)
    dO = torch.from_numpy(rng.standard_normal((B, T, H, dv)).astype(np.float32)).to(dev).to(torch.bfloat16)
    dST = torch.from_numpy((rng.standard_normal((B, H, dk, dv)) * 0.5).astype(np.float32)).to(dev)

    ref = g.gdn2_chunk_bwd(d["q"], d["k"], d["v"], d["alpha"], d["b"], d["w"], S0, dO, dST)
    torch.cuda.synchronize()
    out = {n: torch.full_like(ref[n], float("nan")) for n in NAMES}
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    for call in range(2):
        with torch.cuda.device(dev):
            st = lib.gdn2_chunk_bwd_noalloc(
                _ptr(d["q"]), _ptr(d["k"]), _ptr(d["v"]), _ptr(d["alpha"]), _ptr(d["b"]), _ptr(d["w"]), _ptr(S0),
                _ptr(dO), _ptr(dST), *(_ptr(out[n]) for n in NAMES), B, T, H, dk, dv, g.GDN2_BF16, stream)
        assert st == g.GDN2_OK, lib.gdn2_last_error().decode()
        torch.cuda.synchronize()
        for n in NAMES:
            tol = TOL_BF16 if n in ("dq", "dk", "dv") else TOL_F32
            e = _rel(out[n], ref[n])
            assert e <= tol, f"call {call}: {n} differs from gdn2_chunk_bwd by {e:.3e} > {tol}"
        for n in NAMES:
            out[n].fill_(float("nan"))
