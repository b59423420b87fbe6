"""Seeded synthetic inputs for the Gated DeltaNet-2 recurrence.

This module is the only code shared by the CUDA path's tests/bench and the FP64
oracle.  It draws random numbers and applies the input activations that the
method places *before* the recurrence; it holds none of the recurrence's own
arithmetic.

Recipe (per token and head; "Token processing and parallel training" and
"Independent decisions on two axes" of the Gated DeltaNet-2 analysis):
  q, k  ~ N(0,1), then L2-normalised over the key channels
  v     = SiLU(N(0,1))
  alpha = exp(-softplus(N(-2,1)))     channel-wise decay, one value per key channel
  b     = sigmoid(N(0,1))             erase gate, per key channel
  w     = sigmoid(N(0,1))             write gate, per value channel
  S0    ~ N(0, s0_std^2) in FP32, or absent (zeros)

All draws are float32 from ``numpy.random.default_rng(seed)`` in the fixed
order q, k, v, alpha, b, w, S0.  For ``dtype="bf16"`` the activated q, k, v are
rounded to bfloat16 (round to nearest even) once, here, and both sides receive
exactly those values; gates and states are always float32.

Gate variants:
  "gdn2"  the general case above
  "kda"   b = w = beta broadcast over channels, beta = sigmoid(N(0,1)) per (b,t,h)
          (drawn in place of b; w is not drawn)
  "gdn"   as "kda", and alpha is one value per (b,t,h) broadcast over channels
"""
from __future__ import annotations

import numpy as np


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); result is float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def _silu(x):
    return x / (1.0 + np.exp(-x))


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def _softplus(x):
    return np.logaddexp(np.float32(0.0), x)


def _l2norm(x):
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / n).astype(np.float32)


def _draw(rng, lead, dk, dv, dtype, gates):
    """Draw q, k, v, alpha, b, w with leading shape ``lead`` (channels last)."""
    f32 = np.float32
    q = _l2norm(rng.standard_normal(lead + (dk,), dtype=f32))
    k = _l2norm(rng.standard_normal(lead + (dk,), dtype=f32))
    v = _silu(rng.standard_normal(lead + (dv,), dtype=f32)).astype(f32)
    if gates == "gdn":
        a1 = np.exp(-_softplus(rng.standard_normal(lead, dtype=f32) - f32(2.0))).astype(f32)
        alpha = np.ascontiguousarray(np.broadcast_to(a1[..., None], lead + (dk,)))
    else:
        alpha = np.exp(-_softplus(rng.standard_normal(lead + (dk,), dtype=f32) - f32(2.0))).astype(f32)
    if gates == "gdn2":
        bg = _sigmoid(rng.standard_normal(lead + (dk,), dtype=f32)).astype(f32)
        wg = _sigmoid(rng.standard_normal(lead + (dv,), dtype=f32)).astype(f32)
        beta = None
    elif gates in ("kda", "gdn"):
        beta = _sigmoid(rng.standard_normal(lead, dtype=f32)).astype(f32)
        bg = np.ascontiguousarray(np.broadcast_to(beta[..., None], lead + (dk,)))
        wg = np.ascontiguousarray(np.broadcast_to(beta[..., None], lead + (dv,)))
    else:
        raise ValueError(f"unknown gate variant {gates!r}")
    if dtype == "bf16":
        q, k, v = round_to_bf16(q), round_to_bf16(k), round_to_bf16(v)
    elif dtype != "fp32":
        raise ValueError(f"unknown dtype {dtype!r}")
    out = dict(q=q, k=k, v=v, alpha=alpha, b=bg, w=wg)
    if beta is not None:
        out["beta"] = beta
        if gates == "gdn":
            out["alpha_scalar"] = alpha[..., 0].copy()
    return out


def chunk_inputs(B, T, H, dk, dv, *, dtype="bf16", seed=0, s0_std=None, gates="gdn2"):
    """Inputs for one prefill call: tensors [B,T,H,d] and S0 [B,H,dk,dv] (or None)."""
    rng = np.random.default_rng(seed)
    out = _draw(rng, (B, T, H), dk, dv, dtype, gates)
    out["S0"] = None
    if s0_std is not None:
        out["S0"] = (rng.standard_normal((B, H, dk, dv), dtype=np.float32) * np.float32(s0_std)).astype(np.float32)
    out.update(B=B, T=T, H=H, dk=dk, dv=dv, dtype=dtype)
    return out


def logit_inputs(B, T, H, dk, dv, *, seed=0, s0_std=None, a_shift=-2.0):
    """Pre-activation inputs for the logits prefill: xq, xk, xv, xb, xw ~ N(0, 1) and
    xa ~ N(0, 1) + a_shift, each rounded to BF16 (the kernel reads BF16), [B,T,H,d];
    S0 [B,H,dk,dv] or None.  With a_shift = -2 the decays have the distribution of
    chunk_inputs' alpha."""
    rng = np.random.default_rng(seed)
    f32 = np.float32
    out = {}
    for n, d in (("xq", dk), ("xk", dk), ("xv", dv), ("xa", dk), ("xb", dk), ("xw", dv)):
        x = rng.standard_normal((B, T, H, d), dtype=f32)
        if n == "xa":
            x = x + f32(a_shift)
        out[n] = round_to_bf16(x)
    out["S0"] = None
    if s0_std is not None:
        out["S0"] = (rng.standard_normal((B, H, dk, dv), dtype=f32) * f32(s0_std)).astype(f32)
    out.update(B=B, T=T, H=H, dk=dk, dv=dv, dtype="bf16")
    return out


def decode_inputs(steps, B, H, dk, dv, *, dtype="bf16", seed=0, s0_std=0.02, gates="gdn2"):
    """Inputs for ``steps`` decode steps: tensors [steps,B,H,d] and S0 [B,H,dk,dv]."""
    rng = np.random.default_rng(seed)
    out = _draw(rng, (steps, B, H), dk, dv, dtype, gates)
    out["S0"] = (rng.standard_normal((B, H, dk, dv), dtype=np.float32) * np.float32(s0_std)).astype(np.float32)
    out.update(steps=steps, B=B, H=H, dk=dk, dv=dv, dtype=dtype)
    return out


# The workloads, by name and size.
TINY_FP32 = dict(B=1, T=256, H=2, dk=64, dv=64, dtype="fp32")
PREFILL_4K = dict(B=4, T=4096, H=16, dk=128, dv=128, dtype="bf16")
DECODE_B256 = dict(steps=64, B=256, H=16, dk=128, dv=128, dtype="bf16", s0_std=0.02)
LONG_RAGGED = dict(B=1, T=65573, H=16, dk=128, dv=128, dtype="bf16", s0_std=0.02)
