"""Pins for the FP64 oracle (CPU only).

The oracle is tied to facts outside itself, from "Gated DeltaNet-2: Decoupling
Erase and Write in Linear Attention" (iplexlaw.co.kr analysis) and plain algebra:

* KDA reduction -- when the erase and write gates are both the same per-token
  scalar beta, the method is KDA ("Independent decisions on two axes"); checked
  against a separately coded transition-matrix recurrence
  (I - beta k k^T) diag(alpha) S + beta k v^T.
* Gated DeltaNet reduction -- scalar decay on top of the tie recovers Gated
  DeltaNet; checked against alpha (I - beta k k^T) S + beta k v^T.
* Delta-rule identity -- with b = 1 and a unit key, S_t^T k_t = z_t exactly for any
  decay and prior state (S_t^T k = Sbar^T k + (k^T k)(z - Sbar^T k)); with q = k the
  output is w*v.  (The delta rule writes the gap between the new value and what the
  state currently returns for the key: "From a growing cache to a fixed state".)
* b = 0 -- no erase, so the output is a decayed causal linear-attention sum,
  computed by an explicit O(T^2) loop.
* alpha = 1, b = 0, w = 1 -- plain causal linear attention tril(Q K^T) V, a
  textbook special case computed with numpy matmul.
* k = 0 -- pure decay: S_T = diag(prod alpha) S0, o_t = (diag(prod_{<=t} alpha) S0)^T q_t.
* Chaining -- a fixed-size state carries all history, so run(T) equals run(T1)
  followed by run(T - T1) from S_{T1}, bit for bit.

``test_pins_catch_planted_mistakes`` plants plausible mistakes in a copy of the
oracle's C source (on the CPU) and checks that every mutant fails some pin.
"""
import os
import subprocess

import numpy as np
import pytest

import gdn2_inputs as gi
import oracle


def rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.sqrt(np.mean(np.square(b))), 1e-300))


def _small(seed=1, gates="gdn2", B=2, T=37, H=3, dk=8, dv=6, s0=0.5):
    return gi.chunk_inputs(B, T, H, dk, dv, dtype="fp32", seed=seed, s0_std=s0, gates=gates)


def pin_errors(lib=None, dk=8, dv=6):
    """Every pin's error for the oracle library ``lib`` (default build if None)."""
    err = {}
    # KDA reduction
    x = _small(seed=1, gates="kda", dk=dk, dv=dv)
    o1, S1 = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], lib=lib)
    o2, S2 = oracle.kda(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], lib=lib)
    err["kda"] = max(rel(o1, o2), rel(S1, S2))
    # Gated DeltaNet reduction
    x = _small(seed=2, gates="gdn", dk=dk, dv=dv)
    o1, S1 = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], lib=lib)
    o2, S2 = oracle.gdn(x["q"], x["k"], x["v"], x["alpha_scalar"], x["beta"], x["S0"], lib=lib)
    err["gdn"] = max(rel(o1, o2), rel(S1, S2))
    # delta-rule identity: b = 1, unit keys, q = k  =>  o_t = w_t * v_t
    x = _small(seed=3, dk=dk, dv=dv)
    ones = np.ones_like(x["b"])
    k64 = x["k"].astype(np.float64)
    k64 /= np.linalg.norm(k64, axis=-1, keepdims=True)      # unit norm in double precision
    o1, _ = oracle.gdn2(k64, k64, x["v"], x["alpha"], ones, x["w"], x["S0"], lib=lib)
    err["identity"] = rel(o1, x["w"].astype(np.float64) * x["v"])
    # b = 0 closed-form causal sum
    x = _small(seed=4, T=21, dk=dk, dv=dv)
    zero = np.zeros_like(x["b"])
    o1, _ = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], zero, x["w"], x["S0"], lib=lib)
    o2 = oracle.b0_sum(x["q"], x["k"], x["v"], x["alpha"], x["w"], x["S0"], lib=lib)
    err["b0"] = rel(o1, o2)
    # alpha = 1, b = 0, w = 1, S0 = 0: causal linear attention
    x = _small(seed=5, T=19, dk=dk, dv=dv)
    q, k, v = (x[n].astype(np.float64) for n in ("q", "k", "v"))
    o1, _ = oracle.gdn2(q, k, v, np.ones_like(x["alpha"]), zero[:, :19], np.ones_like(x["w"]), None, lib=lib)
    qh, kh, vh = (np.transpose(a, (0, 2, 1, 3)) for a in (q, k, v))   # [B,H,T,d]
    o2 = np.transpose(np.tril(qh @ np.swapaxes(kh, -1, -2)) @ vh, (0, 2, 1, 3))
    err["linear_attention"] = rel(o1, o2)
    # k = 0: pure decay of S0
    x = _small(seed=6, dk=dk, dv=dv)
    o1, S1 = oracle.gdn2(x["q"], np.zeros_like(x["k"]), x["v"], x["alpha"], x["b"], x["w"], x["S0"], lib=lib)
    decay = np.cumprod(x["alpha"].astype(np.float64), axis=1)                   # [B,T,H,dk]
    S0 = x["S0"].astype(np.float64)                                              # [B,H,dk,dv]
    o2 = np.einsum("bthi,bthi,bhij->bthj", x["q"].astype(np.float64), decay, S0)
    S2 = decay[:, -1][..., None] * S0
    err["pure_decay"] = max(rel(o1, o2), rel(S1, S2))
    # chaining: exact
    x = _small(seed=7, T=50, dk=dk, dv=dv)
    args = [x[n] for n in ("q", "k", "v", "alpha", "b", "w")]
    o, S = oracle.gdn2(*args, x["S0"], lib=lib)
    oa, Sa = oracle.gdn2(*(a[:, :23] for a in args), x["S0"], lib=lib)
    ob, Sb = oracle.gdn2(*(a[:, 23:] for a in args), Sa, lib=lib)
    err["chaining"] = max(float(np.max(np.abs(np.concatenate([oa, ob], 1) - o))), float(np.max(np.abs(Sb - S))))
    return err


TOL = {"kda": 1e-12, "gdn": 1e-12, "identity": 1e-12, "b0": 1e-12, "linear_attention": 1e-12,
       "pure_decay": 1e-12, "chaining": 0.0}


def test_oracle_pins():
    err = pin_errors()
    bad = {k: v for k, v in err.items() if not v <= TOL[k]}
    assert not bad, f"oracle pins failed: {bad}"


def test_pins_square_state():
    """Same pins with d_k = d_v (the shapes the CUDA library supports)."""
    err = pin_errors(dk=8, dv=8)
    bad = {k: v for k, v in err.items() if not v <= TOL[k]}
    assert not bad, f"oracle pins failed: {bad}"


def test_gdn2_step_is_one_token():
    x = gi.decode_inputs(2, 3, 2, 8, 8, dtype="fp32", seed=3, s0_std=0.3)
    S = x["S0"].astype(np.float64)
    for s in range(2):
        o, S_new = oracle.gdn2_step(*(x[n][s] for n in ("q", "k", "v", "alpha", "b", "w")), S)
        o2, S2 = oracle.gdn2(*(x[n][s][:, None] for n in ("q", "k", "v", "alpha", "b", "w")), S)
        assert np.array_equal(o, o2[:, 0]) and np.array_equal(S_new, S2)
        S = S_new


# Planted mistakes: (name, text in oracle_gdn2's body, replacement).  Each is a
# plausible slip in writing the recurrence; dk = dv so index swaps stay in bounds.
MUTANTS = [
    ("drop_erase_gate", "e[i] = VEC(bgate, b, t, h, i, T, H, dk) * VEC(k, b, t, h, i, T, H, dk);",
     "e[i] = VEC(k, b, t, h, i, T, H, dk);"),
    ("drop_write_gate", "z[j] = VEC(wgate, b, t, h, j, T, H, dv) * VEC(v, b, t, h, j, T, H, dv);",
     "z[j] = VEC(v, b, t, h, j, T, H, dv);"),
    ("wrong_sign", "S[(size_t)i * dv + j] += ki * (z[j] - r[j]);", "S[(size_t)i * dv + j] += ki * (z[j] + r[j]);"),
    ("decay_on_value_axis", "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a;",
     "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= VEC(alpha, b, t, h, j, T, H, dk);"),
    ("read_before_decay", "for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * e[i];",
     "for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * e[i] / VEC(alpha, b, t, h, i, T, H, dk);"),
    ("transposed_read", "for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * e[i];",
     "for (int i = 0; i < dk; ++i) acc += S[(size_t)j * dv + i] * e[i];"),
    ("output_reads_old_state",
     "for (int i = 0; i < dk; ++i) acc += S[(size_t)i * dv + j] * VEC(q, b, t, h, i, T, H, dk);",
     "for (int i = 0; i < dk; ++i) acc += (S[(size_t)i * dv + j] - VEC(k, b, t, h, i, T, H, dk) * (z[j] - r[j]))"
     " * VEC(q, b, t, h, i, T, H, dk);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistakes(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")).read()
    body_start = src.index("void oracle_gdn2(")
    body_end = src.index("static void transition_step(")
    body = src[body_start:body_end]
    assert body.count(old) == 1, f"mutation site for {name} not unique"
    mutated = src[:body_start] + body.replace(old, new) + src[body_end:]
    c = tmp_path / "mutant.c"
    c.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c), "-lm"])
    lib = oracle._bind(str(so))
    err = pin_errors(lib=lib, dk=8, dv=8)
    caught = {k: v for k, v in err.items() if not v <= TOL[k]}
    assert caught, f"mutant {name} passed every pin: {err}"
