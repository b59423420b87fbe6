"""Pins of the oracle's input preparation (oracle_gdn2_prep): the activations that
turn pre-activation logits into q, k, v, alpha, b, w ("Token processing and
parallel training": SiLU then L2 normalisation on the query and key paths, SiLU
on the value path; "Independent decisions on two axes": sigmoid gates b and w;
alpha = exp(-softplus), this package's reading of the unparameterised decay).

Each pin checks the oracle against a different formula for the same function
(tanh forms of the sigmoid, the closed form 1 / (1 + e^x) of exp(-softplus(x)),
norms from numpy), limits, or hand-checked values; planted mistakes in the C
source must each fail one of them.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle


def _tanh_sigmoid(x):
    return 0.5 * (1.0 + np.tanh(0.5 * x))


def _logits(shape, seed, scale=3.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def pin_errors(lib=None):
    """Largest deviation of each prepared tensor from its independent form."""
    d = 16
    xq, xk, xv, xa, xb, xw = (_logits((3, 5, 2, d), s) for s in range(6))
    xq[0, 0, 0] = 0.0                                  # a zero row: its SiLU is zero, so is q
    xa[0, 0, 0, :4] = [40.0, -20.0, 0.0, 15.0]         # far tails of the decay
    out = oracle.gdn2_prep(xq, xk, xv, xa, xb, xw, lib=lib)
    err = {}
    for name, x in (("q", xq), ("k", xk)):
        s = x * _tanh_sigmoid(x)
        n = np.linalg.norm(s, axis=-1, keepdims=True)
        ref = np.where(n > 0, s / np.where(n > 0, n, 1.0), 0.0)
        err[name] = float(np.max(np.abs(out[name] - ref)))
        norms = np.linalg.norm(out[name], axis=-1)
        nz = np.linalg.norm(s, axis=-1) > 0
        err[name + "_unit"] = float(np.max(np.abs(norms[nz] - 1.0)))
    err["q_zero_row"] = float(np.max(np.abs(out["q"][0, 0, 0])))
    err["v"] = float(np.max(np.abs(out["v"] - xv * _tanh_sigmoid(xv))))
    # exp(-softplus(x)) = 1 / (1 + e^x), written without overflow as e^-x / (1 + e^-x) for x > 0
    en = np.exp(-np.abs(xa))
    ref_a = np.where(xa > 0, en / (1.0 + en), 1.0 / (1.0 + en))
    err["alpha"] = float(np.max(np.abs(out["alpha"] - ref_a) / np.maximum(ref_a, 1e-300)))
    err["alpha_tail"] = abs(out["alpha"][0, 0, 0, 0] / math.exp(-40.0) - 1.0)
    err["alpha_one"] = abs((1.0 - out["alpha"][0, 0, 0, 1]) / (math.exp(-20.0) / (1.0 + math.exp(-20.0))) - 1.0)
    err["alpha_half"] = abs(out["alpha"][0, 0, 0, 2] - 0.5)
    err["b"] = float(np.max(np.abs(out["b"] - _tanh_sigmoid(xb))))
    err["w"] = float(np.max(np.abs(out["w"] - _tanh_sigmoid(xw))))
    return err


TOL = {"q": 1e-14, "k": 1e-14, "q_unit": 1e-14, "k_unit": 1e-14, "q_zero_row": 0.0, "v": 1e-13,
       "alpha": 1e-12, "alpha_tail": 1e-10, "alpha_one": 1e-6, "alpha_half": 1e-15, "b": 1e-15, "w": 1e-15}


def test_prep_pins():
    err = pin_errors()
    bad = {k: v for k, v in err.items() if not v <= TOL[k]}
    assert not bad, f"prep pins failed: {bad}"


def test_prep_hand_values():
    """SiLU(1) = 1 / (1 + e^-1) = 0.7310585786300049; SiLU(-1) = -0.2689414213699951;
    the row (1, -1) after SiLU and the norm; sigmoid(0) = 1/2; exp(-softplus(ln 3)) = 1/4."""
    x1 = np.array([[1.0, -1.0]])
    out = oracle.gdn2_prep(x1, x1, x1, np.array([[math.log(3.0), 0.0]]), np.zeros((1, 2)), np.zeros((1, 2)))
    assert out["v"][0, 0] == pytest.approx(0.7310585786300049, abs=1e-15)
    assert out["v"][0, 1] == pytest.approx(-0.2689414213699951, abs=1e-15)
    n = math.hypot(0.7310585786300049, 0.2689414213699951)
    assert out["q"][0, 0] == pytest.approx(0.7310585786300049 / n, abs=1e-15)
    assert out["alpha"][0, 0] == pytest.approx(0.25, abs=1e-15)
    assert out["b"][0, 0] == 0.5 and out["w"][0, 1] == 0.5


def test_logit_path_composes_prep_and_recurrence():
    """gdn2_from_logits is the recurrence on the prepared inputs (not a separate formula)."""
    xs = [_logits((1, 9, 2, 8), 10 + s, scale=1.0) for s in range(6)]
    o1, S1 = oracle.gdn2_from_logits(*xs)
    p = oracle.gdn2_prep(*xs)
    o2, S2 = oracle.gdn2(p["q"], p["k"], p["v"], p["alpha"], p["b"], p["w"])
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


# Planted mistakes in oracle_gdn2_prep and its helpers: each must fail a pin.
MUTANTS = [
    ("no_silu_before_norm", "y[i] = x[i] * prep_sigmoid(x[i]);", "y[i] = x[i];"),
    ("norm_by_square", "const double inv = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;",
     "const double inv = ss > 0.0 ? 1.0 / ss : 0.0;"),
    ("alpha_is_softplus", "alpha[ok + i] = exp(-prep_softplus(xa[ok + i]));",
     "alpha[ok + i] = prep_softplus(xa[ok + i]);"),
    ("alpha_sign", "alpha[ok + i] = exp(-prep_softplus(xa[ok + i]));",
     "alpha[ok + i] = exp(-prep_softplus(-xa[ok + i]));"),
    ("gate_sign", "b[ok + i] = prep_sigmoid(xb[ok + i]);", "b[ok + i] = prep_sigmoid(-xb[ok + i]);"),
    ("v_not_silu", "v[ov + j] = xv[ov + j] * prep_sigmoid(xv[ov + j]);", "v[ov + j] = prep_sigmoid(xv[ov + j]);"),
    ("softplus_branch", "x > 0 ? x + log1p(exp(-x)) : log1p(exp(x))", "x > 0 ? log1p(exp(-x)) : log1p(exp(x))"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistakes(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")).read()
    start = src.index("static double prep_sigmoid(")
    body = src[start:]
    assert body.count(old) == 1, f"mutation site for {name} not unique"
    mutated = src[:start] + body.replace(old, new)
    c = tmp_path / "mutant.c"
    c.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c), "-lm"])
    err = pin_errors(lib=oracle._bind(str(so)))
    caught = {k: v for k, v in err.items() if not v <= TOL[k]}
    assert caught, f"mutant {name} passed every pin: {err}"
