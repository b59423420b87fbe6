"""Pins of the oracle's output epilogue (oracle_output_gate: RMS norm over a head's
d_v channels with a per-channel weight and epsilon, then a sigmoid output gate;
"Token processing and parallel training").  Each pin ties it to a closed form,
an invariance, a limit or a hand value; planted mistakes must fail one of them.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle


def pin_errors(lib=None):
    rng = np.random.default_rng(3)
    o = rng.standard_normal((4, 5, 16)) * rng.uniform(0.1, 10.0, (4, 5, 1))
    g = rng.standard_normal((4, 5, 16)) * 3.0
    w = rng.uniform(0.5, 1.5, 16)
    err = {}
    # gate wide open (g -> +inf), unit weight, eps = 0: every row has RMS exactly 1
    y = oracle.output_gate(o, np.full_like(o, 800.0), np.ones(16), 0.0, lib=lib)
    err["unit_rms"] = float(np.max(np.abs(np.sqrt(np.mean(y ** 2, axis=-1)) - 1.0)))
    # eps = 0: invariant to scaling the row by c > 0
    y1 = oracle.output_gate(o, g, w, 0.0, lib=lib)
    y2 = oracle.output_gate(7.5 * o, g, w, 0.0, lib=lib)
    err["scale_invariance"] = float(np.max(np.abs(y1 - y2)))
    # the gate multiplies channel by channel: y(g) / y(g') = sigmoid(g) / sigmoid(g')
    y3 = oracle.output_gate(o, -g, w, 1e-3, lib=lib)
    y4 = oracle.output_gate(o, g, w, 1e-3, lib=lib)
    ratio = np.where(np.abs(y3) > 1e-12, y4 / np.where(np.abs(y3) > 1e-12, y3, 1.0), np.exp(g))
    err["gate_ratio"] = float(np.max(np.abs(ratio / np.exp(g) - 1.0)))
    # weight enters linearly, per channel
    y5 = oracle.output_gate(o, g, 2.0 * w, 1e-3, lib=lib)
    err["weight_linear"] = float(np.max(np.abs(y5 - 2.0 * y4)))
    # eps: a row of equal values c gives c / sqrt(c^2 + eps) (times the gate and weight)
    row = np.full((1, 16), 0.3)
    y6 = oracle.output_gate(row, np.full_like(row, 800.0), np.ones(16), 0.01, lib=lib)
    err["eps"] = float(np.max(np.abs(y6 - 0.3 / math.sqrt(0.09 + 0.01))))
    return err


TOL = {"unit_rms": 1e-14, "scale_invariance": 1e-14, "gate_ratio": 1e-12, "weight_linear": 1e-15, "eps": 1e-15}


def test_output_gate_pins():
    err = pin_errors()
    bad = {k: v for k, v in err.items() if not v <= TOL[k]}
    assert not bad, f"output gate pins failed: {bad}"


def test_output_gate_hand_values():
    """o = (3, 4): RMS = sqrt(12.5); g = 0 halves; weight (1, 2)."""
    y = oracle.output_gate(np.array([[3.0, 4.0]]), np.zeros((1, 2)), np.array([1.0, 2.0]), 0.0)
    r = math.sqrt(12.5)
    assert y[0, 0] == pytest.approx(0.5 * 3.0 / r, abs=1e-15)
    assert y[0, 1] == pytest.approx(0.5 * 2.0 * 4.0 / r, abs=1e-15)


MUTANTS = [
    ("sum_not_mean", "ms /= dv;", "ms /= 1;"),
    ("no_sqrt", "const double inv = 1.0 / sqrt(ms + eps);", "const double inv = 1.0 / (ms + eps);"),
    ("gate_sign", "/ (1.0 + exp(-grow[j]))", "/ (1.0 + exp(grow[j]))"),
    ("eps_outside", "const double inv = 1.0 / sqrt(ms + eps);", "const double inv = 1.0 / sqrt(ms) + eps;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistakes(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "gdn2_oracle.c")).read()
    start = src.index("void oracle_output_gate(")
    body = src[start:]
    assert body.count(old) == 1, f"mutation site for {name} not unique"
    c = tmp_path / "mutant.c"
    c.write_text(src[:start] + body.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", str(so), str(c), "-lm"])
    err = pin_errors(lib=oracle._bind(str(so)))
    caught = {k: v for k, v in err.items() if not v <= TOL[k]}
    assert caught, f"mutant {name} passed every pin: {err}"
