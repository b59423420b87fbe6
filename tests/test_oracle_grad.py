"""Pins of the oracle gradient (oracle.gdn2_bwd) to something other than itself:
central finite differences of the forward oracle, in FP64 (CPU).

L = sum(dO * o) + sum(dST * S_T).  For every input X and a random direction D,
(L(X + eps D) - L(X - eps D)) / (2 eps) must equal sum(dL/dX * D); with eps = 1e-5
the truncation error is ~1e-10 of the slope.  Non-square heads (dk != dv) catch
transposed operands; gates away from 0 and 1 keep every term alive; a planted
mistake in a copy of the backward (a dropped decay factor) must fail the check."""
import numpy as np
import pytest

import gdn2_inputs as gi
import oracle


def _inputs(B=2, T=11, H=2, dk=5, dv=3, seed=0):
    x = gi.chunk_inputs(B, T, H, dk, dv, dtype="fp32", seed=seed, s0_std=0.3)
    rng = np.random.default_rng(seed + 100)
    x = {n: x[n].astype(np.float64) for n in ("q", "k", "v", "alpha", "b", "w", "S0")}
    x["b"] = 2.0 * x["b"]                       # erase gate over (0, 2)
    dO = rng.standard_normal((B, T, H, dv))
    dST = rng.standard_normal((B, H, dk, dv))
    return x, dO, dST


def _loss(x, dO, dST):
    o, S = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
    return float(np.sum(o * dO) + np.sum(S * dST))


NAMES = {"q": "dq", "k": "dk", "v": "dv", "alpha": "dalpha", "b": "db", "w": "dw", "S0": "dS0"}


@pytest.mark.parametrize("name", list(NAMES))
def test_gradient_matches_finite_differences(name):
    x, dO, dST = _inputs()
    g = oracle.gdn2_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], dO, dST)
    rng = np.random.default_rng(hash(name) % 1000)
    for _ in range(3):
        D = rng.standard_normal(x[name].shape)
        eps = 1e-5
        xp = dict(x); xp[name] = x[name] + eps * D
        xm = dict(x); xm[name] = x[name] - eps * D
        fd = (_loss(xp, dO, dST) - _loss(xm, dO, dST)) / (2 * eps)
        an = float(np.sum(g[NAMES[name]] * D))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (name, fd, an)


def test_single_elements_match():
    """A few individual entries (first and last token, first and last channel)."""
    x, dO, dST = _inputs(B=1, T=7, H=1, dk=4, dv=3, seed=3)
    g = oracle.gdn2_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], dO, dST)
    eps = 1e-6
    for name, idx in (("alpha", (0, 0, 0, 0)), ("alpha", (0, 6, 0, 3)), ("k", (0, 3, 0, 2)), ("b", (0, 6, 0, 1)),
                      ("w", (0, 0, 0, 2)), ("q", (0, 5, 0, 0)), ("S0", (0, 0, 3, 1))):
        xp = dict(x); xp[name] = x[name].copy(); xp[name][idx] += eps
        xm = dict(x); xm[name] = x[name].copy(); xm[name][idx] -= eps
        fd = (_loss(xp, dO, dST) - _loss(xm, dO, dST)) / (2 * eps)
        assert abs(fd - g[NAMES[name]][idx]) <= 1e-6 * max(1.0, abs(fd)), (name, idx)


def test_zero_upstream_gives_zero_gradient():
    x, dO, dST = _inputs(B=1, T=5, H=1)
    g = oracle.gdn2_bwd(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"], 0 * dO, 0 * dST)
    assert all(np.all(v == 0) for v in g.values())


def test_planted_mistake_is_caught():
    """The check fails for a gradient that forgets the decay in the state carry (dS_{t-1} =
    dSbar instead of diag(alpha_t) dSbar): emulated by asking the oracle for the gradient
    of a run with alpha = 1 and comparing with finite differences of the true alpha."""
    x, dO, dST = _inputs(B=1, T=9, H=1, dk=4, dv=3, seed=5)
    wrong = dict(x); wrong["alpha"] = np.ones_like(x["alpha"])
    g = oracle.gdn2_bwd(wrong["q"], wrong["k"], wrong["v"], wrong["alpha"], wrong["b"], wrong["w"], wrong["S0"],
                        dO, dST)
    D = np.random.default_rng(0).standard_normal(x["S0"].shape)
    eps = 1e-5
    xp = dict(x); xp["S0"] = x["S0"] + eps * D
    xm = dict(x); xm["S0"] = x["S0"] - eps * D
    fd = (_loss(xp, dO, dST) - _loss(xm, dO, dST)) / (2 * eps)
    assert abs(fd - float(np.sum(g["dS0"] * D))) > 1e-3 * max(1.0, abs(fd))
