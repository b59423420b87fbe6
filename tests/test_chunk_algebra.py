"""The chunkwise algebra the CUDA kernels implement, checked in FP64 against the
token-by-token oracle (CPU only).

"Token processing and parallel training" (Gated DeltaNet-2 analysis) outlines
the parallel form only: 64-token blocks whose accumulated per-channel decay is
folded into the erase-side and key-side factors, so that each block needs one
unit-triangular system and matrix products.  Our re-derivation, per chunk of n
tokens starting from state S:

  gamma_t = prod_{j<=t} alpha_j  (per key channel),   rho_t = 1 / gamma_t
  Etil = e * gamma,  Qtil = q * gamma,  Ktil = k * rho        (e = b*k, z = w*v)
  A = strict_tril(Etil Ktil^T),  P = tril(Qtil Ktil^T)
  U = (I + A)^{-1} (Z - Etil S)      -- the per-token corrections z_t - r_t
  O = Qtil S + P U
  S <- diag(gamma_n) (S + Ktil^T U)

Chunking is an exact re-association of the token recurrence ("identical
mathematics" of the two modes), so this must match the oracle to rounding.
"""
import numpy as np
import pytest

import gdn2_inputs as gi
import oracle


def chunk_model(q, k, v, alpha, b, w, S0, C=64, form="factored"):
    """FP64 chunkwise forward for one (batch, head): inputs [T, d], S0 [dk, dv]."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.astype(np.float64).copy()
    o = np.zeros((T, dv))
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        qc, kc, vc, ac, bc, wc = (x[sl].astype(np.float64) for x in (q, k, v, alpha, b, w))
        n = qc.shape[0]
        e, z = bc * kc, wc * vc
        if form == "factored":
            gamma = np.cumprod(ac, axis=0)
            rho = np.cumprod(1.0 / ac, axis=0)
            Et, Qt, Kt = e * gamma, qc * gamma, kc * rho
            A = np.tril(Et @ Kt.T, -1)
            P = np.tril(Qt @ Kt.T)
            U = np.linalg.solve(np.eye(n) + A, z - Et @ S)
            o[sl] = Qt @ S + P @ U
            S = gamma[-1][:, None] * (S + Kt.T @ U)
        else:  # difference-of-logs form used by the FP32 CUDA-core kernel
            g = np.cumsum(np.log(ac), axis=0)
            D = np.exp(g[:, None, :] - g[None, :, :])           # [t, s, i] decay ratio, used for s <= t
            mask = np.tril(np.ones((n, n)), -1)
            A = np.einsum("ti,si,tsi->ts", e, kc, D) * mask
            P = np.einsum("ti,si,tsi->ts", qc, kc, D) * (mask + np.eye(n))
            Et, Qt = e * np.exp(g), qc * np.exp(g)
            Kh = kc * np.exp(g[-1][None, :] - g)
            U = np.linalg.solve(np.eye(n) + A, z - Et @ S)
            o[sl] = Qt @ S + P @ U
            S = np.exp(g[-1])[:, None] * S + Kh.T @ U
    return o, S


@pytest.mark.parametrize("form", ["factored", "logdiff"])
@pytest.mark.parametrize("T,C", [(150, 64), (64, 64), (1, 64), (65, 64), (37, 16)])
def test_chunk_algebra_matches_token_recurrence(form, T, C):
    x = gi.chunk_inputs(1, T, 2, 16, 12, dtype="fp32", seed=11, s0_std=0.3)
    o_ref, S_ref = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], x["S0"])
    for h in range(2):
        args = [x[n][0, :, h] for n in ("q", "k", "v", "alpha", "b", "w")]
        o, S = chunk_model(*args, x["S0"][0, h], C=C, form=form)
        scale = np.sqrt(np.mean(o_ref[0, :, h] ** 2))
        assert np.max(np.abs(o - o_ref[0, :, h])) <= 1e-12 * scale
        assert np.max(np.abs(S - S_ref[0, h])) <= 1e-12 * np.sqrt(np.mean(S_ref[0, h] ** 2))


def test_chunk_algebra_gdn2_specific_gates():
    """Erase gate above 1 (the pages ablate b in [0, 2]) and a write gate that differs from it."""
    x = gi.chunk_inputs(1, 100, 1, 8, 8, dtype="fp32", seed=5, s0_std=0.5)
    b2 = 2.0 * x["b"]
    o_ref, S_ref = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], b2, x["w"], x["S0"])
    args = [x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0], x["alpha"][0, :, 0], b2[0, :, 0], x["w"][0, :, 0]]
    o, S = chunk_model(*args, x["S0"][0, 0])
    assert np.max(np.abs(o - o_ref[0, :, 0])) <= 1e-11 * np.sqrt(np.mean(o_ref ** 2))
    assert np.max(np.abs(S - S_ref[0, 0])) <= 1e-11 * np.sqrt(np.mean(S_ref ** 2))


def chunk_bwd_model(q, k, v, alpha, b, w, S0, dO, dST, C=64):
    """FP64 chunkwise backward for one (batch, head), the algebra of the CUDA backward.

    Per chunk with start state S, from the forward quantities (factored form)
      U = (I + A)^{-1} (Z - Etil S),  O = Qtil S + P U,  S' = diag(gamma_n) S + Khat^T U,
    and the gradients dO of the chunk's outputs and dS' of its end state:
      dU = P^T dO + Khat dS';  dR = T^T dU  (T = (I + A)^{-1});  dA = -dR U^T (strict);
      dP = dO U^T (lower);  dS = Qtil^T dO + diag(gamma_n) dS' - Etil^T dR;
      dq = gamma (S dO + dP Ktil),  de = gamma (-S dR + dA Ktil),
      dk_key = (dA^T Etil + dP^T Qtil) / gamma + (U dS'^T) gamma_n / gamma,
      db = de k,  dk = dk_key + de b,  dw = dR v,  dv = dR w,
      dlog gamma = de e + dq q - dk_key k  (+ at the last token: gamma_n rowsum(S dS')
                   + sum_s Khat_s (U dS'^T)_s),
      dalpha = (reverse cumulative sum of dlog gamma) / alpha."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else S0.astype(np.float64).copy()
    starts = []
    for c0 in range(0, T, C):                       # forward: the chunk start states
        sl = slice(c0, min(T, c0 + C))
        starts.append(S.copy())
        qc, kc, vc, ac, bc, wc = (x[sl].astype(np.float64) for x in (q, k, v, alpha, b, w))
        n = qc.shape[0]
        gam = np.cumprod(ac, axis=0)
        Et, Kt = bc * kc * gam, kc / gam
        A = np.tril(Et @ Kt.T, -1)
        U = np.linalg.solve(np.eye(n) + A, wc * vc - Et @ S)
        S = gam[-1][:, None] * (S + Kt.T @ U)
    grads = {n_: np.zeros_like(x, dtype=np.float64) for n_, x in (("dq", q), ("dk", k), ("dv", v), ("dalpha", alpha),
                                                                  ("db", b), ("dw", w))}
    dS = np.zeros((dk, dv)) if dST is None else dST.astype(np.float64).copy()
    for ci, c0 in reversed(list(enumerate(range(0, T, C)))):
        sl = slice(c0, min(T, c0 + C))
        S = starts[ci]
        qc, kc, vc, ac, bc, wc, dOc = (x[sl].astype(np.float64) for x in (q, k, v, alpha, b, w, dO))
        n = qc.shape[0]
        gam = np.cumprod(ac, axis=0)
        gn = gam[-1]
        e, z = bc * kc, wc * vc
        Et, Qt, Kt, Kh = e * gam, qc * gam, kc / gam, kc * gn / gam
        A = np.tril(Et @ Kt.T, -1)
        P = np.tril(Qt @ Kt.T)
        Tm = np.linalg.inv(np.eye(n) + A)
        R = z - Et @ S
        U = Tm @ R
        dU = P.T @ dOc + Kh @ dS
        dR = Tm.T @ dU
        dA = np.tril(-dR @ U.T, -1)
        dP = np.tril(dOc @ U.T)
        dS_prev = Qt.T @ dOc + gn[:, None] * dS - Et.T @ dR
        dq = gam * (dOc @ S.T + dP @ Kt)
        de = gam * (-dR @ S.T + dA @ Kt)
        dKh = U @ dS.T
        dk_key = (dA.T @ Et + dP.T @ Qt) / gam + dKh * gn / gam
        dlg = de * e + dq * qc - dk_key * kc
        dlg[-1] += gn * np.sum(S * dS, axis=1) + np.sum(Kh * dKh, axis=0)
        grads["dq"][sl] = dq
        grads["db"][sl] = de * kc
        grads["dk"][sl] = dk_key + de * bc
        grads["dw"][sl] = dR * vc
        grads["dv"][sl] = dR * wc
        grads["dalpha"][sl] = np.cumsum(dlg[::-1], axis=0)[::-1] / ac
        dS = dS_prev
    grads["dS0"] = dS
    return grads


@pytest.mark.parametrize("T", [1, 64, 150])
def test_chunk_backward_algebra_matches_oracle_gradient(T):
    """The chunkwise backward (several chunks, ragged last chunk, S0 != 0, erase gate up to 2)
    equals the oracle's token-loop gradient to FP64 rounding."""
    x = gi.chunk_inputs(1, T, 2, 16, 8, dtype="fp32", seed=T, s0_std=0.2)
    rng = np.random.default_rng(T + 1)
    dO = rng.standard_normal((1, T, 2, 8))
    dST = rng.standard_normal((1, 2, 16, 8))
    b2 = 2.0 * x["b"]
    ref = oracle.gdn2_bwd(x["q"], x["k"], x["v"], x["alpha"], b2, x["w"], x["S0"], dO, dST)
    for h in range(2):
        args = [x[n][0, :, h] for n in ("q", "k", "v", "alpha")] + [b2[0, :, h], x["w"][0, :, h]]
        g = chunk_bwd_model(*args, x["S0"][0, h], dO[0, :, h], dST[0, h], C=64)
        for name in ("dq", "dk", "dv", "dalpha", "db", "dw"):
            r = ref[name][0, :, h]
            assert np.max(np.abs(g[name] - r)) <= 1e-9 * max(1.0, np.max(np.abs(r))), (name, h)
        assert np.max(np.abs(g["dS0"] - ref["dS0"][0, h])) <= 1e-9 * max(1.0, np.max(np.abs(ref["dS0"])))
