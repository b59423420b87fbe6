"""FP64 CPU oracle for the Gated DeltaNet-2 recurrence (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``gated_delta_rule_111_b200``) never imports it and has no CPU fallback.

The arithmetic lives in ``gdn2_oracle.c`` (plain C, double precision, token by
token, OpenMP over (batch, head)); this module only marshals numpy arrays.  Each
function cites the passage of "Gated DeltaNet-2: Decoupling Erase and Write in
Linear Attention" (iplexlaw.co.kr analysis) that it follows.

Pins (what ties this oracle to something other than itself) are in
``tests/test_oracle.py``: the KDA and Gated DeltaNet reductions against
separately coded transition-matrix recurrences, the delta-rule identity
S_t^T k_t = z_t for b = 1 and unit keys, the b = 0 closed-form causal sum,
the k = 0 pure-decay closed form, and state chaining.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
_LIB = os.path.join(_HERE, "_build", "liboracle_gdn2.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP, no fast-math) if stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path):
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    i = ctypes.c_int
    lib.oracle_gdn2.argtypes = [i] * 5 + [dp] * 9
    lib.oracle_kda.argtypes = [i] * 5 + [dp] * 8
    lib.oracle_gdn.argtypes = [i] * 5 + [dp] * 8
    lib.oracle_b0_sum.argtypes = [i] * 5 + [dp] * 7
    lib.oracle_gdn2_bwd.argtypes = [i] * 5 + [dp] * 16
    lib.oracle_gdn2_prep.argtypes = [ctypes.c_longlong, i, i] + [dp] * 12
    lib.oracle_output_gate.argtypes = [ctypes.c_longlong, i, dp, dp, dp, ctypes.c_double, dp]
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _load(lib=None):
    """The default oracle library, or ``lib`` (a CDLL from :func:`_bind`) if given."""
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = _bind(build())
    return _lib


def _f64(x):
    return None if x is None else np.ascontiguousarray(x, dtype=np.float64)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    """OpenMP threads the oracle runs on (set OMP_NUM_THREADS to change)."""
    return int(_load().oracle_num_threads())


def _dims(q, v):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    return B, T, H, dk, dv


def gdn2(q, k, v, alpha, b, w, S0=None, *, lib=None):
    """GDN-2 recurrence, token by token ("Independent decisions on two axes").

    Per head and token: Sbar = diag(alpha_t) S_{t-1}; e = b_t*k_t; z = w_t*v_t;
    r = Sbar^T e; S_t = Sbar + k_t (z - r)^T; o_t = S_t^T q_t.
    Inputs [B,T,H,d] (any float dtype, upcast exactly to float64); S0 [B,H,dk,dv]
    or None for zeros.  Returns (o [B,T,H,dv], S_T [B,H,dk,dv]) in float64.
    """
    q, k, v, alpha, b, w, S0 = map(_f64, (q, k, v, alpha, b, w, S0))
    B, T, H, dk, dv = _dims(q, v)
    o = np.empty((B, T, H, dv))
    ST = np.empty((B, H, dk, dv))
    _load(lib).oracle_gdn2(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                        _ptr(S0), _ptr(o), _ptr(ST))
    return o, ST


def gdn2_step(q, k, v, alpha, b, w, S):
    """One decode step of the same recurrence (the T = 1 case of :func:`gdn2`).

    q,k,v,alpha,b,w are [B,H,d]; S is [B,H,dk,dv].  Returns (o [B,H,dv], S_new).
    """
    o, ST = gdn2(*(np.asarray(x)[:, None] for x in (q, k, v, alpha, b, w)), S0=S)
    return o[:, 0], ST


def kda(q, k, v, alpha, beta, S0=None, *, lib=None):
    """Kimi Delta Attention in transition-matrix form.

    S_t = (I - beta_t k_t k_t^T) diag(alpha_t) S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t
    ("From a growing cache to a fixed state"; tying both GDN-2 gates to one
    scalar beta recovers it, "Independent decisions on two axes").
    alpha [B,T,H,dk], beta [B,T,H].
    """
    q, k, v, alpha, beta, S0 = map(_f64, (q, k, v, alpha, beta, S0))
    B, T, H, dk, dv = _dims(q, v)
    o = np.empty((B, T, H, dv))
    ST = np.empty((B, H, dk, dv))
    _load(lib).oracle_kda(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                       _ptr(S0), _ptr(o), _ptr(ST))
    return o, ST


def gdn(q, k, v, alpha, beta, S0=None, *, lib=None):
    """Gated DeltaNet in transition-matrix form.

    S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, o_t = S_t^T q_t
    (scalar decay; "Independent decisions on two axes").  alpha, beta [B,T,H].
    """
    q, k, v, alpha, beta, S0 = map(_f64, (q, k, v, alpha, beta, S0))
    B, T, H, dk, dv = _dims(q, v)
    o = np.empty((B, T, H, dv))
    ST = np.empty((B, H, dk, dv))
    _load(lib).oracle_gdn(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                       _ptr(S0), _ptr(o), _ptr(ST))
    return o, ST


def b0_sum(q, k, v, alpha, w, S0=None, *, lib=None):
    """Explicit O(T^2) causal sum for the b = 0 case (no erase).

    o_t = sum_{s<=t} (sum_i q_t[i] k_s[i] prod_{m=s+1..t} alpha_m[i]) (w_s*v_s)
          + (diag(prod_{m<=t} alpha_m) S0)^T q_t.
    """
    q, k, v, alpha, w, S0 = map(_f64, (q, k, v, alpha, w, S0))
    B, T, H, dk, dv = _dims(q, v)
    o = np.empty((B, T, H, dv))
    _load(lib).oracle_b0_sum(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(w),
                          _ptr(S0), _ptr(o))
    return o


def gdn2_bwd(q, k, v, alpha, b, w, S0=None, dO=None, dST=None, *, lib=None):
    """Gradients of L = sum(dO * o) + sum(dST * S_T) for the recurrence of :func:`gdn2`,
    by reverse mode through the same token loop (the gate-aware backward pass the
    "Token processing and parallel training" section calls for: channel-wise decay
    and separate erase / write gates each get their own gradient).  dO [B,T,H,dv]
    (None = zeros), dST [B,H,dk,dv] (None = zeros).  Returns a dict of float64
    arrays dq, dk, dv, dalpha, db, dw, dS0.  Keeps every forward state: T x dk x dv
    doubles per head, so meant for test-sized inputs."""
    q, k, v, alpha, b, w, S0, dO, dST = map(_f64, (q, k, v, alpha, b, w, S0, dO, dST))
    B, T, H, dk, dv = _dims(q, v)
    if dO is None:
        dO = np.zeros((B, T, H, dv))
    out = {n: np.empty_like(x) for n, x in (("dq", q), ("dk", k), ("dv", v), ("dalpha", alpha), ("db", b), ("dw", w))}
    out["dS0"] = np.empty((B, H, dk, dv))
    _load(lib).oracle_gdn2_bwd(B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w),
                               _ptr(S0), _ptr(dO), _ptr(dST), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                               _ptr(out["dalpha"]), _ptr(out["db"]), _ptr(out["dw"]), _ptr(out["dS0"]))
    return out


def gdn2_prep(xq, xk, xv, xa, xb, xw, *, lib=None):
    """The recurrence's inputs from pre-activation logits (per token and head):
    q, k = L2-normalised SiLU of xq, xk; v = SiLU(xv); alpha = exp(-softplus(xa));
    b, w = sigmoid(xb), sigmoid(xw) -- the query/key/value paths of "Token processing
    and parallel training" and the sigmoid gates of "Independent decisions on two axes"
    (alpha's parameterisation is this package's reading: the pages leave it open).
    Inputs [..., d] (any leading shape, channels last); returns a dict of float64 arrays
    q, k, v, alpha, b, w of the same shapes."""
    xq, xk, xv, xa, xb, xw = map(_f64, (xq, xk, xv, xa, xb, xw))
    dk, dv = xq.shape[-1], xv.shape[-1]
    rows = xq.size // dk
    out = {n: np.empty_like(x) for n, x in (("q", xq), ("k", xk), ("v", xv), ("alpha", xa), ("b", xb), ("w", xw))}
    _load(lib).oracle_gdn2_prep(rows, dk, dv, _ptr(xq), _ptr(xk), _ptr(xv), _ptr(xa), _ptr(xb), _ptr(xw),
                                _ptr(out["q"]), _ptr(out["k"]), _ptr(out["v"]), _ptr(out["alpha"]), _ptr(out["b"]),
                                _ptr(out["w"]))
    return out


def gdn2_from_logits(xq, xk, xv, xa, xb, xw, S0=None, *, lib=None):
    """:func:`gdn2` applied to :func:`gdn2_prep` of the logits ([B,T,H,d] each)."""
    x = gdn2_prep(xq, xk, xv, xa, xb, xw, lib=lib)
    return gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"], S0, lib=lib)


def output_gate(o, g, weight, eps=1e-6, *, lib=None):
    """Output epilogue of "Token processing and parallel training" (RMS norm, then a
    separate output gate): per row of the last axis, y = o / sqrt(mean(o^2) + eps) * weight
    * sigmoid(g).  The norm's per-channel weight, the epsilon and the sigmoid form of the
    gate are this package's readings.  o, g [..., dv]; weight [dv].  Returns float64."""
    o, g, weight = map(_f64, (o, g, weight))
    dv = o.shape[-1]
    y = np.empty_like(o)
    _load(lib).oracle_output_gate(o.size // dv, dv, _ptr(o), _ptr(g), _ptr(weight), float(eps), _ptr(y))
    return y
