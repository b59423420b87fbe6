"""Python binding of libgdn2, the B200 (sm_100a) Gated DeltaNet-2 recurrence.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libgdn2.so`` behind the C ABI declared in ``include/gdn2.h``.  There
is no CPU implementation and no fallback; without the compiled library or a CUDA
device these functions raise.

Functions (same names as the C ABI):
  gdn2_chunk_fwd(q, k, v, alpha, b, w, S0=None, ...)  -> (o, S_T)   chunkwise prefill
  gdn2_chunk_fwd_from_host(q, k, v, alpha, b, w, S0=None, ...)
                                                      -> (o, S_T)   the same from pinned host tensors, streamed
  gdn2_chunk_fwd_varlen(q, k, v, alpha, b, w, cu_seqlens, S0=None, ...)
                                                      -> (o, S_T)   packed variable-length batch
  gdn2_chunk_fwd_segmented(q, k, v, alpha, b, w, S0=None, segments=0, ...)
                                                      -> (o, S_T)   segment-parallel prefill (long sequences)
  gdn2_chunk_fwd_segmented_workspace_size(B, T, H, dk, dv, segments) -> bytes
  gdn2_chunk_fwd_segments(B, T, H, dk, dv, segments)  -> int        segments that call would use
  gdn2_chunk_fwd_logits(xq, xk, xv, xa, xb, xw, S0=None, ...) -> (o, S_T)  prefill from BF16 logits
  gdn2_recurrent_step(q, k, v, alpha, b, w, S, ...)   -> o          in-place decode step
  gdn2_output_gate(o, g, weight, eps, ...)            -> y          RMS norm + sigmoid output gate
  gdn2_chunk_bwd(q, k, v, alpha, b, w, S0, dO, dST, ...) -> dict    gradients of every input
  gdn2_chunk_bwd_workspace_size(B, T, H, dk, dv)      -> bytes      workspace of gdn2_chunk_bwd
  gdn2_chunk_bwd_noalloc(..., out)                    -> dict       the same, workspace inside the library
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

__all__ = ["gdn2_chunk_fwd", "gdn2_chunk_fwd_from_host", "gdn2_chunk_fwd_varlen", "gdn2_chunk_fwd_segmented", "gdn2_chunk_fwd_segmented_workspace_size",
           "gdn2_chunk_fwd_segments", "gdn2_chunk_fwd_logits", "gdn2_output_gate", "gdn2_recurrent_step", "gdn2_chunk_bwd",
           "gdn2_chunk_bwd_workspace_size", "gdn2_chunk_bwd_noalloc", "gdn2_device_error", "gdn2_set_wait_limit", "library_path",
           "load_library", "exported_symbols",
           "GDN2_OK", "GDN2_ERR_INVALID_ARG", "GDN2_ERR_UNSUPPORTED", "GDN2_ERR_CUDA", "Gdn2Error"]

GDN2_OK, GDN2_ERR_INVALID_ARG, GDN2_ERR_UNSUPPORTED, GDN2_ERR_CUDA = 0, 1, 2, 3
GDN2_BF16, GDN2_FP32 = 0, 1
HEADER = os.path.join(_build.ROOT, "include", "gdn2.h")

_lib = None


class Gdn2Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


def library_path() -> str:
    return _build.LIB


def load_library(rebuild_if_stale: bool = True) -> ctypes.CDLL:
    """Load libgdn2.so (compiling it first if it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build() if rebuild_if_stale else _build.LIB
    if not os.path.exists(path):
        raise ImportError(f"libgdn2.so not found at {path}; run python -m gated_delta_rule_111_b200.build")
    lib = ctypes.CDLL(path)
    vp, fp, i, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    lib.gdn2_chunk_fwd.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, i, i, i, i, i, i, vp]
    lib.gdn2_chunk_fwd.restype = i
    lib.gdn2_chunk_fwd_varlen.argtypes = [vp, vp, vp, fp, fp, fp, vp, i, fp, vp, fp, i, i, i, i, i, vp]
    lib.gdn2_chunk_fwd_varlen.restype = i
    lib.gdn2_chunk_fwd_segmented.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, i, i, i, i, i, i, i, vp, sz, vp]
    lib.gdn2_chunk_fwd_segmented.restype = i
    lib.gdn2_chunk_fwd_segmented_workspace_size.argtypes = [i, i, i, i, i, i]
    lib.gdn2_chunk_fwd_segmented_workspace_size.restype = sz
    lib.gdn2_chunk_fwd_segments.argtypes = [i, i, i, i, i, i]
    lib.gdn2_chunk_fwd_segments.restype = i
    lib.gdn2_chunk_fwd_logits.argtypes = [vp, vp, vp, vp, vp, vp, fp, vp, fp, i, i, i, i, i, vp]
    lib.gdn2_chunk_fwd_logits.restype = i
    lib.gdn2_output_gate.argtypes = [vp, vp, fp, ctypes.c_float, vp, i, i, i, i, i, vp]
    lib.gdn2_output_gate.restype = i
    lib.gdn2_recurrent_step.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, i, i, i, i, i, vp]
    lib.gdn2_recurrent_step.restype = i
    lib.gdn2_chunk_bwd.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, vp, vp, vp, fp, fp, fp, fp, vp, sz,
                                   i, i, i, i, i, i, vp]
    lib.gdn2_chunk_bwd.restype = i
    lib.gdn2_chunk_bwd_noalloc.argtypes = [vp, vp, vp, fp, fp, fp, fp, vp, fp, vp, vp, vp, fp, fp, fp, fp,
                                           i, i, i, i, i, i, vp]
    lib.gdn2_chunk_bwd_noalloc.restype = i
    lib.gdn2_chunk_bwd_workspace_size.argtypes = [i, i, i, i, i]
    lib.gdn2_chunk_bwd_workspace_size.restype = sz
    lib.gdn2_status_string.argtypes = [i]
    lib.gdn2_status_string.restype = ctypes.c_char_p
    lib.gdn2_last_error.argtypes = []
    lib.gdn2_last_error.restype = ctypes.c_char_p
    lib.gdn2_version.restype = i
    lib.gdn2_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint), i]
    lib.gdn2_device_error.restype = i
    lib.gdn2_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.gdn2_set_wait_limit.restype = i
    _lib = lib
    return lib


def exported_symbols() -> list[str]:
    """Function names declared in include/gdn2.h."""
    text = open(HEADER).read()
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(gdn2_\w+)\s*\(", text, flags=re.M)


def _check(status: int):
    if status != GDN2_OK:
        lib = load_library()
        msg = lib.gdn2_last_error().decode()
        raise Gdn2Error(status, f"{lib.gdn2_status_string(status).decode()}: {msg}")


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN2_BF16
    if t.dtype == torch.float32:
        return GDN2_FP32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, name, dtype, shape, device):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise ValueError(f"{name}: expected device {device}, got {t.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def gdn2_device_error(clear: bool = True) -> int:
    """Synchronously read (and by default clear) the kernels' device-side failure flag."""
    lib = load_library()
    code = ctypes.c_uint(0)
    _check(lib.gdn2_device_error(ctypes.byref(code), int(clear)))
    return int(code.value)


def gdn2_set_wait_limit(cycles: int = 0) -> None:
    """Test hook: SM cycles before a kernel's internal wait gives up (0 = default, ~2 s)."""
    _check(load_library().gdn2_set_wait_limit(int(cycles)))


def gdn2_chunk_fwd(q, k, v, alpha, b, w, S0=None, *, o=None, S_T=None, output_final_state=True,
                   stream=None):
    """Chunkwise prefill.  q,k [B,T,H,dk], v [B,T,H,dv] (bf16 or fp32); alpha,b [B,T,H,dk] and
    w [B,T,H,dv] fp32; S0 [B,H,dk,dv] fp32 or None.  Returns (o, S_T); S_T is None when
    ``output_final_state`` is False and no S_T buffer is given.  S_T may be S0 (in place)."""
    lib = load_library()
    if q.device.type != "cuda":
        raise ValueError("gdn2_chunk_fwd needs CUDA tensors (there is no CPU implementation)")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for name, t, d in (("q", q, dk), ("k", k, dk), ("v", v, dv)):
        _need(t, name, dt, (B, T, H, d), dev)
    for name, t, d in (("alpha", alpha, dk), ("b", b, dk), ("w", w, dv)):
        _need(t, name, torch.float32, (B, T, H, d), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _need(o, "o", dt, (B, T, H, dv), dev)
    if S_T is None and output_final_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    elif S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dk, dv), dev)
    with torch.cuda.device(dev):
        _check(lib.gdn2_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(o),
                                  _ptr(S_T), B, T, H, dk, dv, code, _stream(stream, dev)))
    return o, S_T


_copy_streams = {}


def _streams(device):
    """Two side streams per device (host-to-device and device-to-host copies), created once."""
    key = device.index
    if key not in _copy_streams:
        _copy_streams[key] = (torch.cuda.Stream(device), torch.cuda.Stream(device))
    return _copy_streams[key]


def gdn2_chunk_fwd_from_host(q, k, v, alpha, b, w, S0=None, *, device=None, work=None, o=None, S_T=None,
                             piece_tokens=None, stream=None):
    """Chunkwise prefill from host tensors, arguments as gdn2_chunk_fwd but in (pinned) CPU memory;
    returns host (o, S_T).  The batch is streamed in pieces of ``piece_tokens`` tokens of one
    sequence (rounded down to a multiple of the 64-token chunk; None: whole sequences, the
    fastest on the 4 x 4096 x 16 workload, where smaller pieces add more enqueue overhead than
    they save at the tail): a piece's inputs go to the device on one copy
    stream, its prefill (a gdn2_chunk_fwd call on ``stream``, started from the state the previous
    piece of the sequence left) runs as soon as they have arrived, and its outputs come back on a
    second copy stream while the next piece is copied in.  Pieces are whole chunks, so the result
    equals one call over the batch bit for bit (unless a very strong decay makes the kernel cut a
    chunk short, which moves later chunk boundaries; the result is then equally exact, to
    rounding).

    ``work``: dict of device tensors q, k, v, alpha, b, w (and S0 when given), o, S_T with the
    inputs' shapes, reused across calls (allocated here when None).  ``o`` / ``S_T``: host output
    tensors (pinned; allocated here when None).  On return every copy and launch is enqueued and
    ``stream`` waits for the last of them; host outputs are valid after it synchronises."""
    if q.device.type != "cpu":
        raise ValueError("gdn2_chunk_fwd_from_host takes host tensors")
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    names = ("q", "k", "v", "alpha", "b", "w")
    src = dict(zip(names, (q, k, v, alpha, b, w)))
    if work is None:
        work = {n: torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in src.items()}
        if S0 is not None:
            work["S0"] = torch.empty(S0.shape, dtype=S0.dtype, device=dev)
        work["o"] = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
        work["S_T"] = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    missing = [n for n in list(src) + (["S0"] if S0 is not None else []) + ["o", "S_T"] if n not in work]
    if missing:
        raise ValueError(f"work: missing device buffers {missing}")
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype).pin_memory()
    if S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32).pin_memory()
    tp = max(T, 1) if piece_tokens is None else max(64, (int(piece_tokens) // 64) * 64)
    with torch.cuda.device(dev):
        main = torch.cuda.current_stream(dev) if stream is None else stream
        s_in, s_out = _streams(dev)
        s_in.wait_stream(main)
        s_out.wait_stream(main)
        for i in range(B):
            if S0 is not None:
                with torch.cuda.stream(s_in):
                    work["S0"][i].copy_(S0[i], non_blocking=True)
            state = work["S0"][i:i + 1] if S0 is not None else None
            for t0 in range(0, max(T, 1), tp):
                t1 = min(T, t0 + tp)
                with torch.cuda.stream(s_in):
                    for n in names:
                        work[n][i, t0:t1].copy_(src[n][i, t0:t1], non_blocking=True)
                main.wait_stream(s_in)
                piece = {n: work[n][i:i + 1, t0:t1] for n in names}
                gdn2_chunk_fwd(*(piece[n] for n in names), state, o=work["o"][i:i + 1, t0:t1],
                               S_T=work["S_T"][i:i + 1], stream=main)
                state = work["S_T"][i:i + 1]       # the next piece starts where this one ended
                s_out.wait_stream(main)
                with torch.cuda.stream(s_out):
                    o[i, t0:t1].copy_(work["o"][i, t0:t1], non_blocking=True)
            with torch.cuda.stream(s_out):
                S_T[i].copy_(work["S_T"][i], non_blocking=True)
        main.wait_stream(s_out)
    return o, S_T


def gdn2_chunk_fwd_segmented_workspace_size(B, T, H, dk, dv, segments=0) -> int:
    """Workspace bytes of gdn2_chunk_fwd_segmented (segments = 0 resolves against the current device)."""
    return int(load_library().gdn2_chunk_fwd_segmented_workspace_size(B, T, H, dk, dv, segments))


def gdn2_chunk_fwd_segments(B, T, H, dk, dv, segments=0) -> int:
    """The number of segments gdn2_chunk_fwd_segmented uses for this shape (1: the plain call)."""
    return int(load_library().gdn2_chunk_fwd_segments(B, T, H, dk, dv, segments))


def gdn2_chunk_fwd_segmented(q, k, v, alpha, b, w, S0=None, *, segments=0, workspace=None, o=None, S_T=None,
                             output_final_state=True, stream=None):
    """Segment-parallel chunkwise prefill: arguments and result as gdn2_chunk_fwd; each sequence is cut
    into ``segments`` pieces (0: chosen from the shape and the device) processed in parallel.
    ``workspace``: a uint8 CUDA tensor of at least gdn2_chunk_fwd_segmented_workspace_size(...)
    bytes, allocated here when None."""
    lib = load_library()
    if q.device.type != "cuda":
        raise ValueError("gdn2_chunk_fwd_segmented needs CUDA tensors (there is no CPU implementation)")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for name, t, d in (("q", q, dk), ("k", k, dk), ("v", v, dv)):
        _need(t, name, dt, (B, T, H, d), dev)
    for name, t, d in (("alpha", alpha, dk), ("b", b, dk), ("w", w, dv)):
        _need(t, name, torch.float32, (B, T, H, d), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=dt, device=dev)
    else:
        _need(o, "o", dt, (B, T, H, dv), dev)
    if S_T is None and output_final_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    elif S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dk, dv), dev)
    with torch.cuda.device(dev):
        need = int(lib.gdn2_chunk_fwd_segmented_workspace_size(B, T, H, dk, dv, int(segments)))
        if workspace is None:
            workspace = torch.empty((max(need, 1),), dtype=torch.uint8, device=dev)
        elif workspace.dtype != torch.uint8 or workspace.device != dev or not workspace.is_contiguous():
            raise ValueError("workspace: expected a contiguous uint8 tensor on the inputs' device")
        _check(lib.gdn2_chunk_fwd_segmented(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0),
                                            _ptr(o), _ptr(S_T), B, T, H, dk, dv, code, int(segments),
                                            _ptr(workspace) if need > 0 else None, workspace.numel(),
                                            _stream(stream, dev)))
    return o, S_T


def gdn2_chunk_fwd_varlen(q, k, v, alpha, b, w, cu_seqlens, S0=None, *, o=None, S_T=None,
                          output_final_state=True, stream=None):
    """Chunkwise prefill of a packed batch.  q,k [T,H,dk], v [T,H,dv] (bf16 or fp32); alpha,b
    [T,H,dk], w [T,H,dv] fp32; cu_seqlens int32 [N+1] on the same device (sequence n is rows
    cu_seqlens[n] .. cu_seqlens[n+1]-1); S0 [N,H,dk,dv] fp32 or None.  Returns (o [T,H,dv],
    S_T [N,H,dk,dv] or None)."""
    lib = load_library()
    if q.device.type != "cuda":
        raise ValueError("gdn2_chunk_fwd_varlen needs CUDA tensors (there is no CPU implementation)")
    T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for name, t, d in (("q", q, dk), ("k", k, dk), ("v", v, dv)):
        _need(t, name, dt, (T, H, d), dev)
    for name, t, d in (("alpha", alpha, dk), ("b", b, dk), ("w", w, dv)):
        _need(t, name, torch.float32, (T, H, d), dev)
    if cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens: expected a 1-D tensor of N + 1 offsets")
    N = cu_seqlens.numel() - 1
    _need(cu_seqlens, "cu_seqlens", torch.int32, (N + 1,), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (N, H, dk, dv), dev)
    if o is None:
        o = torch.empty((T, H, dv), dtype=dt, device=dev)
    else:
        _need(o, "o", dt, (T, H, dv), dev)
    if S_T is None and output_final_state:
        S_T = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    elif S_T is not None:
        _need(S_T, "S_T", torch.float32, (N, H, dk, dv), dev)
    with torch.cuda.device(dev):
        _check(lib.gdn2_chunk_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(cu_seqlens),
                                         N, _ptr(S0), _ptr(o), _ptr(S_T), T, H, dk, dv, code, _stream(stream, dev)))
    return o, S_T


def gdn2_chunk_fwd_logits(xq, xk, xv, xa, xb, xw, S0=None, *, o=None, S_T=None, output_final_state=True,
                          stream=None):
    """Chunkwise prefill from BF16 pre-activation logits [B,T,H,128] each (activations and
    gates computed inside the kernel); S0 [B,H,128,128] fp32 or None.  Returns (o, S_T)."""
    lib = load_library()
    if xq.device.type != "cuda":
        raise ValueError("gdn2_chunk_fwd_logits needs CUDA tensors (there is no CPU implementation)")
    B, T, H, dk = xq.shape
    dv = xv.shape[-1]
    dev = xq.device
    for name, t, d in (("xq", xq, dk), ("xk", xk, dk), ("xv", xv, dv), ("xa", xa, dk), ("xb", xb, dk),
                       ("xw", xw, dv)):
        _need(t, name, torch.bfloat16, (B, T, H, d), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    else:
        _need(o, "o", torch.bfloat16, (B, T, H, dv), dev)
    if S_T is None and output_final_state:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    elif S_T is not None:
        _need(S_T, "S_T", torch.float32, (B, H, dk, dv), dev)
    with torch.cuda.device(dev):
        _check(lib.gdn2_chunk_fwd_logits(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(xa), _ptr(xb), _ptr(xw), _ptr(S0),
                                         _ptr(o), _ptr(S_T), B, T, H, dk, dv, _stream(stream, dev)))
    return o, S_T


def gdn2_output_gate(o, g, weight, eps=1e-6, *, y=None, stream=None):
    """Output epilogue: y = o / sqrt(mean(o^2) + eps) * weight * sigmoid(g) per (token, head) row.
    o, g [B,T,H,dv] (bf16 or fp32, same dtype), weight [dv] fp32; y may be o (in place)."""
    lib = load_library()
    if o.device.type != "cuda":
        raise ValueError("gdn2_output_gate needs CUDA tensors (there is no CPU implementation)")
    B, T, H, dv = o.shape
    dev, dt = o.device, o.dtype
    code = _dtype_code(o)
    _need(g, "g", dt, (B, T, H, dv), dev)
    _need(weight, "weight", torch.float32, (dv,), dev)
    if y is None:
        y = torch.empty_like(o)
    else:
        _need(y, "y", dt, (B, T, H, dv), dev)
    with torch.cuda.device(dev):
        _check(lib.gdn2_output_gate(_ptr(o), _ptr(g), _ptr(weight), float(eps), _ptr(y), B, T, H, dv, code,
                                    _stream(stream, dev)))
    return y


def gdn2_recurrent_step(q, k, v, alpha, b, w, S, *, o=None, stream=None):
    """One decode step, state updated in place.  q,k [B,H,dk], v [B,H,dv] (bf16 or fp32);
    alpha,b [B,H,dk], w [B,H,dv] fp32; S [B,H,dk,dv] fp32 (overwritten).  Returns o [B,H,dv]."""
    lib = load_library()
    if q.device.type != "cuda":
        raise ValueError("gdn2_recurrent_step needs CUDA tensors (there is no CPU implementation)")
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for name, t, d in (("q", q, dk), ("k", k, dk), ("v", v, dv)):
        _need(t, name, dt, (B, H, d), dev)
    for name, t, d in (("alpha", alpha, dk), ("b", b, dk), ("w", w, dv)):
        _need(t, name, torch.float32, (B, H, d), dev)
    _need(S, "S", torch.float32, (B, H, dk, dv), dev)
    if o is None:
        o = torch.empty((B, H, dv), dtype=dt, device=dev)
    else:
        _need(o, "o", dt, (B, H, dv), dev)
    with torch.cuda.device(dev):
        _check(lib.gdn2_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S), _ptr(o),
                                       B, H, dk, dv, code, _stream(stream, dev)))
    return o


def gdn2_chunk_bwd_workspace_size(B: int, T: int, H: int, dk: int, dv: int) -> int:
    """Bytes of device workspace gdn2_chunk_bwd needs (0 for unsupported head sizes)."""
    return int(load_library().gdn2_chunk_bwd_workspace_size(B, T, H, dk, dv))


def gdn2_chunk_bwd(q, k, v, alpha, b, w, S0=None, dO=None, dST=None, *, workspace=None, out=None,
                   stream=None):
    """Gradients of a loss through gdn2_chunk_fwd.  Inputs as for gdn2_chunk_fwd; dO [B,T,H,dv] in
    q's dtype (None = zero), dST [B,H,dk,dv] fp32 or None.  Returns a dict with dq, dk, dv (q's
    dtype), dalpha, db, dw, dS0 (fp32).  ``workspace`` (uint8 CUDA tensor of at least
    gdn2_chunk_bwd_workspace_size bytes) and ``out`` (a dict of preallocated gradients) are
    optional; missing buffers are allocated here."""
    lib = load_library()
    if q.device.type != "cuda":
        raise ValueError("gdn2_chunk_bwd needs CUDA tensors (there is no CPU implementation)")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for name, t, d in (("q", q, dk), ("k", k, dk), ("v", v, dv)):
        _need(t, name, dt, (B, T, H, d), dev)
    for name, t, d in (("alpha", alpha, dk), ("b", b, dk), ("w", w, dv)):
        _need(t, name, torch.float32, (B, T, H, d), dev)
    if S0 is not None:
        _need(S0, "S0", torch.float32, (B, H, dk, dv), dev)
    if dO is None:
        dO = torch.zeros((B, T, H, dv), dtype=dt, device=dev)
    _need(dO, "dO", dt, (B, T, H, dv), dev)
    if dST is not None:
        _need(dST, "dST", torch.float32, (B, H, dk, dv), dev)
    shapes = {"dq": ((B, T, H, dk), dt), "dk": ((B, T, H, dk), dt), "dv": ((B, T, H, dv), dt),
              "dalpha": ((B, T, H, dk), torch.float32), "db": ((B, T, H, dk), torch.float32),
              "dw": ((B, T, H, dv), torch.float32), "dS0": ((B, H, dk, dv), torch.float32)}
    g = dict(out or {})
    for name, (shape, dtype) in shapes.items():
        if g.get(name) is None:
            g[name] = torch.empty(shape, dtype=dtype, device=dev)
        else:
            _need(g[name], name, dtype, shape, dev)
    need = gdn2_chunk_bwd_workspace_size(B, T, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    elif workspace.device != dev or not workspace.is_contiguous():
        raise ValueError("workspace: expected a contiguous tensor on the inputs' device")
    ws_bytes = workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        _check(lib.gdn2_chunk_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0), _ptr(dO),
                                  _ptr(dST), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]), _ptr(g["dalpha"]),
                                  _ptr(g["db"]), _ptr(g["dw"]), _ptr(g["dS0"]), _ptr(workspace), ws_bytes,
                                  B, T, H, dk, dv, code, _stream(stream, dev)))
    return g


def gdn2_chunk_bwd_noalloc(q, k, v, alpha, b, w, S0, dO, dST, out, *, stream=None):
    """gdn2_chunk_bwd with the library's fixed 32 MiB device workspace (no allocation in
    the call).  ``out`` is a dict of preallocated gradient tensors dq, dk, dv, dalpha, db,
    dw, dS0 (dS0 may be None); dO must be given.  Returns ``out``."""
    lib = load_library()
    if q.device.type != "cuda":
        raise ValueError("gdn2_chunk_bwd_noalloc needs CUDA tensors (there is no CPU implementation)")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev, dt = q.device, q.dtype
    code = _dtype_code(q)
    for name, t, d in (("q", q, dk), ("k", k, dk), ("v", v, dv), ("dO", dO, dv)):
        _need(t, name, dt, (B, T, H, d), dev)
    for name, t, d in (("alpha", alpha, dk), ("b", b, dk), ("w", w, dv)):
        _need(t, name, torch.float32, (B, T, H, d), dev)
    for name, t in (("S0", S0), ("dST", dST)):
        if t is not None:
            _need(t, name, torch.float32, (B, H, dk, dv), dev)
    shapes = {"dq": ((B, T, H, dk), dt), "dk": ((B, T, H, dk), dt), "dv": ((B, T, H, dv), dt),
              "dalpha": ((B, T, H, dk), torch.float32), "db": ((B, T, H, dk), torch.float32),
              "dw": ((B, T, H, dv), torch.float32), "dS0": ((B, H, dk, dv), torch.float32)}
    for name, (shape, dtype) in shapes.items():
        if name == "dS0" and out.get(name) is None:
            continue
        _need(out[name], name, dtype, shape, dev)
    with torch.cuda.device(dev):
        _check(lib.gdn2_chunk_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(b), _ptr(w), _ptr(S0),
                                          _ptr(dO), _ptr(dST), _ptr(out["dq"]), _ptr(out["dk"]), _ptr(out["dv"]),
                                          _ptr(out["dalpha"]), _ptr(out["db"]), _ptr(out["dw"]), _ptr(out.get("dS0")),
                                          B, T, H, dk, dv, code, _stream(stream, dev)))
    return out
