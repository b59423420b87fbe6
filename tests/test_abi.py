"""The C ABI of libgdn2 without a GPU: the library loads, exports every function
declared in include/gdn2.h, and rejects bad arguments on the host before any
CUDA call.  Every call below returns during host-side validation."""
import ctypes
import subprocess

import pytest
import torch

import gated_delta_rule_111_b200 as g

BF16, FP32 = 0, 1
A16 = 0x10000          # a fake, 16-byte aligned "device" address; never dereferenced


@pytest.fixture(scope="module")
def lib():
    return g.load_library()


def test_exports_every_declared_symbol(lib):
    declared = g.exported_symbols()
    assert set(declared) >= {"gdn2_chunk_fwd", "gdn2_recurrent_step", "gdn2_status_string",
                             "gdn2_last_error", "gdn2_version"}
    out = subprocess.check_output(["nm", "-D", "--defined-only", g.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [s for s in declared if s not in exported]
    assert not missing, f"declared but not exported: {missing}"
    for s in declared:
        getattr(lib, s)


def test_status_strings(lib):
    assert lib.gdn2_status_string(0) == b"GDN2_OK"
    assert lib.gdn2_status_string(1) == b"GDN2_ERR_INVALID_ARG"
    assert lib.gdn2_status_string(2) == b"GDN2_ERR_UNSUPPORTED"
    assert lib.gdn2_status_string(3) == b"GDN2_ERR_CUDA"
    assert lib.gdn2_version() >= 100


def _chunk(lib, q=A16, k=A16, v=A16, a=A16, b=A16, w=A16, S0=None, o=A16 * 64, ST=None,
           B=1, T=4, H=1, dk=128, dv=128, dt=BF16):
    P = ctypes.c_void_p
    return lib.gdn2_chunk_fwd(P(q), P(k), P(v), P(a), P(b), P(w), P(S0), P(o), P(ST), B, T, H, dk, dv, dt, None)


def _step(lib, q=A16, k=A16, v=A16, a=A16, b=A16, w=A16, S=A16 * 128, o=A16 * 512, B=1, H=1, dk=128, dv=128,
          dt=BF16):
    P = ctypes.c_void_p
    return lib.gdn2_recurrent_step(P(q), P(k), P(v), P(a), P(b), P(w), P(S), P(o), B, H, dk, dv, dt, None)


@pytest.mark.parametrize("dk,dv", [(32, 128), (128, 96), (256, 256), (0, 128)])
def test_unsupported_head_sizes(lib, dk, dv):
    assert _chunk(lib, dk=dk, dv=dv) == g.GDN2_ERR_UNSUPPORTED
    assert _step(lib, dk=dk, dv=dv) == g.GDN2_ERR_UNSUPPORTED


def test_unknown_dtype(lib):
    assert _chunk(lib, dt=7) == g.GDN2_ERR_UNSUPPORTED
    assert _step(lib, dt=-1) == g.GDN2_ERR_UNSUPPORTED


@pytest.mark.parametrize("field", ["q", "k", "v", "a", "b", "w", "o"])
def test_null_pointer_rejected(lib, field):
    assert _chunk(lib, **{field: None}) == g.GDN2_ERR_INVALID_ARG
    assert b"null pointer" in lib.gdn2_last_error()


@pytest.mark.parametrize("field", ["q", "k", "v", "a", "b", "w", "o", "S0", "ST"])
def test_misaligned_pointer_rejected(lib, field):
    assert _chunk(lib, **{field: A16 * 1024 + 4}) == g.GDN2_ERR_INVALID_ARG
    assert b"aligned" in lib.gdn2_last_error()


def test_step_null_state_rejected(lib):
    assert _step(lib, S=None) == g.GDN2_ERR_INVALID_ARG


def test_negative_sizes(lib):
    assert _chunk(lib, T=-1) == g.GDN2_ERR_INVALID_ARG
    assert _chunk(lib, B=-2) == g.GDN2_ERR_INVALID_ARG
    assert _step(lib, H=-1) == g.GDN2_ERR_INVALID_ARG


def test_empty_batch_is_noop(lib):
    # B = 0 or H = 0 returns before any CUDA call, even with null pointers.
    assert _chunk(lib, q=None, o=None, B=0) == g.GDN2_OK
    assert _chunk(lib, q=None, o=None, H=0) == g.GDN2_OK
    assert _step(lib, q=None, S=None, B=0) == g.GDN2_OK


def test_t0_inplace_state_is_noop(lib):
    # T = 0 with S_T aliasing S0 leaves the state as it is; nothing to enqueue.
    assert _chunk(lib, q=None, o=None, T=0, S0=A16 * 4096, ST=A16 * 4096) == g.GDN2_OK


def test_overlapping_output_rejected(lib):
    # o overlapping an input, and a state that partially overlaps S0.
    assert _chunk(lib, q=A16 * 64, o=A16 * 64) == g.GDN2_ERR_INVALID_ARG
    assert b"overlaps" in lib.gdn2_last_error()
    assert _chunk(lib, S0=A16 * 4096, ST=A16 * 4096 + 16) == g.GDN2_ERR_INVALID_ARG
    assert _step(lib, o=A16 * 128, S=A16 * 128) == g.GDN2_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        g.gdn2_chunk_fwd(x, x, x, x, x, x)
    y = torch.zeros(1, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        g.gdn2_recurrent_step(y, y, y, y, y, y, torch.zeros(1, 1, 64, 64))


def test_product_package_does_not_import_oracle():
    import pathlib
    pkg = pathlib.Path(g.__file__).parent
    for p in list(pkg.rglob("*.py")) + list(pkg.rglob("*.cu")) + list(pkg.rglob("*.cuh")):
        text = p.read_text()
        assert "oracle" not in text.replace("oracle-free", ""), f"{p} mentions the oracle"


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the compiled library the binding raises; there is no fallback path."""
    from gated_delta_rule_111_b200 import build as b
    monkeypatch.setattr(g, "_lib", None)
    monkeypatch.setattr(b, "LIB", str(tmp_path / "libgdn2.so"))
    with pytest.raises(ImportError, match="libgdn2.so not found"):
        g.load_library(rebuild_if_stale=False)


def _varlen(lib, cu=A16 * 8192, N=3, T=10, H=1, dk=128, dv=128, dt=BF16, o=A16 * 64):
    P = ctypes.c_void_p
    return lib.gdn2_chunk_fwd_varlen(P(A16), P(A16), P(A16), P(A16), P(A16), P(A16), P(cu), N, None, P(o), None,
                                     T, H, dk, dv, dt, None)


def test_varlen_host_checks(lib):
    assert _varlen(lib, cu=None) == g.GDN2_ERR_INVALID_ARG
    assert b"cu_seqlens" in lib.gdn2_last_error()
    assert _varlen(lib, cu=A16 * 8192 + 2) == g.GDN2_ERR_INVALID_ARG
    assert _varlen(lib, N=-1) == g.GDN2_ERR_INVALID_ARG
    assert _varlen(lib, dk=96) == g.GDN2_ERR_UNSUPPORTED
    assert _varlen(lib, N=0, cu=None) == g.GDN2_OK          # nothing to do, before any CUDA call
    assert _varlen(lib, o=A16) == g.GDN2_ERR_INVALID_ARG    # o overlaps the inputs


def test_varlen_binding_validates_offsets_tensor():
    x = torch.zeros(8, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        g.gdn2_chunk_fwd_varlen(x, x, x, x, x, x, torch.zeros(3, dtype=torch.int32))


def _bwd(lib, ws=A16 * 4096, ws_bytes=1 << 40, B=1, T=10, H=1, dk=128, dv=128, dt=BF16, dq=A16 * 64,
         S0=None, dST=None, dS0=None):
    # inputs at A16..A16*8, outputs spaced far apart so that only the named overlaps exist
    q, k, v, a, b, w, dO = (A16 * (1 + i) for i in range(7))
    outs = [dq, A16 * 128, A16 * 192, A16 * 256, A16 * 320, A16 * 384]
    return lib.gdn2_chunk_bwd(q, k, v, a, b, w, S0, dO, dST, *outs, dS0, ws, ws_bytes, B, T, H, dk, dv, dt, None)


def test_backward_host_checks(lib):
    assert _bwd(lib, dk=96) == g.GDN2_ERR_UNSUPPORTED
    assert _bwd(lib, dt=7) == g.GDN2_ERR_UNSUPPORTED
    assert _bwd(lib, T=-1) == g.GDN2_ERR_INVALID_ARG
    assert _bwd(lib, B=0) == g.GDN2_OK and _bwd(lib, H=0) == g.GDN2_OK
    assert _bwd(lib, B=4096, H=16) == g.GDN2_ERR_UNSUPPORTED        # B * H beyond the grid's 65535
    need = lib.gdn2_chunk_bwd_workspace_size(1, 10, 1, 128, 128)
    # chunk states and gradients, T and P, U and dR per token, and the key block
    # (five [64][132] tiles, two [64][132], one [128][132], 128 decay factors)
    key_block = 5 * 64 * 132 + 2 * 64 * 132 + 128 * 132 + 128
    # and the gradient kernels' hand-over: dP and dA, S dO / S dR / dS' U, row sums
    grad_block = 2 * 64 * 64 + 3 * 64 * 128 + 128
    assert need == 4 * (2 * 128 * 128 + 2 * 64 * 64 + 2 * 10 * 128 + key_block + grad_block)
    assert _bwd(lib, ws_bytes=need - 4) == g.GDN2_ERR_INVALID_ARG
    assert b"workspace" in lib.gdn2_last_error()
    assert _bwd(lib, ws=None) == g.GDN2_ERR_INVALID_ARG
    assert _bwd(lib, dq=A16 + 8) == g.GDN2_ERR_INVALID_ARG          # misaligned
    assert _bwd(lib, dq=A16 * 2) == g.GDN2_ERR_INVALID_ARG          # dq overlaps k
    assert b"overlaps" in lib.gdn2_last_error()
    assert _bwd(lib, ws=A16 * 128) == g.GDN2_ERR_INVALID_ARG        # workspace overlaps dk
    assert lib.gdn2_chunk_bwd_workspace_size(1, 10, 1, 96, 128) == 0


def test_backward_binding_refuses_cpu_tensors():
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        g.gdn2_chunk_bwd(x, x, x, x, x, x)


def test_logits_host_checks(lib):
    args = [A16 * (1 + i) for i in range(6)]
    assert lib.gdn2_chunk_fwd_logits(*args, None, A16 * 64, None, 1, 10, 1, 64, 64, None) == g.GDN2_ERR_UNSUPPORTED
    assert lib.gdn2_chunk_fwd_logits(*args, None, A16 * 64, None, 1, -1, 1, 128, 128, None) == g.GDN2_ERR_INVALID_ARG
    assert lib.gdn2_chunk_fwd_logits(*args, None, A16 * 64, None, 0, 10, 1, 128, 128, None) == g.GDN2_OK
    bad = list(args)
    bad[3] = A16 + 4
    assert lib.gdn2_chunk_fwd_logits(*bad, None, A16 * 64, None, 1, 10, 1, 128, 128, None) == g.GDN2_ERR_INVALID_ARG
    assert lib.gdn2_chunk_fwd_logits(*args, None, A16 * 2, None, 1, 10, 1, 128, 128, None) == g.GDN2_ERR_INVALID_ARG
    assert b"overlaps" in lib.gdn2_last_error()


def test_output_gate_host_checks(lib):
    c = ctypes.c_float
    assert lib.gdn2_output_gate(A16, A16 * 2, A16 * 3, c(1e-6), A16 * 64, 1, 4, 2, 96, BF16, None) == g.GDN2_ERR_UNSUPPORTED
    assert lib.gdn2_output_gate(A16, A16 * 2, A16 * 3, c(-1.0), A16 * 64, 1, 4, 2, 128, BF16, None) == g.GDN2_ERR_INVALID_ARG
    assert lib.gdn2_output_gate(A16, A16 * 2, A16 * 3, c(1e-6), A16 * 64, 0, 4, 2, 128, BF16, None) == g.GDN2_OK
    assert lib.gdn2_output_gate(A16 + 2, A16 * 2, A16 * 3, c(1e-6), A16 * 64, 1, 4, 2, 128, BF16, None) == g.GDN2_ERR_INVALID_ARG
    # y partially overlapping o is refused; exact aliasing would be allowed
    assert lib.gdn2_output_gate(A16, A16 * 2, A16 * 3, c(1e-6), A16 + 16, 1, 4, 2, 128, BF16, None) == g.GDN2_ERR_INVALID_ARG
    assert b"overlaps" in lib.gdn2_last_error()


WS = 0x10000000        # a fake, 256-byte aligned workspace address, clear of the fake inputs


def _seg(lib, segments=3, ws=WS, ws_bytes=None, dt=BF16, B=1, T=300, H=1, o=A16 * 64):
    P = ctypes.c_void_p
    if ws_bytes is None:
        ws_bytes = lib.gdn2_chunk_fwd_segmented_workspace_size(B, T, H, 128, 128, max(segments, 0))
    return lib.gdn2_chunk_fwd_segmented(P(A16), P(A16), P(A16), P(A16), P(A16), P(A16), None, P(o), None, B, T, H,
                                        128, 128, dt, segments, P(ws), ws_bytes, None)


def test_segmented_host_checks(lib):
    """Segment counts, the workspace size formula and every host-side refusal (each call below
    fails validation; none reaches a launch)."""
    assert lib.gdn2_chunk_fwd_segments(1, 65573, 16, 128, 128, 3) == 3   # 1,025 chunks: 342 per segment
    assert lib.gdn2_chunk_fwd_segments(3, 130, 2, 128, 128, 8) == 3      # capped at the 3 chunks
    assert lib.gdn2_chunk_fwd_segments(1, 64, 2, 128, 128, 8) == 1       # one chunk: the plain call
    assert lib.gdn2_chunk_fwd_segments(1, 1000, 1, 128, 128, 1) == 1
    assert lib.gdn2_chunk_fwd_segments(1, 1000, 1, 64, 64, 4) == 1       # not the tensor-core shape
    state = 128 * 128 * 4
    # token ranges of both launches (256-byte aligned), then C and M of segments 0 .. P-2 and every
    # segment's start state
    assert lib.gdn2_chunk_fwd_segmented_workspace_size(1, 65573, 16, 128, 128, 3) == \
        256 + 256 + 2 * 2 * 16 * state + 3 * 16 * state
    assert lib.gdn2_chunk_fwd_segmented_workspace_size(1, 1000, 1, 128, 128, 1) == 0
    need = lib.gdn2_chunk_fwd_segmented_workspace_size(1, 300, 1, 128, 128, 3)
    assert need == 256 + 256 + 4 * state + 3 * state
    assert _seg(lib, segments=-1) == g.GDN2_ERR_INVALID_ARG
    assert _seg(lib, dt=FP32) == g.GDN2_ERR_UNSUPPORTED
    assert _seg(lib, ws_bytes=need - 256) == g.GDN2_ERR_INVALID_ARG
    assert b"workspace" in lib.gdn2_last_error()
    assert _seg(lib, ws=None) == g.GDN2_ERR_INVALID_ARG
    assert _seg(lib, ws=WS + 16) == g.GDN2_ERR_INVALID_ARG                 # not 256-byte aligned
    assert _seg(lib, ws=A16 * 2) == g.GDN2_ERR_INVALID_ARG                 # overlaps the inputs
    assert b"overlaps" in lib.gdn2_last_error()
    assert _seg(lib, o=A16) == g.GDN2_ERR_INVALID_ARG                      # o overlaps the inputs


def test_segmented_binding_refuses_cpu_tensors():
    x = torch.zeros(1, 4, 1, 128)
    with pytest.raises(ValueError, match="CUDA"):
        g.gdn2_chunk_fwd_segmented(x, x, x, x, x, x)
