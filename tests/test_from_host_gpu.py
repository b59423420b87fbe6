"""gdn2_chunk_fwd_from_host: the prefill from pinned host tensors, streamed in token pieces
through two copy streams with the state chained on the device, against one gdn2_chunk_fwd call
over the whole batch on the device (bit for bit: pieces are whole 64-token chunks and the gates
here force no early chunk cut), with and without S0, and with the device buffers reused by a
second call."""
import numpy as np
import pytest
import torch

import gdn2_inputs as gi

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "alpha", "b", "w")


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import gated_delta_rule_111_b200 as mod
    mod.load_library()
    return mod


def _host(x):
    out = {}
    for n in NAMES:
        t = torch.from_numpy(np.ascontiguousarray(x[n]))
        out[n] = (t.to(torch.bfloat16) if n in ("q", "k", "v") else t).pin_memory()
    out["S0"] = None if x.get("S0") is None else torch.from_numpy(x["S0"]).pin_memory()
    return out


@pytest.mark.parametrize("s0,piece", [(0.05, 1024), (None, 1024), (0.05, 64), (None, 128)])
def test_from_host_matches_device_call(g, s0, piece):
    """One piece per sequence, or pieces of 64 / 128 tokens chained through the state (T = 200:
    the last piece ragged)."""
    x = gi.chunk_inputs(3, 200, 2, 128, 128, dtype="bf16", seed=40, s0_std=s0)
    h = _host(x)
    o_h, S_h = g.gdn2_chunk_fwd_from_host(*(h[n] for n in NAMES), h["S0"], piece_tokens=piece)
    d = {n: h[n].cuda() for n in NAMES}
    o_d, S_d = g.gdn2_chunk_fwd(*(d[n] for n in NAMES), None if h["S0"] is None else h["S0"].cuda())
    torch.cuda.synchronize()
    assert o_h.device.type == "cpu" and S_h.device.type == "cpu"
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(S_h, S_d.cpu())


def test_from_host_reuses_device_buffers(g):
    x = gi.chunk_inputs(2, 130, 2, 128, 128, dtype="bf16", seed=41, s0_std=0.05)
    y = gi.chunk_inputs(2, 130, 2, 128, 128, dtype="bf16", seed=42, s0_std=0.05)
    hx, hy = _host(x), _host(y)
    dev = torch.device("cuda", torch.cuda.current_device())
    work = {n: torch.empty(hx[n].shape, dtype=hx[n].dtype, device=dev) for n in NAMES + ("S0",)}
    work["o"] = torch.empty((2, 130, 2, 128), dtype=torch.bfloat16, device=dev)
    work["S_T"] = torch.empty((2, 2, 128, 128), dtype=torch.float32, device=dev)
    o1, S1 = g.gdn2_chunk_fwd_from_host(*(hx[n] for n in NAMES), hx["S0"], work=work)
    o2, S2 = g.gdn2_chunk_fwd_from_host(*(hy[n] for n in NAMES), hy["S0"], work=work)
    torch.cuda.synchronize()
    for h, o, S in ((hx, o1, S1), (hy, o2, S2)):
        d = {n: h[n].cuda() for n in NAMES}
        o_d, S_d = g.gdn2_chunk_fwd(*(d[n] for n in NAMES), h["S0"].cuda())
        torch.cuda.synchronize()
        assert torch.equal(o, o_d.cpu()) and torch.equal(S, S_d.cpu())
