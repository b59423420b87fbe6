"""Values the pages print, as fixtures under tests/golden/ (each file cites its source).

The pages give no worked numeric example of the recurrence itself; what they do
state is checked here against the oracle (CPU)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import gdn2_inputs as gi  # noqa: E402
import oracle  # noqa: E402

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _read(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split()
                out[k] = int(v)
    return out


def test_state_size_per_batch_item():
    """The oracle's final state for one batch item at the pages' head count and state
    dimensions has exactly the stated number of values (one d_k x d_v matrix per head)."""
    g = _read("state_size.txt")
    x = gi.chunk_inputs(1, 3, g["heads"], g["d_k"], g["d_v"], dtype="fp32", seed=0)
    _, S = oracle.gdn2(x["q"], x["k"], x["v"], x["alpha"], x["b"], x["w"])
    assert S.shape == (1, g["heads"], g["d_k"], g["d_v"])
    assert S[0].size == g["state_values"] == g["heads"] * g["d_k"] * g["d_v"]
    assert np.all(np.isfinite(S))
