"""The stored expected logit rows (tests/golden/) against the oracle.

logit_rows_<workload>.npz holds rows computed by the oracle's forward on one
sequence prefix; by causality they are the whole batch's rows.  Pinned here
two ways: a row of the full-batch oracle run stored in step_<workload>.npz is
reproduced from its sequence prefix alone, and a stored prefix row is
recomputed."""
import os

import numpy as np

import oracle as O
from synth import get_config, make_batch, make_params

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _prefix_row(cfg, row):
    tok, _ = make_batch(cfg)
    T = cfg["ctx"]
    b, t = divmod(int(row), T)
    p = make_params(cfg, O.param_layout(cfg)).astype(np.float64)
    sub = dict(cfg, batch=1, ctx=t + 1)
    _, z, _ = O.forward_backward(sub, p, np.ascontiguousarray(tok[b:b + 1, :t + 1]),
                                 want_grads=False)
    return z[t]


def test_prefix_forward_reproduces_a_full_batch_row():
    cfg = get_config("c4")
    z = np.load(os.path.join(GOLDEN, f"step_{cfg['name']}.npz"))
    k = int(np.argmin(z["logit_rows"] % cfg["ctx"]))  # the row with the shortest prefix
    got = _prefix_row(cfg, z["logit_rows"][k])
    want = z["logit_rowvals"][k]
    assert np.max(np.abs(got - want)) <= 1e-12 * np.max(np.abs(want))


def test_stored_block_rows_are_the_oracle_rows():
    for name in ("c2", "c3"):
        cfg = get_config(name)
        z = np.load(os.path.join(GOLDEN, f"logit_rows_{cfg['name']}.npz"))
        N = cfg["batch"] * cfg["ctx"]
        rows = list(z["rows"])
        assert rows[0] == 0 and rows[-1] == N - 1  # first and last row blocks
        assert all(r < 128 or r >= N - 128 for r in rows)
        for k in (1, len(rows) - 2):
            want = _prefix_row(cfg, rows[k])
            got = z["vals"][k].astype(np.float64)
            # stored as float32
            assert np.max(np.abs(got - want)) <= 1e-6 * np.max(np.abs(want))
