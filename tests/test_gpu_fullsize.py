"""GPU parity at full workload size, in the launch configuration the
benchmark times, against sampled outputs of the float64 oracle.

The expected values in tests/golden/step_<workload>.npz were written by
tests/golden/make_golden.py, which calls only the oracle and the seeded input
generators: the loss, 4096 sampled logits and 4 full logit rows, and per
parameter tensor 256 sampled gradient elements with the post-AdamW parameter
and moments there (t = 1).  Errors are norm-wise relative over the samples.
"""
import os

import numpy as np
import pytest
import torch

from synth import get_config, make_batch, make_params
from tests.gpu_util import TOL

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
WORKLOADS = ["c2", "c3", "c4", "c5"]


def _rel(a, b):
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a))


@pytest.mark.parametrize("name", WORKLOADS)
def test_full_size_step_matches_oracle_samples(name):
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config(name)
    path = os.path.join(GOLDEN, f"step_{cfg['name']}.npz")
    if not os.path.exists(path):
        pytest.skip(f"golden file {os.path.basename(path)} not generated yet "
                    "(tests/golden/make_golden.py)")
    z = np.load(path)
    tol = TOL[cfg["compute"]]
    m = LlamaStep(cfg)
    p = make_params(cfg, m.layout)
    tok, tgt = make_batch(cfg)
    P = torch.tensor(p, device="cuda")
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
    logits = m.forward(P, td).view(-1)
    li = torch.tensor(z["logit_idx"], device="cuda")
    lg = logits[li].double().cpu().numpy()
    rows = z["logit_rows"]
    lrows = logits.view(-1, cfg["vocab"])[torch.tensor(rows, device="cuda")].double().cpu().numpy()
    del logits
    loss = m.step(P, G, M, V, 1, td, yd, cfg["lr"], cfg["wd"])
    assert m.status() == 0
    gi = torch.tensor(z["g_idx"], device="cuda")
    g = G[gi].double().cpu().numpy()
    pn = P[gi].double().cpu().numpy()
    mn = M[gi].double().cpu().numpy()
    vn = V[gi].double().cpu().numpy()
    errs = {"loss": abs(float(loss.item()) - float(z["loss"])) / abs(float(z["loss"])),
            "logits": _rel(lg, z["logit_val"]), "logit_rows": _rel(lrows, z["logit_rowvals"])}
    assert errs["loss"] <= tol["loss"], errs
    assert errs["logits"] <= tol["logits"], errs
    assert errs["logit_rows"] <= tol["logits"], errs
    worst = {"grads": 0.0, "params": 0.0, "m": 0.0, "v": 0.0}
    for k, (off, cnt) in enumerate(zip(z["t_off"], z["t_cnt"])):
        sl = slice(int(off), int(off + cnt))
        for key, got, ref in (("grads", g, z["g_val"]), ("params", pn, z["p_val"]),
                              ("m", mn, z["m_val"]), ("v", vn, z["v_val"])):
            e = _rel(got[sl], ref[sl])
            worst[key] = max(worst[key], e)
            if tol[key] is not None:
                assert e <= tol[key], (str(z["names"][k]), key, e)
    print(cfg["name"], errs, worst)
