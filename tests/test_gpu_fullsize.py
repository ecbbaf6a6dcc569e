"""GPU parity at full workload size, in the launch configuration the
benchmark times, against sampled outputs of the float64 oracle.

The expected values in tests/golden/step_<workload>.npz were written by
tests/golden/make_golden.py, which calls only the oracle and the seeded input
generators: the loss, 4096 sampled logits and 4 full logit rows, and per
parameter tensor 256 sampled gradient elements with the post-AdamW parameter
and moments there (t = 1).  tests/golden/logit_rows_<workload>.npz (the same
script, --rows) adds full logit rows from the first and the last 128-row block,
the lm_head GEMM's first and last output tiles.  Errors are norm-wise relative
over the samples, with the element-wise max-abs gate and the bf16 parameter
gate of tests/gpu_util.py beside them.
"""
import os

import numpy as np
import pytest
import torch

from synth import get_config, make_batch, make_params
from tests.gpu_util import MAXABS_C, MAXABS_SAMPLED_C, SIGN_BAND, TOL, maxabs_ratio

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
    tiles = os.path.join(GOLDEN, f"logit_rows_{cfg['name']}.npz")
    if os.path.exists(tiles):
        zt = np.load(tiles)
        trows = logits.view(-1, cfg["vocab"])[torch.tensor(zt["rows"], device="cuda")]
        trows = trows.double().cpu().numpy()
        for k, r in enumerate(zt["rows"]):
            want = zt["vals"][k].astype(np.float64)
            e, ea = _rel(trows[k], want), maxabs_ratio(trows[k], want)
            assert e <= tol["logits"] and ea <= MAXABS_C * tol["logits"], (int(r), e, ea)
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
    errs["maxabs_logits"] = maxabs_ratio(lg, z["logit_val"])  # sampled
    errs["maxabs_logit_rows"] = max(maxabs_ratio(lrows[k], z["logit_rowvals"][k])
                                    for k in range(len(rows)))  # whole rows
    assert errs["loss"] <= tol["loss"], errs
    assert errs["logits"] <= tol["logits"], errs
    assert errs["logit_rows"] <= tol["logits"], errs
    assert errs["maxabs_logits"] <= MAXABS_SAMPLED_C * tol["logits"], errs
    assert errs["maxabs_logit_rows"] <= MAXABS_C * tol["logits"], errs
    bf16 = cfg["compute"] == "bf16"
    p0 = p.astype(np.float64)[z["g_idx"]]  # the parameters before the step, at the samples
    lr = float(np.float32(cfg["lr"]))
    # maxabs: the largest sampled max-abs ratio as a multiple of its tolerance
    worst = {"grads": 0.0, "params": 0.0, "m": 0.0, "v": 0.0, "maxabs": 0.0, "band": 0.0}
    for k, (off, cnt) in enumerate(zip(z["t_off"], z["t_cnt"])):
        sl = slice(int(off), int(off + cnt))
        name = str(z["names"][k])
        for key, got, ref in (("grads", g, z["g_val"]), ("params", pn, z["p_val"]),
                              ("m", mn, z["m_val"]), ("v", vn, z["v_val"])):
            if key == "params" and bf16:
                # sign-determined samples at the tolerance, the band by the
                # t = 1 bound (tests/gpu_util.py); the RMS is the whole tensor's
                n_el = int(np.prod([r for r in _shape(m.layout, name)]))
                rms = float(z["g_norm"][k]) / np.sqrt(n_el)
                det = np.abs(z["g_val"][sl]) >= SIGN_BAND * rms
                e = _rel(got[sl][det], ref[sl][det]) if det.any() else 0.0
                worst[key] = max(worst[key], e)
                assert e <= tol[key], (name, "params_det", e)
                if (~det).any():
                    du = np.abs((got[sl] - p0[sl]) - (ref[sl] - p0[sl]))[~det]
                    worst["band"] = max(worst["band"], float(np.max(du)) / (2 * lr))
                    assert float(np.max(du)) <= 2 * lr * (1 + 1e-3), (name, "params_band")
                continue
            e = _rel(got[sl], ref[sl])
            worst[key] = max(worst[key], e)
            assert e <= tol[key], (name, key, e)
            ea = maxabs_ratio(got[sl], ref[sl])  # over the samples
            worst["maxabs"] = max(worst["maxabs"], ea / tol[key])
            assert ea <= MAXABS_SAMPLED_C * tol[key], (name, "maxabs_" + key, ea)
    print(cfg["name"], errs, worst)


def _shape(layout, name):
    for nm, _, rows, cols in layout:
        if nm == name:
            return rows, cols
    raise KeyError(name)
