"""GPU parity of L-infinity gradient clipping (llm_set_grad_clip_mode, randyGPT:
clipping by the largest absolute gradient element) against the oracle: two
clipped steps, the reported norm exactly (a maximum is order-free), and the
mode switch after a captured step graph."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import train_terms as TT
from synth import get_config, make_batch, make_params
from tests.gpu_util import TOL, compare

pytestmark = pytest.mark.gpu


def _run(cfg, p, tok, tgt, clip, steps, mode):
    from scratch_llama_decoder_b200 import LlamaStep
    m = LlamaStep(cfg)
    m.set_grad_clip_mode(mode)
    m.set_grad_clip(clip)
    P = torch.tensor(p, device="cuda")
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
    logits = m.forward(P, td).double().cpu().numpy().reshape(-1, cfg["vocab"])
    out = {"logits": logits, "steps": []}
    for t in range(1, steps + 1):
        loss = m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"])
        out["steps"].append(dict(status=m.status(), loss=float(loss.item()),
                                 grads=G.double().cpu().numpy(), params=P.double().cpu().numpy(),
                                 m=M.double().cpu().numpy(), v=V.double().cpu().numpy(),
                                 norm=m.read_grad_norm()))
    m.close()
    return out


@pytest.mark.parametrize("name,over", [("c1", {}), ("c3", dict(batch=2, ctx=96, n_layer=2))])
def test_linf_clipped_steps_match_oracle(name, over):
    cfg = get_config(name, **over)
    lay = O.param_layout(cfg)
    p = make_params(cfg, lay)
    tok, tgt = make_batch(cfg)
    _, _, g = O.forward_backward(cfg, p, tok, tgt, want_logits=False)
    clip = 0.25 * float(np.abs(g).max())  # inside the clipping regime at both steps
    gpu = _run(cfg, p, tok, tgt, clip, 2, 1)
    # the oracle with L-infinity clipping before each AdamW
    pp = p.astype(np.float64)
    m = np.zeros_like(pp)
    v = np.zeros_like(pp)
    _, logits, _ = O.forward_backward(cfg, pp, tok, tgt, want_grads=False)
    ref = {"logits": logits, "steps": []}
    for t in (1, 2):
        loss, _, gr = O.forward_backward(cfg, pp, tok, tgt, want_logits=False)
        gc, n, _ = TT.clip(gr, clip, "linf")
        pp, m, v = O.adamw(pp, gc, m, v, t, cfg["lr"], cfg["wd"])
        ref["steps"].append(dict(loss=loss, grads=gc, params=pp.copy(), m=m.copy(), v=v.copy(),
                                 norm=n))
    compare(cfg, lay, gpu, ref, prev_params=p.astype(np.float64))
    for gs, rs in zip(gpu["steps"], ref["steps"]):
        # the reported norm is the largest |g| before clipping
        assert abs(gs["norm"] - rs["norm"]) <= TOL[cfg["compute"]]["grads"] * rs["norm"]
        if rs["norm"] > clip:  # clipped: the largest stored |g| is the threshold
            assert np.abs(gs["grads"]).max() == pytest.approx(clip, rel=1e-6)


def test_clip_mode_arguments():
    import scratch_llama_decoder_b200 as L
    m = L.LlamaStep(get_config("c1"))
    assert L.lib.llm_set_grad_clip_mode(m.ctx, 2) == L.LLM_ERR_ARG
    assert L.lib.llm_set_grad_clip_mode(m.ctx, 1) == 0
    assert L.lib.llm_set_grad_clip_mode(m.ctx, 0) == 0
    m.close()
