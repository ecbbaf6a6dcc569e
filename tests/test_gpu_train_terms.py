"""GPU parity of global-norm gradient clipping inside llm_step (C ABI)
against the float64 oracle: gradients clipped with the oracle's formula
(MicroGPT in Rust, Gradient Clipping) before AdamW, the reported norm, a
threshold above the norm leaving the step bit-identical to no clipping, and
a changed threshold taking effect after a step graph was captured."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import get_config, make_batch, make_params
from tests.gpu_util import TOL, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def _inputs(cfg):
    lay = O.param_layout(cfg)
    return lay, make_params(cfg, lay), *make_batch(cfg)


@pytest.mark.parametrize("name,over", [("c1", {}), ("c3", dict(batch=2, ctx=96, n_layer=2)),
                                       ("c4", dict(batch=1, ctx=128, n_layer=1))])
def test_clipped_steps_match_oracle(name, over):
    cfg = get_config(name, **over)
    lay, p, tok, tgt = _inputs(cfg)
    _, _, g = O.forward_backward(cfg, p, tok, tgt, want_logits=False)
    max_norm = 0.5 * float(np.linalg.norm(g))  # well inside the clipping regime
    gpu = run_gpu(cfg, p, tok, tgt, steps=2, clip=max_norm)
    ref = run_oracle(cfg, p, tok, tgt, steps=2, clip=max_norm)
    w = compare(cfg, lay, gpu, ref, prev_params=p.astype(np.float64))
    tol = TOL[cfg["compute"]]["grads"]
    for gs, rs in zip(gpu["steps"], ref["steps"]):
        assert abs(gs["norm"] - rs["norm"]) <= tol * rs["norm"], (gs["norm"], rs["norm"])
        # the stored gradient is the clipped one: its norm is the threshold
        assert np.linalg.norm(gs["grads"]) == pytest.approx(max_norm, rel=1e-4)
    print(name, w)


def test_threshold_above_norm_is_bit_identical_to_no_clipping():
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c3", batch=2, ctx=64, n_layer=1)
    lay, p, tok, tgt = _inputs(cfg)
    res = []
    for clip in (None, 1e30):
        m = LlamaStep(cfg)
        if clip is not None:
            m.set_grad_clip(clip)
        P = torch.tensor(p, device="cuda")
        G, M, V = (torch.zeros_like(P) for _ in range(3))
        td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
        for t in range(1, 4):
            m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"])
        assert m.status() == 0
        if clip is not None:
            assert 0.0 < m.read_grad_norm() < 1e30
        res.append([x.cpu() for x in (P, G, M, V)])
        m.close()
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_threshold_change_after_graph_capture():
    import scratch_llama_decoder_b200 as L
    cfg = get_config("c3", batch=2, ctx=64, n_layer=1)
    lay, p, tok, tgt = _inputs(cfg)
    m = L.LlamaStep(cfg)
    with pytest.raises(L.LLMError):
        m.read_grad_norm()  # no clipped step yet
    P = torch.tensor(p, device="cuda")
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
    for t in (1, 2, 3):  # the second call captures the step graph, the third replays it
        m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"])
    n_free = float(torch.linalg.vector_norm(G.double()))
    m.set_grad_clip(0.25 * n_free)
    m.step(P, G, M, V, 4, td, yd, cfg["lr"], cfg["wd"])
    assert m.status() == 0
    n4 = m.read_grad_norm()
    assert n4 > 0.25 * n_free
    assert float(torch.linalg.vector_norm(G.double())) == pytest.approx(0.25 * n_free, rel=1e-4)
    m.set_grad_clip(0.0)  # off again: the gradient is left as computed
    m.step(P, G, M, V, 5, td, yd, cfg["lr"], cfg["wd"])
    assert float(torch.linalg.vector_norm(G.double())) > 0.25 * n_free * 1.5
    assert L.lib.llm_set_grad_clip(m.ctx, float("nan")) == L.LLM_ERR_ARG
    m.close()
