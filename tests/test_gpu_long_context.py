"""GPU parity beyond the trained context: RoPE position interpolation
(llm_set_rope_scale: positions t / factor in the forward, the backward and
decode) against the oracle with the same scale, and a 4096-position context
(past the 2048 of the largest workload) against the oracle's forward."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import get_config, make_batch, make_params
from tests.gpu_util import TOL, compare, rel, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over", [("c1", dict(batch=2)),
                                       ("c3", dict(batch=2, ctx=96, n_layer=2)),
                                       ("c4", dict(batch=1, ctx=160, n_layer=1))])
def test_rope_scale_step_matches_oracle(name, over):
    cfg = get_config(name, rope_scale=2.0, **over)
    lay = O.param_layout(cfg)
    p = make_params(cfg, lay)
    tok, tgt = make_batch(cfg)
    gpu = run_gpu(cfg, p, tok, tgt, steps=1)
    ref = run_oracle(cfg, p, tok, tgt, steps=1)
    w = compare(cfg, lay, gpu, ref, prev_params=p.astype(np.float64))
    print(name, w)


def test_context_4096_forward_matches_oracle():
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c4", batch=1, ctx=4096, n_layer=1)
    lay = O.param_layout(cfg)
    p = make_params(cfg, lay)
    tok, tgt = make_batch(cfg)
    loss_ref, zref, _ = O.forward_backward(cfg, p, tok, tgt, want_grads=False)
    m = LlamaStep(cfg)
    P = torch.tensor(p, device="cuda")
    z = m.forward(P, torch.tensor(tok, device="cuda")).double().cpu().numpy().reshape(zref.shape)
    tol = TOL["bf16"]
    assert rel(z, zref) <= tol["logits"]
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    loss = m.step(P, G, M, V, 1, torch.tensor(tok, device="cuda"),
                  torch.tensor(tgt, device="cuda"), cfg["lr"], cfg["wd"])
    assert m.status() == 0
    assert abs(float(loss.item()) - loss_ref) <= tol["loss"] * abs(loss_ref)
    assert torch.isfinite(G).all()
    m.close()


def test_decode_with_rope_scale_matches_full_forward():
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c4", batch=2, ctx=128, n_layer=2, rope_scale=2.0)
    p = make_params(cfg, O.param_layout(cfg))
    tok, _ = make_batch(cfg)
    tok = tok.reshape(2, 128)
    _, zref, _ = O.forward_backward(cfg, p, tok, want_grads=False)
    zref = zref.reshape(2, 128, -1)
    m = LlamaStep(cfg)
    m.set_rope_scale(2.0)
    P = torch.tensor(p, device="cuda")
    m.forward(P, torch.tensor(tok, device="cuda"))
    worst = 0.0
    for t in range(64, 128):
        z = m.decode(P, torch.tensor(tok[:, t], device="cuda"), t).double().cpu().numpy()
        worst = max(worst, max(rel(z[b], zref[b, t]) for b in range(2)))
    assert m.status() == 0 and worst <= TOL["bf16"]["logits"], worst
    import scratch_llama_decoder_b200 as L
    assert L.lib.llm_set_rope_scale(m.ctx, 0.0) == L.LLM_ERR_ARG
    assert L.lib.llm_set_rope_scale(m.ctx, float("inf")) == L.LLM_ERR_ARG
    m.close()


@pytest.mark.parametrize("dropout", [0.0, 0.2])
def test_recompute_is_bit_identical_to_stored_activations(dropout):
    from scratch_llama_decoder_b200 import LlamaStep
    res = []
    for rc in (0, 1):
        cfg = get_config("c3", batch=2, ctx=96, n_layer=3, recompute=rc)
        p = make_params(cfg, O.param_layout(cfg))
        tok, tgt = make_batch(cfg)
        m = LlamaStep(cfg)
        if dropout:
            m.set_dropout(dropout, 77)
        P = torch.tensor(p, device="cuda")
        G, M, V = (torch.zeros_like(P) for _ in range(3))
        loss = torch.zeros(1, device="cuda")
        td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
        for t in (1, 2):
            m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"], loss)
        assert m.status() == 0
        res.append([x.cpu() for x in (P, G, M, V, loss)])
        if rc:
            import scratch_llama_decoder_b200 as L
            lg = torch.empty(2, cfg["vocab"], device="cuda")
            assert L.lib.llm_decode(m.ctx, P.data_ptr(), td[:, 0].contiguous().data_ptr(), 0,
                                    lg.data_ptr()) == L.LLM_ERR_CONFIG
        m.close()
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_decode_refuses_a_hidden_size_past_its_split_plan():
    """Decode adds at most 16 K slices of 1024 rows per product: a d_ff past
    16384 is refused on the host (nothing launched); training still runs."""
    import scratch_llama_decoder_b200 as L
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c1", batch=1, ctx=8, d_ff=16448)
    m = LlamaStep(cfg)
    P = torch.tensor(make_params(cfg, O.param_layout(cfg)), device="cuda")
    tok, _ = make_batch(cfg)
    td = torch.tensor(tok, device="cuda")
    m.forward(P, td)
    lg = torch.empty(1, cfg["vocab"], device="cuda")
    assert L.lib.llm_decode(m.ctx, P.data_ptr(), td[:, 0].contiguous().data_ptr(), 0,
                            lg.data_ptr()) == L.LLM_ERR_CONFIG
    assert m.status() == 0
    m.close()
