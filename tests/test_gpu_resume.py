"""Resume equals an uninterrupted run (strata, train/optim: a resumed run must
match the uninterrupted one): the library keeps no training state of its own
beyond the caller's params, m, v and the step count t -- and, with dropout,
the mask counter (llm_get_dropout_calls / llm_set_dropout_calls) -- so steps
1..4 in one context equal steps 1..2, a checkpoint of those to host memory, a
new context and steps 3..4, bit for bit."""
import pytest
import torch

import oracle as O
from synth import get_config, make_batch, make_params

pytestmark = pytest.mark.gpu

P_DROP, SEED = 0.15, 0x0DD5EED


def _ctx(cfg, dropout):
    from scratch_llama_decoder_b200 import LlamaStep
    m = LlamaStep(cfg)
    if dropout:
        m.set_dropout(P_DROP, SEED)
    return m


@pytest.mark.parametrize("dropout", [False, True])
@pytest.mark.parametrize("name,over", [("c1", dict(batch=2)),
                                       ("c4", dict(batch=1, ctx=96, n_layer=2))])
def test_resumed_run_equals_uninterrupted_run(name, over, dropout):
    cfg = get_config(name, **over)
    p = make_params(cfg, O.param_layout(cfg))
    tok, tgt = make_batch(cfg)
    td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
    lr, wd = cfg["lr"], cfg["wd"]

    def fresh():
        P = torch.tensor(p, device="cuda")
        return P, torch.zeros_like(P), torch.zeros_like(P), torch.zeros_like(P)

    # uninterrupted
    m = _ctx(cfg, dropout)
    P, G, M, V = fresh()
    losses = []
    for t in range(1, 5):
        losses.append(float(m.step(P, G, M, V, t, td, yd, lr, wd).item()))
    assert m.status() == 0
    ref = [x.cpu() for x in (P, G, M, V)]
    m.close()
    # steps 1..2, checkpoint to host, a new context, steps 3..4
    m = _ctx(cfg, dropout)
    P, G, M, V = fresh()
    got = []
    for t in (1, 2):
        got.append(float(m.step(P, G, M, V, t, td, yd, lr, wd).item()))
    ck = {"P": P.cpu(), "M": M.cpu(), "V": V.cpu(), "t": 2,
          "calls": m.dropout_calls()}
    assert ck["calls"] == (2 if dropout else 0)
    m.close()
    del P, G, M, V
    m = _ctx(cfg, dropout)
    m.set_dropout_calls(ck["calls"])
    P, M, V = (ck[k].cuda() for k in ("P", "M", "V"))
    G = torch.zeros_like(P)
    for t in (3, 4):
        got.append(float(m.step(P, G, M, V, t, td, yd, lr, wd).item()))
    assert m.status() == 0
    for a, b in zip([x.cpu() for x in (P, G, M, V)], ref):
        assert torch.equal(a, b)
    assert got == losses
    if dropout:  # without the counter the resumed masks would be the first ones
        m.set_dropout_calls(0)
        assert m.dropout_calls() == 0
    m.close()


def test_dropout_calls_arguments():
    import scratch_llama_decoder_b200 as L
    m = _ctx(get_config("c1"), True)
    assert L.lib.llm_set_dropout_calls(m.ctx, -1) == L.LLM_ERR_ARG
    assert L.lib.llm_set_dropout_calls(m.ctx, 1 << 31) == L.LLM_ERR_ARG
    assert L.lib.llm_set_dropout_calls(m.ctx, 7) == 0
    assert m.dropout_calls() == 7
    m.close()
