"""GPU parity of inverted dropout (llm_set_dropout) through the C ABI against
the float64 oracle with the same masks: the loss and gradients of training
calls 0 and 1 (different masks) at fp32 and bf16, MHA and GQA; rate 0 is the
step without dropout bit for bit; evaluation (llm_forward) never drops; a
replayed step graph draws the same masks as individual launches; contexts over
halves of a batch with sequence offsets (llm_set_dropout_offset, as the
data-parallel wrappers set them) draw the whole batch's masks."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import get_config, make_batch, make_params
from tests.gpu_util import TOL, rel

pytestmark = pytest.mark.gpu

P_DROP, SEED = 0.2, 0x5EED_1234_ABCD


def _setup(cfg, stream=None):
    from scratch_llama_decoder_b200 import LlamaStep
    lay = O.param_layout(cfg)
    p = make_params(cfg, lay)
    tok, tgt = make_batch(cfg)
    m = LlamaStep(cfg, stream=stream)
    torch.cuda.synchronize()
    return lay, p, tok, tgt, m


@pytest.mark.parametrize("name,over", [("c1", dict(batch=2)),
                                       ("c3", dict(batch=2, ctx=64, n_layer=2)),
                                       ("c4", dict(batch=1, ctx=96, n_layer=2)),
                                       # several 64-row tiles with ragged tails (head 32, head 64 GQA)
                                       ("c3", dict(batch=1, ctx=130, n_layer=1)),
                                       ("c4", dict(batch=1, ctx=200, n_layer=1)),
                                       # the tiled fp32 kernels: T % 4 == 0 (a mask group
                                       # per 4 keys) and T % 4 != 0 (a group per element)
                                       ("c2", dict(batch=2, ctx=68, n_layer=2)),
                                       ("c2", dict(batch=1, ctx=131, n_layer=1))])
def test_dropout_grads_match_oracle(name, over):
    cfg = get_config(name, **over)
    lay, p, tok, tgt, m = _setup(cfg)
    tol = TOL[cfg["compute"]]
    m.set_dropout(P_DROP, SEED)
    P = torch.tensor(p, device="cuda")
    G = torch.zeros_like(P)
    td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
    pd = float(np.float32(P_DROP))
    gs = []
    for n in range(2):  # training calls 0 and 1 draw different masks
        loss = m.grad(P, G, td, yd)
        assert m.status() == 0
        lr_, _, gr_ = O.forward_backward(cfg, p, tok, tgt, want_logits=False,
                                         dropout=(pd, SEED, n))
        assert abs(float(loss.item()) - lr_) <= tol["loss"] * abs(lr_), (n, loss.item(), lr_)
        g = G.double().cpu().numpy()
        for nm, off, rows, cols in lay:
            e = rel(g[off:off + rows * cols], gr_[off:off + rows * cols])
            assert e <= tol["grads"], (n, nm, e)
        gs.append(g)
    # the call number reached the masks: the two calls' gradients differ
    assert rel(gs[1], gs[0]) > 10 * tol["grads"]
    m.close()


def test_zero_rate_and_evaluation_do_not_drop():
    cfg = get_config("c3", batch=2, ctx=64, n_layer=1)
    res = []
    for rate in (None, 0.0):
        lay, p, tok, tgt, m = _setup(cfg)
        if rate is not None:
            m.set_dropout(rate, SEED)
        P = torch.tensor(p, device="cuda")
        G, M, V = (torch.zeros_like(P) for _ in range(3))
        td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
        for t in (1, 2):
            m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"])
        res.append([x.cpu() for x in (P, G, M, V)])
        m.close()
    for a, b in zip(*res):
        assert torch.equal(a, b)
    # llm_forward is evaluation: the same logits with dropout set
    lay, p, tok, tgt, m = _setup(cfg)
    P = torch.tensor(p, device="cuda")
    td = torch.tensor(tok, device="cuda")
    z0 = m.forward(P, td).clone()
    m.set_dropout(0.5, SEED)
    z1 = m.forward(P, td)
    assert torch.equal(z0, z1)
    m.close()


def test_dropout_step_graph_matches_launches():
    cfg = get_config("c3", batch=2, ctx=64, n_layer=2)
    res = []
    for graphs in (True, False):
        stream = torch.cuda.Stream()
        lay, p, tok, tgt, m = _setup(cfg, stream=stream)
        m.set_graphs(graphs)
        m.set_dropout(P_DROP, SEED)
        P = torch.tensor(p, device="cuda")
        G, M, V = (torch.zeros_like(P) for _ in range(3))
        td, yd = torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")
        loss = torch.zeros(1, device="cuda")  # one buffer: the graph key stays the same
        torch.cuda.synchronize()
        losses = []
        for t in (1, 2, 3, 4):  # the second call captures, the later ones replay
            m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"], loss)
            stream.synchronize()
            losses.append(float(loss.item()))
        assert m.status() == 0
        res.append([x.cpu() for x in (P, G, M, V)] + [torch.tensor(losses)])
        m.close()
    for a, b in zip(*res):
        assert torch.equal(a, b)


def test_set_dropout_arguments():
    import scratch_llama_decoder_b200 as L
    cfg = get_config("c1")
    m = L.LlamaStep(cfg)
    for bad in (1.0, -0.1, float("nan"), 1.5):
        assert L.lib.llm_set_dropout(m.ctx, bad, 1) == L.LLM_ERR_ARG
    assert L.lib.llm_set_dropout(m.ctx, 0.0, 1) == 0
    m.close()


@pytest.mark.parametrize("name,over", [("c4", dict(batch=2, ctx=96, n_layer=1)),   # mma, T % 4 == 0
                                       ("c3", dict(batch=2, ctx=66, n_layer=1)),   # mma, T % 4 != 0
                                       ("c2", dict(batch=2, ctx=68, n_layer=1))])  # fp32 tiled
def test_halves_with_offsets_draw_the_whole_batch_masks(name, over):
    from scratch_llama_decoder_b200 import LlamaStep
    full = get_config(name, **over)
    half = dict(full, batch=full["batch"] // 2)
    hb = half["batch"]
    lay = O.param_layout(full)
    p = make_params(full, lay)
    tok, tgt = make_batch(full)
    tok, tgt = tok.reshape(full["batch"], -1), tgt.reshape(full["batch"], -1)
    tol = TOL[full["compute"]]
    ranks = [LlamaStep(half), LlamaStep(half)]
    P = torch.tensor(p, device="cuda")
    lr_, _, gr_ = O.forward_backward(full, p, tok, tgt, want_logits=False,
                                     dropout=(float(np.float32(P_DROP)), SEED, 0))

    def halves(offsets):
        G, loss = torch.zeros_like(P), 0.0
        for r, m in enumerate(ranks):
            m.set_dropout(P_DROP, SEED)  # the mask counter restarts at 0
            m.set_dropout_offset(offsets[r])
            Gr = torch.zeros_like(P)
            td = torch.tensor(tok[r * hb:(r + 1) * hb], device="cuda").contiguous()
            yd = torch.tensor(tgt[r * hb:(r + 1) * hb], device="cuda").contiguous()
            loss += float(m.grad(P, Gr, td, yd).item()) / 2
            assert m.status() == 0
            G += Gr
        return (G / 2).double().cpu().numpy(), loss

    g, loss = halves([0, hb])  # the mean of the halves' mean gradients
    assert abs(loss - lr_) <= tol["loss"] * abs(lr_), (loss, lr_)
    for nm, off, rows, cols in lay:
        e = rel(g[off:off + rows * cols], gr_[off:off + rows * cols])
        assert e <= tol["grads"], (nm, e)
    # without the offset the second half draws the first half's masks
    g0, _ = halves([0, 0])
    assert rel(g0, gr_) > 10 * tol["grads"]
    for m in ranks:
        m.close()


def test_dropout_offset_arguments():
    import scratch_llama_decoder_b200 as L
    lay, p, tok, tgt, m = _setup(get_config("c1"))
    assert L.lib.llm_set_dropout_offset(m.ctx, -1) == L.LLM_ERR_ARG
    assert L.lib.llm_set_dropout_offset(m.ctx, 1 << 31) == L.LLM_ERR_ARG
    assert L.lib.llm_set_dropout_offset(None, 0) == L.LLM_ERR_ARG
    assert L.lib.llm_set_dropout_offset(m.ctx, 5) == 0
    m.close()
