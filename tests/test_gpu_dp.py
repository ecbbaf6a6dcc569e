"""GPU checks of the data-parallel entry points at one rank (C ABI):
llm_grad then llm_adamw gives llm_step's results bit for bit, grad_scale
undoes an exact scaling of the gradient, DataParallelStep without a process
group is the plain step, and an error word brought in by llm_flag_in skips the
update.  (Every call in this environment has one GPU; the rank logic with two
ranks is tested on CPU in test_dp_ranks.py.)"""
import pytest
import torch

import oracle as O
from synth import get_config, make_batch, make_params

pytestmark = pytest.mark.gpu

CFG = dict(name="c3", over=dict(batch=2, ctx=96, n_layer=2))


def _setup():
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config(CFG["name"], **CFG["over"])
    p = make_params(cfg, O.param_layout(cfg))
    tok, tgt = make_batch(cfg)
    m = LlamaStep(cfg)
    P = torch.tensor(p, device="cuda")
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    return cfg, m, P, G, M, V, torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda")


def _state(P, G, M, V, loss):
    return [x.clone().cpu() for x in (P, G, M, V, loss)]


def test_grad_then_adamw_is_step():
    cfg, m, P, G, M, V, td, yd = _setup()
    loss = torch.zeros(1, device="cuda")
    for t in range(1, 4):
        m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"], loss)
    ref = _state(P, G, M, V, loss)
    assert m.status() == 0
    m.close()
    for variant in ("plain", "scaled"):
        cfg, m, P, G, M, V, td, yd = _setup()
        for t in range(1, 4):
            m.grad(P, G, td, yd, loss)
            if variant == "plain":
                m.adamw(P, G, M, V, t, cfg["lr"], cfg["wd"])
            else:  # twice the gradient, halved by grad_scale: exact in float
                G.mul_(2.0)
                m.adamw(P, G, M, V, t, cfg["lr"], cfg["wd"], grad_scale=0.5)
        assert m.status() == 0
        for a, b in zip(_state(P, G, M, V, loss), ref):
            assert torch.equal(a, b), variant
        m.close()


def test_data_parallel_step_on_one_rank_is_step():
    from scratch_llama_decoder_b200.dp import DataParallelStep
    cfg, m, P, G, M, V, td, yd = _setup()
    loss = torch.zeros(1, device="cuda")
    for t in range(1, 3):
        m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"], loss)
    ref = _state(P, G, M, V, loss)
    m.close()
    cfg, m, P, G, M, V, td, yd = _setup()
    dp = DataParallelStep(m)
    assert dp.world == 1
    for t in range(1, 3):
        dp.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"], loss)
    torch.cuda.synchronize()
    for a, b in zip(_state(P, G, M, V, loss), ref):
        assert torch.equal(a, b)
    m.close()


def test_error_word_in_and_out():
    import scratch_llama_decoder_b200 as L
    cfg, m, P, G, M, V, td, yd = _setup()
    loss = torch.zeros(1, device="cuda")
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    m.grad(P, G, td, yd, loss)
    m.flag_out(word)
    assert int(word.item()) == 0
    # another rank's error: the update is skipped
    P0, M0, V0 = P.clone(), M.clone(), V.clone()
    m.flag_in(torch.ones(1, dtype=torch.int32, device="cuda"))
    m.adamw(P, G, M, V, 1, cfg["lr"], cfg["wd"])
    torch.cuda.synchronize()
    assert torch.equal(P, P0) and torch.equal(M, M0) and torch.equal(V, V0)
    assert m.status() == 0  # the local status only reports local errors
    # a bad token here: the word says so
    bad = td.clone()
    bad[0, 0] = cfg["vocab"]
    m.grad(P, G, bad, yd, loss)
    m.flag_out(word)
    assert int(word.item()) != 0
    assert m.status() == L.LLM_ERR_TOKEN
    assert L.lib.llm_adamw(m.ctx, P.data_ptr(), G.data_ptr(), M.data_ptr(), V.data_ptr(), 0,
                           1e-3, 0.1, 1.0) == L.LLM_ERR_ARG
    assert L.lib.llm_adamw(m.ctx, P.data_ptr(), G.data_ptr(), M.data_ptr(), V.data_ptr(), 1,
                           1e-3, 0.1, float("inf")) == L.LLM_ERR_ARG
    m.close()


def test_sharded_step_on_one_rank_is_step():
    """ShardedDataParallelStep without a process group (one chunk holding
    every parameter) gives llm_step's parameters, gradient and moments bit
    for bit; its buffers are padded past the parameters."""
    from scratch_llama_decoder_b200.dp import ShardedDataParallelStep
    cfg, m, P, G, M, V, td, yd = _setup()
    loss = torch.zeros(1, device="cuda")
    for t in range(1, 3):
        m.step(P, G, M, V, t, td, yd, cfg["lr"], cfg["wd"], loss)
    ref = _state(P, G, M, V, loss)
    m.close()
    cfg, m, P, G, M, V, td, yd = _setup()
    dp = ShardedDataParallelStep(m, m.n_params)
    assert dp.world == 1 and dp.count == m.n_params and dp.chunk % 4 == 0
    Pp, Gp, Mp, Vp = dp.buffers()
    n = m.n_params
    Pp[:n].copy_(P)
    for t in range(1, 3):
        dp.step(Pp, Gp, Mp, Vp, t, td, yd, cfg["lr"], cfg["wd"], loss)
    torch.cuda.synchronize()
    got = [Pp[:n].cpu(), Gp[:n].cpu(), Mp[:n].cpu(), Vp[:n].cpu(), loss.cpu()]
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    assert not Gp[n:].any()  # the pad past the parameters stays zero
    m.close()


def test_grad_buckets_events_and_identical_gradient():
    """llm_set_grad_buckets: the gradient is bit-identical with the bucket
    events on, and a second stream that waits for bucket k (llm_grad_bucket_wait)
    reads that bucket's final values; waiting before a bucketed llm_grad is
    refused."""
    import scratch_llama_decoder_b200 as L
    cfg, m, P, G, M, V, td, yd = _setup()
    loss = torch.zeros(1, device="cuda")
    side = torch.cuda.Stream()
    with pytest.raises(L.LLMError):
        m.grad_bucket_wait(0, side)
    m.grad(P, G, td, yd, loss)
    ref = G.clone()
    m.set_grad_buckets(True)
    buckets = m.grad_buckets()
    assert len(buckets) == cfg["n_layer"] + 2
    G.zero_()
    m.grad(P, G, td, yd, loss)
    copies = []
    for k, (off, cnt) in enumerate(buckets):
        m.grad_bucket_wait(k, side)
        with torch.cuda.stream(side):
            copies.append(G[off:off + cnt].clone())
    torch.cuda.synchronize()
    assert m.status() == 0
    assert torch.equal(G, ref)
    for (off, cnt), c in zip(buckets, copies):
        assert torch.equal(c, ref[off:off + cnt])
    with pytest.raises(L.LLMError):
        m.grad_bucket_wait(len(buckets), side)
    m.set_grad_buckets(False)
    with pytest.raises(L.LLMError):
        m.grad_bucket_wait(0, side)
    m.close()
