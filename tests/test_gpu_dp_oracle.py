"""GPU parity of the data-parallel step against the float64 oracle, on one GPU.

Two contexts stand for two ranks: each runs llm_grad on its half of the batch,
a device add of the two gradient buffers stands for the exchange (the sum an
all-reduce or a reduce-scatter would deliver), and the update runs as the data
parallel forms run it:
  - llm_adamw with grad_scale 1/2 (the replicated form, DataParallelStep);
  - llm_adamw_range on two chunks of the parameters, one per context (the
    sharded-optimiser form, ShardedDataParallelStep);
  - with clipping: llm_grad_norm_part on each chunk, the two float64 parts
    combined (sum for the L2 norm, max for the L-infinity norm: the all-reduce
    a sharded run makes), then llm_adamw_range_clip on each chunk.
The result must match the oracle's step on the whole batch (the mean of the
two halves' mean gradients is the batch-mean gradient) at the step's
tolerances: loss, gradients, post-AdamW parameters, m and v (MicroGPT in
Rust, Gradient Clipping; Transformer-In-Rust, by global norm; randyGPT, the
L-infinity form, for the clipped cases)."""
import numpy as np
import pytest
import torch

import oracle as O
from oracle import train_terms as TT
from synth import get_config, make_batch, make_params
from tests.gpu_util import TOL, compare

pytestmark = pytest.mark.gpu

CASES = [("c2", dict(batch=4, ctx=64, n_layer=2)),                 # fp32, CUDA-core path
         ("c3", dict(batch=4, ctx=96, n_layer=2)),                 # bf16, head 32
         ("c4", dict(batch=4, ctx=160, n_layer=2, vocab=1000))]    # bf16 GQA, head 64
IDS = ["fp32", "bf16-h32", "bf16-gqa-h64"]


def _setup(name, over):
    from scratch_llama_decoder_b200 import LlamaStep
    full = get_config(name, **over)
    half = dict(full, batch=full["batch"] // 2)
    lay = O.param_layout(full)
    p = make_params(full, lay)
    tok, tgt = make_batch(full)
    ranks = [LlamaStep(half), LlamaStep(half)]
    return full, lay, p, tok.reshape(full["batch"], -1), tgt.reshape(full["batch"], -1), ranks


def _grads(ranks, P, tok, tgt):
    """llm_grad per context on its half; returns the summed gradient and the
    mean of the two losses (the whole batch's mean loss)."""
    hb = tok.shape[0] // 2
    Gs, losses = [], []
    for r, m in enumerate(ranks):
        G = torch.zeros_like(P)
        td = torch.tensor(tok[r * hb:(r + 1) * hb], device="cuda").contiguous()
        yd = torch.tensor(tgt[r * hb:(r + 1) * hb], device="cuda").contiguous()
        losses.append(m.grad(P, G, td, yd))
        Gs.append(G)
    torch.cuda.synchronize()
    G = Gs[0] + Gs[1]  # the exchange's sum
    return G, (losses[0] + losses[1]).item() / 2


def _chunks(n):
    c = ((n + 1) // 2 + 3) // 4 * 4  # 16-byte aligned chunk starts
    return [(0, c), (c, n - c)]


def _oracle(full, p, tok, tgt, clip=None, kind="l2"):
    pp = p.astype(np.float64)
    loss, _, g = O.forward_backward(full, pp, tok, tgt, want_logits=False)
    norm = None
    if clip is not None:
        g, norm, _ = TT.clip(g, clip, kind)
    z = np.zeros_like(pp)
    p2, m2, v2 = O.adamw(pp, g, z, z, 1, full["lr"], full["wd"], full["beta1"], full["beta2"],
                         full["adam_eps"])
    return dict(loss=loss, grads=g, params=p2, m=m2, v=v2, norm=norm)


def _check(full, lay, p, got, ref):
    gpu = {"logits": np.zeros(0), "steps": [got]}
    orc = {"logits": np.zeros(0), "steps": [ref]}
    return compare(full, lay, gpu, orc, prev_params=p.astype(np.float64))


def _state(status, loss, G, P, M, V):
    return dict(status=status, loss=loss, grads=G.double().cpu().numpy(),
                params=P.double().cpu().numpy(), m=M.double().cpu().numpy(),
                v=V.double().cpu().numpy())


@pytest.mark.parametrize("name,over", CASES, ids=IDS)
def test_half_batches_summed_then_adamw_match_the_oracle(name, over):
    full, lay, p, tok, tgt, ranks = _setup(name, over)
    P = torch.tensor(p, device="cuda")
    M, V = torch.zeros_like(P), torch.zeros_like(P)
    G, loss = _grads(ranks, P, tok, tgt)
    ranks[0].adamw(P, G, M, V, 1, full["lr"], full["wd"], grad_scale=0.5)
    st = ranks[0].status() | ranks[1].status()
    _check(full, lay, p, _state(st, loss, G, P, M, V), _oracle(full, p, tok, tgt))
    for m in ranks:
        m.close()


@pytest.mark.parametrize("name,over", CASES, ids=IDS)
def test_half_batches_summed_then_adamw_on_two_chunks_match_the_oracle(name, over):
    full, lay, p, tok, tgt, ranks = _setup(name, over)
    P = torch.tensor(p, device="cuda")
    M, V = torch.zeros_like(P), torch.zeros_like(P)
    G, loss = _grads(ranks, P, tok, tgt)
    for m, (lo, cnt) in zip(ranks, _chunks(P.numel())):
        sl = slice(lo, lo + cnt)
        m.adamw_range(P[sl], G[sl], M[sl], V[sl], 1, full["lr"], full["wd"], grad_scale=0.5)
    st = ranks[0].status() | ranks[1].status()
    _check(full, lay, p, _state(st, loss, G, P, M, V), _oracle(full, p, tok, tgt))
    for m in ranks:
        m.close()


@pytest.mark.parametrize("kind", ["l2", "linf"])
@pytest.mark.parametrize("name,over", CASES, ids=IDS)
def test_sharded_clipping_matches_the_oracle(name, over, kind):
    full, lay, p, tok, tgt, ranks = _setup(name, over)
    ref0 = _oracle(full, p, tok, tgt)
    norm = TT.grad_norm(ref0["grads"], kind)
    clip = 0.5 * norm  # every element's update is scaled
    ref = _oracle(full, p, tok, tgt, clip=clip, kind=kind)
    for m in ranks:
        m.set_grad_clip(clip)
        m.set_grad_clip_mode(1 if kind == "linf" else 0)
    P = torch.tensor(p, device="cuda")
    M, V = torch.zeros_like(P), torch.zeros_like(P)
    G, loss = _grads(ranks, P, tok, tgt)
    parts = [torch.zeros(1, dtype=torch.float64, device="cuda") for _ in ranks]
    chunks = _chunks(P.numel())
    for m, part, (lo, cnt) in zip(ranks, parts, chunks):
        m.grad_norm_part(G[lo:lo + cnt], 0.5, part)
    total = torch.maximum(parts[0], parts[1]) if kind == "linf" else parts[0] + parts[1]
    for m, (lo, cnt) in zip(ranks, chunks):
        sl = slice(lo, lo + cnt)
        m.adamw_range_clip(P[sl], G[sl], M[sl], V[sl], 1, full["lr"], full["wd"], total)
    st = ranks[0].status() | ranks[1].status()
    _check(full, lay, p, _state(st, loss, G, P, M, V), ref)
    tol = TOL[full["compute"]]["grads"]
    for m in ranks:  # both ranks report the whole gradient's norm
        assert abs(m.read_grad_norm() - ref["norm"]) <= tol * ref["norm"]
        m.close()


def test_sharded_clipping_entries_refuse_bad_arguments():
    import scratch_llama_decoder_b200 as L
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c1")
    m = LlamaStep(cfg)
    P = torch.zeros(64, device="cuda")
    part = torch.zeros(2, dtype=torch.float64, device="cuda")
    with pytest.raises(L.LLMError):
        m.grad_norm_part(P[1:9], 1.0, part)          # misaligned gradient range
    with pytest.raises(L.LLMError):
        m.grad_norm_part(P[:8], float("inf"), part)  # non-finite scale
    with pytest.raises(L.LLMError):
        m.grad_norm_part(P[:8], 1.0, part[1:].view(torch.float32)[1:])  # misaligned part
    m.set_grad_clip(1.0)
    rc = L.lib.llm_adamw_range_clip(m.ctx, P.data_ptr(), P.data_ptr(), P.data_ptr(),
                                    P.data_ptr(), 8, 1, 1e-3, 0.0, None)
    assert rc == L.LLM_ERR_ARG  # clipping on needs the combined part
    m.close()
