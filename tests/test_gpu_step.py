"""GPU parity of the full training step (C ABI) against the float64 oracle.

Live comparisons at sizes the oracle finishes in seconds; each spans several
GEMM and attention tiles.  Full-size workloads are compared on sampled
outputs in test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

from synth import get_config, make_batch, make_params
from tests.gpu_util import compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def _inputs(cfg, seed=None):
    import oracle as O
    lay = O.param_layout(cfg)
    p = make_params(cfg, lay, seed=seed)
    tok, tgt = make_batch(cfg, seed=seed)
    return lay, p, tok, tgt


def test_tiny_three_steps():
    cfg = get_config("c1")
    lay, p, tok, tgt = _inputs(cfg)
    gpu = run_gpu(cfg, p, tok, tgt, steps=3)
    ref = run_oracle(cfg, p, tok, tgt, steps=3)
    w = compare(cfg, lay, gpu, ref, prev_params=p.astype(np.float64))
    print("tiny", w)


# Reduced-batch versions of the workloads: every layer, head and vocabulary
# size of the full config, fewer sequences.
REDUCED = [
    ("c2", dict(batch=2)),
    ("c3", dict(batch=2)),
    ("c4", dict(batch=1, n_layer=2)),
    ("c5", dict(batch=1, ctx=256, n_layer=2)),
]


@pytest.mark.parametrize("name,over", REDUCED, ids=[r[0] for r in REDUCED])
def test_reduced_workloads(name, over):
    cfg = get_config(name, **over)
    lay, p, tok, tgt = _inputs(cfg)
    gpu = run_gpu(cfg, p, tok, tgt, steps=1)
    ref = run_oracle(cfg, p, tok, tgt, steps=1)
    w = compare(cfg, lay, gpu, ref, prev_params=p.astype(np.float64))
    print(name, w)


# Ragged and degenerate shapes: token counts that are not tile multiples,
# a single position, no layers, MQA.
EDGE = [
    ("ragged_bf16", "c3", dict(batch=1, ctx=200)),
    ("ragged_fp32", "c2", dict(batch=3, ctx=37, n_layer=2)),
    ("T1_bf16", "c4", dict(batch=4, ctx=1, n_layer=1)),
    ("L0_bf16", "c3", dict(batch=2, ctx=64, n_layer=0)),
    ("mqa_bf16", "c4", dict(batch=1, ctx=128, n_layer=1, n_kv_head=1)),
    ("gqa_fp32", "c2", dict(batch=1, ctx=64, n_layer=2, n_head=8, n_kv_head=2)),
]


@pytest.mark.parametrize("tag,name,over", EDGE, ids=[e[0] for e in EDGE])
def test_edge_shapes(tag, name, over):
    cfg = get_config(name, **over)
    lay, p, tok, tgt = _inputs(cfg)
    gpu = run_gpu(cfg, p, tok, tgt, steps=1)
    ref = run_oracle(cfg, p, tok, tgt, steps=1)
    compare(cfg, lay, gpu, ref, prev_params=p.astype(np.float64))


def test_forward_has_no_side_effects_and_is_deterministic():
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c3", batch=2)
    lay, p, tok, tgt = _inputs(cfg)
    m = LlamaStep(cfg)
    P = torch.tensor(p, device="cuda")
    P0 = P.clone()
    td = torch.tensor(tok, device="cuda")
    yd = torch.tensor(tgt, device="cuda")
    z1 = m.forward(P, td).clone()
    z2 = m.forward(P, td).clone()
    assert torch.equal(P, P0)
    assert torch.equal(z1, z2)
    # two identical steps from the same state are bit-identical
    outs = []
    for _ in range(2):
        Pc = P0.clone()
        G, M, V = (torch.zeros_like(P0) for _ in range(3))
        loss = m.step(Pc, G, M, V, 1, td, yd, 1e-4, 0.1)
        outs.append((loss.clone(), G.clone(), Pc.clone()))
    assert m.status() == 0
    assert torch.equal(outs[0][0], outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])
    assert torch.equal(outs[0][2], outs[1][2])


def test_bad_token_reported_and_update_skipped():
    from scratch_llama_decoder_b200 import LLM_ERR_TOKEN, LlamaStep
    cfg = get_config("c1")
    lay, p, tok, tgt = _inputs(cfg)
    m = LlamaStep(cfg)
    P = torch.tensor(p, device="cuda")
    P0 = P.clone()
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    bad = tok.copy()
    bad[0, 3] = cfg["vocab"] + 5
    m.step(P, G, M, V, 1, torch.tensor(bad, device="cuda"), torch.tensor(tgt, device="cuda"),
           1e-2, 0.1)
    assert m.status() == LLM_ERR_TOKEN
    assert torch.equal(P, P0) and torch.count_nonzero(M) == 0
    badt = tgt.copy()
    badt[0, 0] = -1
    m.step(P, G, M, V, 1, torch.tensor(tok, device="cuda"), torch.tensor(badt, device="cuda"),
           1e-2, 0.1)
    assert m.status() == LLM_ERR_TOKEN
    assert torch.equal(P, P0)
    # a clean step afterwards works and clears the status
    m.step(P, G, M, V, 1, torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda"),
           1e-2, 0.1)
    assert m.status() == 0
    assert not torch.equal(P, P0)


def test_nonfinite_loss_reported_and_update_skipped():
    from scratch_llama_decoder_b200 import LLM_ERR_NONFINITE, LlamaStep
    cfg = get_config("c1")
    lay, p, tok, tgt = _inputs(cfg)
    off = [o for n, o, r, k in lay if n == "Wlm"][0]
    p[off + 3] = np.inf
    m = LlamaStep(cfg)
    P = torch.tensor(p, device="cuda")
    P0 = P.clone()
    G, M, V = (torch.zeros_like(P) for _ in range(3))
    m.step(P, G, M, V, 1, torch.tensor(tok, device="cuda"), torch.tensor(tgt, device="cuda"),
           1e-2, 0.1)
    assert m.status() == LLM_ERR_NONFINITE
    assert torch.equal(P, P0) and torch.count_nonzero(V) == 0


@pytest.mark.parametrize("name", ["c2", "c5"])
def test_init_statistics(name):
    """llm_init: matrices ~ N(0, std) (Wo, W2 scaled by 1/sqrt(2L) when asked),
    gains exactly 1.  Mean and std within 5 standard errors per tensor."""
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config(name, batch=1, ctx=16)
    m = LlamaStep(cfg)
    P = m.new_params()
    m.init(P, 1234, cfg["init_std"], cfg["scale_out_proj"])
    assert m.status() == 0
    p = P.double().cpu().numpy()
    for nm, off, r, k in m.layout:
        x = p[off:off + r * k]
        base = nm.split(".")[-1]
        if base in ("g1", "g2", "gf"):
            assert np.all(x == 1.0)
            continue
        s = cfg["init_std"]
        if cfg["scale_out_proj"] and base in ("Wo", "W2"):
            s /= np.sqrt(2 * cfg["n_layer"])
        n = x.size
        assert abs(x.mean()) < 5 * s / np.sqrt(n), nm
        assert abs(x.std() - s) < 5 * s / np.sqrt(2 * n), nm
    # a different seed gives different values; the same seed the same values
    P2 = m.new_params()
    m.init(P2, 1234, cfg["init_std"], cfg["scale_out_proj"])
    P3 = m.new_params()
    m.init(P3, 99, cfg["init_std"], cfg["scale_out_proj"])
    assert torch.equal(P, P2) and not torch.equal(P, P3)


def test_step_graph_replay_matches_individual_launches():
    """On a non-default stream llm_step captures the step into a CUDA graph on
    its second call with the same buffers and replays it afterwards.  Five
    steps (step 4 with another token buffer: launched individually, then the
    graph of the first buffers is captured anew) give bit-identical losses,
    parameters, gradients and moments with graphs on and off, with the same
    launch count; with kernel timing on every step runs as launches, so the
    timed GEMM FLOPs and counts agree."""
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c3", batch=2, ctx=128, n_layer=2)
    lay, p, tok, tgt = _inputs(cfg)

    def run(graphs, timing=False):
        s = torch.cuda.Stream()
        m = LlamaStep(cfg, stream=s)
        m.set_graphs(graphs)
        m.set_kernel_timing(timing)
        P = torch.tensor(p, device="cuda")
        G, M, V = (torch.zeros_like(P) for _ in range(3))
        td = torch.tensor(tok, dtype=torch.int32, device="cuda")
        td2 = td.flip(1).contiguous()
        yd = torch.tensor(tgt, dtype=torch.int32, device="cuda")
        loss = torch.zeros(1, device="cuda")
        torch.cuda.synchronize()
        losses, counts = [], []
        for t in range(1, 6):
            m.step(P, G, M, V, t, td2 if t == 4 else td, yd, cfg["lr"], cfg["wd"], loss)
            s.synchronize()
            losses.append(float(loss.item()))
            counts.append(m.last_launch_count())
        st = m.status()
        timing_read = m.read_kernel_timing() if timing else None
        out = (losses, counts, st, P.cpu(), G.cpu(), M.cpu(), V.cpu(), timing_read)
        m.close()
        return out

    a = run(True)
    b = run(False)
    assert a[2] == 0 and b[2] == 0
    assert a[0] == b[0], (a[0], b[0])
    assert a[1] == b[1], (a[1], b[1])
    for x, y in zip(a[3:7], b[3:7]):
        assert torch.equal(x, y)
    # timing: the same GEMM FLOPs per step whether launched or replayed
    ga = run(True, timing=True)[7]
    gb = run(False, timing=True)[7]
    assert ga[2] == gb[2] and abs(ga[1] - gb[1]) <= 1e-6 * gb[1], (ga, gb)
    assert ga[0] > 0 and gb[0] > 0

