"""GPU parity of single-token decode (llm_decode) and sampling (llm_sample)
through the C ABI.

Decode is compared with the float64 oracle's full forward at every decoded
position (strata's gate: a decoder with a key/value cache equals the full
forward), and with the library's own llm_forward on the same tokens; the
tolerances are the training step's logits tolerances (1e-4 fp32, 2e-2 bf16,
norm-wise relative error per position).  Sampling is compared with the
oracle sampler applied to the same float32 logits: greedy ids and top-k sets
exactly; a drawn id must lie on the oracle's float64 cumulative-weight interval
that holds u * total, up to the float32 error bound of the kernel's sums (a
chain of at most ceil(V/1024) + 1024 additions, plus the weights' own
rounding); ids may differ only where u * total is that close to a boundary.
"""
import os

import numpy as np
import pytest
import torch

from synth import get_config, make_batch, make_params
from tests.gpu_util import TOL, rel

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _model(cfg):
    from scratch_llama_decoder_b200 import LlamaStep
    import oracle as O
    m = LlamaStep(cfg)
    p = make_params(cfg, O.param_layout(cfg), seed=cfg.get("index", 0) + 40)
    tok, _ = make_batch(cfg, seed=cfg.get("index", 0) + 41)
    return m, p, tok.reshape(cfg["batch"], cfg["ctx"])


DECODE = [
    ("tiny_fp32", "c1", dict(batch=2)),
    ("ragged_fp32", "c2", dict(batch=2, ctx=37, n_layer=2)),
    ("hd32_bf16", "c3", dict(batch=3, ctx=200, n_layer=2)),
    ("gqa_bf16", "c4", dict(batch=2, ctx=300, n_layer=2)),
    ("mqa_bf16", "c4", dict(batch=2, ctx=140, n_layer=1, n_kv_head=1)),
    ("350m_width_bf16", "c5", dict(batch=2, ctx=260, n_layer=2)),
    ("L0_bf16", "c3", dict(batch=2, ctx=64, n_layer=0)),
]


@pytest.mark.parametrize("name,base,over", DECODE, ids=[d[0] for d in DECODE])
def test_decode_matches_full_forward(name, base, over):
    """Prefill half of each sequence with llm_forward (the later positions hold
    other ids), then decode the rest one position at a time."""
    import oracle as O
    cfg = get_config(base, **over)
    B, T, V = cfg["batch"], cfg["ctx"], cfg["vocab"]
    tol = TOL[cfg["compute"]]["logits"]
    m, p, tok = _model(cfg)
    _, zref, _ = O.forward_backward(cfg, p, tok, want_grads=False)
    zref = zref.reshape(B, T, V)
    P = torch.tensor(p, device="cuda")
    full = m.forward(P, torch.tensor(tok, device="cuda")).double().cpu().numpy()
    t0 = T // 2
    junk = tok.copy()
    junk[:, t0:] = (tok[:, t0:] * 7 + 3) % V
    m.forward(P, torch.tensor(junk, device="cuda"))
    worst_o = worst_f = 0.0
    for t in range(t0, T):
        z = m.decode(P, torch.tensor(tok[:, t], device="cuda"), t).double().cpu().numpy()
        for b in range(B):
            worst_o = max(worst_o, rel(z[b], zref[b, t]))
            worst_f = max(worst_f, rel(z[b], full[b, t]))
    assert m.status() == 0
    assert worst_o <= tol, (worst_o, worst_f)
    assert worst_f <= tol, (worst_o, worst_f)
    print(name, "decode vs oracle", worst_o, "vs llm_forward", worst_f)
    m.close()


def test_decode_overwrites_every_cached_position():
    """A forward over unrelated ids (it casts the weights), then decode from
    position 0: every cached key and value read comes from decode itself."""
    import oracle as O
    cfg = get_config("c4", batch=2, ctx=160, n_layer=2)
    B, T, V = cfg["batch"], cfg["ctx"], cfg["vocab"]
    m, p, tok = _model(cfg)
    _, zref, _ = O.forward_backward(cfg, p, tok, want_grads=False)
    zref = zref.reshape(B, T, V)
    P = torch.tensor(p, device="cuda")
    m.forward(P, torch.tensor((tok + 11) % V, device="cuda"))
    worst = 0.0
    for t in range(T):
        z = m.decode(P, torch.tensor(tok[:, t], device="cuda"), t).double().cpu().numpy()
        worst = max(worst, max(rel(z[b], zref[b, t]) for b in range(B)))
    assert worst <= TOL["bf16"]["logits"], worst
    m.close()


def test_decode_graph_replay_is_bit_exact():
    cfg = get_config("c4", batch=2, ctx=200, n_layer=2)
    out = {}
    for graphs in (True, False):
        m, p, tok = _model(cfg)
        m.set_graphs(graphs)
        P = torch.tensor(p, device="cuda")
        m.forward(P, torch.tensor(tok, device="cuda"))
        tk = torch.empty(cfg["batch"], dtype=torch.int32, device="cuda")
        lg = torch.empty(cfg["batch"], cfg["vocab"], device="cuda")
        res = []
        for t in range(100, 140):
            tk.copy_(torch.tensor(tok[:, t], device="cuda"))
            m.decode(P, tk, t, logits=lg)
            res.append(lg.clone())
        if graphs:
            # the replays enqueue the graph plus the position write
            assert m.last_launch_count() > 2
        out[graphs] = torch.stack(res).cpu()
        assert m.status() == 0
        m.close()
    assert torch.equal(out[True], out[False])


def test_decode_argument_and_token_errors():
    import scratch_llama_decoder_b200 as L
    cfg = get_config("c3", batch=2, ctx=64, n_layer=1)
    m, p, tok = _model(cfg)
    P = torch.tensor(p, device="cuda")
    m.forward(P, torch.tensor(tok, device="cuda"))
    tk = torch.tensor(tok[:, 0], device="cuda")
    lg = torch.empty(2, cfg["vocab"], device="cuda")
    lib = L.lib
    for pos in (-1, cfg["ctx"]):
        assert lib.llm_decode(m.ctx, P.data_ptr(), tk.data_ptr(), pos, lg.data_ptr()) == \
            L.LLM_ERR_ARG
    bad = torch.tensor([1, cfg["vocab"]], dtype=torch.int32, device="cuda")
    assert lib.llm_decode(m.ctx, P.data_ptr(), bad.data_ptr(), 3, lg.data_ptr()) == 0
    assert m.status() == L.LLM_ERR_TOKEN
    assert m.status() == 0
    m.close()
    # a head size that does not divide 128
    cfg = get_config("c3", batch=1, ctx=8, n_layer=1, d_model=96, n_head=2, n_kv_head=2,
                     d_ff=256)
    m2 = L.LlamaStep(cfg)
    P2 = torch.zeros(m2.n_params, device="cuda")
    t2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    l2 = torch.empty(1, cfg["vocab"], device="cuda")
    assert lib.llm_decode(m2.ctx, P2.data_ptr(), t2.data_ptr(), 0, l2.data_ptr()) == \
        L.LLM_ERR_CONFIG
    m2.close()


@pytest.mark.parametrize("name", ["c2", "c3", "c4", "c5"])
def test_full_size_decode_matches_oracle_rows(name):
    """Full workload (every layer, the benchmark's batch and context): prefill
    with llm_forward, then decode at the positions of the oracle's stored full
    logit rows (tests/golden/step_<workload>.npz, written by
    tests/golden/make_golden.py from the oracle alone)."""
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config(name)
    path = os.path.join(GOLDEN, f"step_{cfg['name']}.npz")
    if not os.path.exists(path):
        pytest.skip("golden file not generated")
    zg = np.load(path)
    T, V = cfg["ctx"], cfg["vocab"]
    m = LlamaStep(cfg)
    p = make_params(cfg, m.layout)
    tok, _ = make_batch(cfg)
    tok = tok.reshape(cfg["batch"], T)
    P = torch.tensor(p, device="cuda")
    m.forward(P, torch.tensor(tok, device="cuda"))
    worst = 0.0
    for row, want in zip(zg["logit_rows"], zg["logit_rowvals"]):
        b, t = int(row) // T, int(row) % T
        z = m.decode(P, torch.tensor(tok[:, t], device="cuda"), t)
        worst = max(worst, rel(z[b].double().cpu().numpy(), want))
    assert m.status() == 0
    assert worst <= TOL[cfg["compute"]]["logits"], worst
    print(name, "full-size decode vs oracle rows", worst)
    m.close()


# ----------------------------------------------------------------- sampling


def _check_sample(z, temp, k, u, got):
    """Asserts one GPU draw against the oracle sampler; returns True when it
    is the oracle's id."""
    from oracle import decode as OD
    want = OD.sample(z, temp, k, u)
    if temp <= 0 or k == 1:
        assert got == want, (got, want)
        return True
    S, C, W = OD.sample_cdf(z, temp, k)
    assert got in set(S.tolist()), (got, "outside the top-k set")
    i = int(np.searchsorted(S, got))
    lo = C[i - 1] if i > 0 else 0.0
    target = float(u) * W
    tol = (-(-z.size // 1024) + 1024 + 4) * 2.0 ** -23 * W
    assert lo - tol <= target <= C[i] + tol, (got, want, lo, C[i], target)
    return got == want


def _gpu_sample(m, z, temp, k, u):
    zd = torch.tensor(z, dtype=torch.float32, device="cuda")
    ud = torch.tensor(u, dtype=torch.float32, device="cuda")
    return m.sample(zd, temp, k, ud).cpu().numpy()


@pytest.mark.parametrize("V", [27, 500, 32000])
def test_sample_matches_oracle_sampler(V):
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c3", vocab=V, batch=1, ctx=8, n_layer=0)
    m = LlamaStep(cfg)
    rng = np.random.default_rng(V)
    R = 64
    z = (rng.standard_normal((R, V)) * 3).astype(np.float32)
    # planted ties: equal maxima and a block of equal values around the cut
    z[0, 5] = z[0, 9] = z[0].max() + 1
    z[1, :] = np.round(z[1, :])
    z[2, :] = 0.0
    u = rng.random(R).astype(np.float32)
    u[3], u[4] = 0.0, np.float32(0.99999994)
    same = total = 0
    for temp, k in [(0.0, 0), (1.0, 1), (0.8, 40), (1.0, 0), (0.5, 5), (1.3, V + 5), (2.0, 3)]:
        got = _gpu_sample(m, z, temp, k, u)
        again = _gpu_sample(m, z, temp, k, u)
        np.testing.assert_array_equal(got, again)
        for r in range(R):
            same += _check_sample(z[r], temp, k, u[r], int(got[r]))
            total += 1
    assert same >= 0.9 * total, (same, total)
    m.close()


def test_sample_frequencies_over_20k_draws():
    """strata, sampler row: empirical frequencies over 20k draws against
    softmax(z / temperature) renormalised over the top-k set."""
    from scratch_llama_decoder_b200 import LlamaStep
    V, n, temp, k = 12, 20000, 0.7, 5
    cfg = get_config("c1", vocab=V, batch=1, ctx=4)
    m = LlamaStep(cfg)
    rng = np.random.default_rng(12)
    z = (rng.standard_normal(V) * 2).astype(np.float32)
    Z = np.tile(z, (n, 1))
    draws = _gpu_sample(m, Z, temp, k, rng.random(n).astype(np.float32))
    S = np.argsort(-z.astype(np.float64), kind="stable")[:k]
    p = np.zeros(V)
    p[S] = np.exp(z[S].astype(np.float64) / temp)
    p /= p.sum()
    freq = np.bincount(draws, minlength=V) / n
    assert set(np.unique(draws).tolist()) <= set(S.tolist())
    assert np.all(np.abs(freq - p) <= 4.5 * np.sqrt(p * (1 - p) / n) + 1e-12), (freq, p)
    m.close()


def test_sample_arguments():
    import scratch_llama_decoder_b200 as L
    cfg = get_config("c3", batch=1, ctx=8, n_layer=0)
    m = L.LlamaStep(cfg)
    z = torch.zeros(2, cfg["vocab"], device="cuda")
    u = torch.zeros(2, device="cuda")
    o = torch.empty(2, dtype=torch.int32, device="cuda")
    lib = L.lib
    assert lib.llm_sample(m.ctx, z.data_ptr(), cfg["vocab"] - 1, 2, 1.0, 0, u.data_ptr(),
                          o.data_ptr()) == L.LLM_ERR_ARG
    assert lib.llm_sample(m.ctx, z.data_ptr(), cfg["vocab"], 0, 1.0, 0, u.data_ptr(),
                          o.data_ptr()) == L.LLM_ERR_ARG
    assert lib.llm_sample(m.ctx, z.data_ptr(), cfg["vocab"], 2, float("nan"), 0, u.data_ptr(),
                          o.data_ptr()) == L.LLM_ERR_ARG
    # all-equal logits: greedy takes id 0, a draw at u = 0 takes id 0 too
    assert lib.llm_sample(m.ctx, z.data_ptr(), cfg["vocab"], 2, 1.0, 0, u.data_ptr(),
                          o.data_ptr()) == 0
    assert o.cpu().tolist() == [0, 0]
    m.close()
