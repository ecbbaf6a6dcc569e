"""Pins of the float64 oracle against what the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: values the
pages print, closed forms, invariants, brute force, or an independent library
routine (numpy, PyTorch CPU float64 autograd, torch.optim.AdamW).
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from synth import get_config, make_batch, make_params

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_printed_values.json")

# Shrunk GQA config for gradchecks (V 11, d 16, H 4, H_kv 2, L 2, h 42, T 5, B 2).
GQA_SMALL = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                       ctx=5, batch=2, init_std=0.3, name="gqa-small", index=9)


def _setup(cfg, seed=0, std=None):
    lay = O.param_layout(cfg)
    c = dict(cfg)
    if std is not None:
        c["init_std"] = std
    p = make_params(c, lay, seed=seed).astype(np.float64)
    tok, tgt = make_batch(cfg, seed=seed + 7)
    return lay, p, tok, tgt


# ----------------------------------------------------------------- layout


def test_param_count_matches_page():
    g = json.load(open(GOLDEN))["param_count_hephaistos_small"]
    cfg = get_config("c1", vocab=g["vocab"], d_model=g["d_model"], n_layer=g["n_layer"],
                     n_head=g["n_head"], n_kv_head=g["n_head"], d_ff=(8 * g["d_model"]) // 3,
                     ctx=g["ctx"])
    assert O.n_params(cfg) == g["printed_params"]


def test_param_count_matches_page_scaled_model():
    """Hephaistos' scaled run prints its size to two decimals in millions; the
    layout with SwiGLU hidden floor(8/3 d) = 1024 gives 15,735,168."""
    g = json.load(open(GOLDEN))["param_count_hephaistos_scaled"]
    d = g["d_model"]
    cfg = get_config("c1", vocab=g["vocab"], d_model=d, n_layer=g["n_layer"],
                     n_head=g["n_head"], n_kv_head=g["n_head"], d_ff=(8 * d) // 3, ctx=g["ctx"])
    n = O.n_params(cfg)
    assert round(n / 1e6, g["digits_after_point"]) == g["printed_params_millions"], n


@pytest.mark.parametrize("name,expect", [("c1", 3952), ("c2", 1702016), ("c3", 5742848),
                                         ("c4", 30413312), ("c5", 317195264)])
def test_param_count_closed_form(name, expect):
    c = get_config(name)
    V, d, L, h = c["vocab"], c["d_model"], c["n_layer"], c["d_ff"]
    kvd = d // c["n_head"] * c["n_kv_head"]
    closed = V * d + L * (2 * d + d * (d + 2 * kvd) + d * d + 3 * d * h) + d + d * V
    assert O.n_params(c) == closed == expect
    lay = O.param_layout(c)
    # contiguous, non-overlapping, covering
    pos = 0
    for _, off, r, k in lay:
        assert off == pos
        pos += r * k
    assert pos == closed


# ------------------------------------------------------------------ matmul


def test_matmul_vs_numpy_ragged():
    rng = np.random.default_rng(1)
    A = rng.standard_normal((37, 19))
    B = rng.standard_normal((19, 23))
    np.testing.assert_allclose(O.mm_nn(A, B), A @ B, rtol=1e-13, atol=1e-13)
    A2 = rng.standard_normal((29, 13))
    B2 = rng.standard_normal((29, 7))
    np.testing.assert_allclose(O.mm_tn(A2, B2), A2.T @ B2, rtol=1e-13, atol=1e-13)
    A3 = rng.standard_normal((11, 17))
    B3 = rng.standard_normal((9, 17))
    np.testing.assert_allclose(O.mm_nt(A3, B3), A3 @ B3.T, rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------- RMSNorm


def test_rmsnorm_vs_torch_and_unit_rms():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((9, 24)) * 3.0
    g = rng.standard_normal(24)
    y, r = O.rmsnorm_fwd(x, g, 1e-5)
    yt = F.rms_norm(torch.tensor(x), (24,), torch.tensor(g), eps=1e-5).numpy()
    np.testing.assert_allclose(y, yt, rtol=1e-12, atol=1e-12)
    # with unit gains the output has RMS 1 up to eps
    y1, _ = O.rmsnorm_fwd(x, np.ones(24), 0.0)
    np.testing.assert_allclose(np.sqrt((y1 ** 2).mean(1)), 1.0, rtol=1e-12)
    # scale invariance at eps = 0
    y2, _ = O.rmsnorm_fwd(5.0 * x, g, 0.0)
    y3, _ = O.rmsnorm_fwd(x, g, 0.0)
    np.testing.assert_allclose(y2, y3, rtol=1e-12, atol=1e-12)


def test_rmsnorm_bwd_vs_autograd_and_null_direction():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((6, 20))
    g = rng.standard_normal(20)
    dy = rng.standard_normal((6, 20))
    _, r = O.rmsnorm_fwd(x, g, 1e-5)
    dx, dg = O.rmsnorm_bwd(x, r, g, dy)
    xt = torch.tensor(x, requires_grad=True)
    gt = torch.tensor(g, requires_grad=True)
    F.rms_norm(xt, (20,), gt, eps=1e-5).backward(torch.tensor(dy))
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dg, gt.grad.numpy(), rtol=1e-11, atol=1e-12)
    # at eps = 0 the Jacobian annihilates x: x . dx = 0 per row
    _, r0 = O.rmsnorm_fwd(x, g, 0.0)
    dx0, _ = O.rmsnorm_bwd(x, r0, g, dy)
    assert np.abs((x * dx0).sum(1)).max() < 1e-12


# -------------------------------------------------------------------- RoPE


def test_rope_norm_identity_inverse_and_relative():
    rng = np.random.default_rng(4)
    hd = 16
    q = rng.standard_normal(hd)
    k = rng.standard_normal(hd)
    np.testing.assert_array_equal(O.rope(q, 0), q)  # t = 0 is the identity
    for t in (1, 7, 255, 2047):
        qr = O.rope(q, t)
        assert abs(np.linalg.norm(qr) - np.linalg.norm(q)) < 1e-12
        np.testing.assert_allclose(O.rope(qr, t, sign=-1), q, atol=1e-12)
    # <R_i q, R_j k> depends only on i - j (strata, RoPE relative position)
    for i, j, s in ((5, 2, 11), (9, 9, 100), (3, 0, 40)):
        a = O.rope(q, i) @ O.rope(k, j)
        b = O.rope(q, i + s) @ O.rope(k, j + s)
        assert abs(a - b) < 1e-11
    # rotate-half pairing: component j mixes only with j + hd/2 (first pair at
    # theta_0 = 1 rotates by exactly t radians)
    e = np.zeros(hd)
    e[0] = 1.0
    r = O.rope(e, 3)
    expect = np.zeros(hd)
    expect[0], expect[hd // 2] = math.cos(3.0), math.sin(3.0)
    np.testing.assert_allclose(r, expect, atol=1e-15)
    # last pair: theta = base^(-2(hd/2-1)/hd)
    e = np.zeros(hd)
    e[hd // 2 - 1] = 1.0
    th = 10000.0 ** (-2.0 * (hd // 2 - 1) / hd)
    r = O.rope(e, 5)
    assert abs(r[hd // 2 - 1] - math.cos(5 * th)) < 1e-15
    assert abs(r[hd - 1] - math.sin(5 * th)) < 1e-15


# --------------------------------------------------------------- attention


def _qkv(rng, T, d, H, Hkv):
    hd = d // H
    return rng.standard_normal((T, d + 2 * Hkv * hd))


@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (4, 1)])
def test_attention_vs_torch_sdpa(H, Hkv):
    rng = np.random.default_rng(5)
    T, d = 13, 32
    hd = d // H
    qkv = _qkv(rng, T, d, H, Hkv)
    o, lse, P = O.attention_fwd(qkv, d, H, Hkv, want_probs=True)
    q = torch.tensor(qkv[:, :d]).view(T, H, hd).transpose(0, 1)[None]
    k = torch.tensor(qkv[:, d:d + Hkv * hd]).view(T, Hkv, hd).transpose(0, 1)[None]
    v = torch.tensor(qkv[:, d + Hkv * hd:]).view(T, Hkv, hd).transpose(0, 1)[None]
    ot = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
    ot = ot[0].transpose(0, 1).reshape(T, d).numpy()
    np.testing.assert_allclose(o, ot, rtol=1e-12, atol=1e-12)
    # probability rows sum to one, causal zeros above the diagonal
    np.testing.assert_allclose(P.sum(-1), 1.0, rtol=1e-14)
    assert np.all(P[:, np.triu_indices(T, 1)[0], np.triu_indices(T, 1)[1]] == 0.0)
    # lse matches a direct log-sum-exp of the scaled causal scores
    s = np.einsum("hid,hjd->hij", q[0].numpy(), np.repeat(k[0].numpy(), H // Hkv, 0)) / math.sqrt(hd)
    s = np.where(np.tril(np.ones((T, T))) > 0, s, -np.inf)
    np.testing.assert_allclose(lse, np.log(np.exp(s).sum(-1)), rtol=1e-12)


@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2)])
def test_attention_bwd_vs_autograd(H, Hkv):
    rng = np.random.default_rng(6)
    T, d = 11, 32
    hd = d // H
    qkv = _qkv(rng, T, d, H, Hkv)
    do = rng.standard_normal((T, d))
    dqkv = O.attention_bwd(qkv, do, d, H, Hkv)
    X = torch.tensor(qkv, requires_grad=True)
    q = X[:, :d].view(T, H, hd).transpose(0, 1)[None]
    k = X[:, d:d + Hkv * hd].view(T, Hkv, hd).transpose(0, 1)[None]
    v = X[:, d + Hkv * hd:].view(T, Hkv, hd).transpose(0, 1)[None]
    ot = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
    ot[0].transpose(0, 1).reshape(T, d).backward(torch.tensor(do))
    np.testing.assert_allclose(dqkv, X.grad.numpy(), rtol=1e-11, atol=1e-12)


def test_attention_T1_is_v():
    rng = np.random.default_rng(7)
    qkv = _qkv(rng, 1, 16, 4, 2)
    o, _, _ = O.attention_fwd(qkv, 16, 4, 2)
    v = qkv[0, 16 + 8:]
    np.testing.assert_array_equal(o[0], np.repeat(v.reshape(2, 4), 2, 0).reshape(-1))


# ------------------------------------------------------------------ SwiGLU


def test_swiglu_vs_autograd_and_zero_gate():
    rng = np.random.default_rng(8)
    a = rng.standard_normal(50) * 3
    b = rng.standard_normal(50)
    du = rng.standard_normal(50)
    u = O.swiglu_fwd(a, b)
    at = torch.tensor(a, requires_grad=True)
    bt = torch.tensor(b, requires_grad=True)
    ut = F.silu(at) * bt
    np.testing.assert_allclose(u, ut.detach().numpy(), rtol=1e-13, atol=1e-15)
    ut.backward(torch.tensor(du))
    da, db = O.swiglu_bwd(a, b, du)
    np.testing.assert_allclose(da, at.grad.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=1e-12, atol=1e-14)
    assert np.all(O.swiglu_fwd(np.zeros(5), b[:5]) == 0.0)


# ------------------------------------------------------------ embedding bwd


def test_embed_bwd_vs_add_at():
    rng = np.random.default_rng(12)
    tok = rng.integers(0, 9, 40).astype(np.int32)
    dx = rng.standard_normal((40, 5))
    ref = np.zeros((11, 5))
    np.add.at(ref, tok, dx)
    got = O.embed_bwd(tok, dx, 11)
    np.testing.assert_allclose(got, ref, rtol=1e-14, atol=1e-15)
    assert np.all(got[9:] == 0.0) and np.all(got[~np.isin(np.arange(11), tok)] == 0.0)


# ------------------------------------------------------------ cross-entropy


def test_ce_vs_torch_and_row_sums():
    rng = np.random.default_rng(9)
    z = rng.standard_normal((17, 29)) * 4
    y = rng.integers(0, 29, 17).astype(np.int32)
    s, dz = O.ce_fwd_bwd(z, y)
    zt = torch.tensor(z, requires_grad=True)
    lt = F.cross_entropy(zt, torch.tensor(y, dtype=torch.long), reduction="mean")
    lt.backward()
    assert abs(s / 17 - lt.item()) < 1e-13
    np.testing.assert_allclose(dz, zt.grad.numpy(), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dz.sum(1), 0.0, atol=1e-15)


# ------------------------------------------------------------- whole model


def test_zero_lm_head_gives_ln_vocab_exactly():
    for name in ("c1", "c2"):
        cfg = get_config(name, batch=2, ctx=8)
        lay, p, tok, tgt = _setup(cfg)
        off, r, k = [(o, r, k) for n, o, r, k in lay if n == "Wlm"][0]
        p[off:off + r * k] = 0.0
        loss, logits, grads = O.forward_backward(cfg, p, tok, tgt)
        assert abs(loss - math.log(cfg["vocab"])) < 1e-13
    # the page's printed ln(1024)
    g = json.load(open(GOLDEN))["untrained_loss_uniform_guess"][0]
    cfg = get_config("c1", vocab=g["vocab"], batch=1, ctx=4)
    lay, p, tok, tgt = _setup(cfg)
    off, r, k = [(o, r, k) for n, o, r, k in lay if n == "Wlm"][0]
    p[off:off + r * k] = 0.0
    loss, _, _ = O.forward_backward(cfg, p, tok, tgt, want_grads=False)
    assert round(loss, g["digits"]) == g["ln_vocab_printed"]


def test_untrained_loss_near_ln_vocab():
    # Hephaistos prints 6.9847 against ln(1024) = 6.9315 for an untrained model
    for name in ("c1", "c2"):
        cfg = get_config(name, batch=2, ctx=32)
        lay, p, tok, tgt = _setup(cfg)
        loss, _, _ = O.forward_backward(cfg, p, tok, tgt, want_grads=False)
        assert abs(loss - math.log(cfg["vocab"])) / math.log(cfg["vocab"]) < 0.05


def test_causality_bit_exact():
    cfg = get_config("c1", n_layer=2, ctx=12, batch=1)
    lay, p, tok, tgt = _setup(cfg, std=0.3)
    _, z0, _ = O.forward_backward(cfg, p, tok, tgt, want_grads=False)
    for t in (0, 5, 11):
        tok2 = tok.copy()
        tok2[0, t] = (tok2[0, t] + 5) % cfg["vocab"]
        _, z1, _ = O.forward_backward(cfg, p, tok2, tgt, want_grads=False)
        np.testing.assert_array_equal(z0[:t], z1[:t])
        if t < 11:
            assert np.abs(z0[t:] - z1[t:]).max() > 0


def test_prefix_recompute_parity():
    cfg = get_config("c1", n_layer=2, ctx=12, batch=1, n_kv_head=2)
    lay, p, tok, tgt = _setup(cfg, std=0.3)
    _, z, _ = O.forward_backward(cfg, p, tok, tgt, want_grads=False)
    for t in (1, 4, 9):
        c2 = dict(cfg, ctx=t)
        _, zp, _ = O.forward_backward(c2, p, tok[:, :t], tgt[:, :t], want_grads=False)
        assert np.abs(zp - z[:t]).max() <= 1e-12


def test_zero_layers_reduces_to_norm_and_head():
    cfg = get_config("c2", n_layer=0, batch=2, ctx=6)
    lay, p, tok, tgt = _setup(cfg)
    V, d = cfg["vocab"], cfg["d_model"]
    _, z, _ = O.forward_backward(cfg, p, tok, tgt, want_grads=False)
    wte = p[:V * d].reshape(V, d)
    gf = p[V * d:V * d + d]
    wlm = p[V * d + d:].reshape(d, V)
    x = wte[tok.reshape(-1)]
    xf = gf * x / np.sqrt((x * x).mean(1, keepdims=True) + 1e-5)
    np.testing.assert_allclose(z, xf @ wlm, rtol=1e-12, atol=1e-13)


def _expand_gqa_to_mha(cfg, p):
    """Params of an MHA model equal to the GQA model with K/V columns repeated."""
    H, Hkv, d = cfg["n_head"], cfg["n_kv_head"], cfg["d_model"]
    hd, grp = d // H, H // Hkv
    cm = dict(cfg, n_kv_head=H)
    lay_g = {n: (o, r, k) for n, o, r, k in O.param_layout(cfg)}
    lay_m = O.param_layout(cm)
    out = np.zeros(O.n_params(cm))
    for n, o, r, k in lay_m:
        og, rg, kg = lay_g[n]
        src = p[og:og + rg * kg].reshape(rg, kg)
        if n.endswith("Wqkv"):
            q = src[:, :d]
            kk = src[:, d:d + Hkv * hd].reshape(d, Hkv, hd)
            vv = src[:, d + Hkv * hd:].reshape(d, Hkv, hd)
            kk = np.repeat(kk, grp, axis=1).reshape(d, H * hd)
            vv = np.repeat(vv, grp, axis=1).reshape(d, H * hd)
            src = np.concatenate([q, kk, vv], 1)
        out[o:o + r * k] = src.reshape(-1)
    return cm, out


def test_gqa_equals_repeated_kv_mha():
    cfg = GQA_SMALL
    lay, p, tok, tgt = _setup(cfg, std=0.3)
    lg, zg, gg = O.forward_backward(cfg, p, tok, tgt)
    cm, pm = _expand_gqa_to_mha(cfg, p)
    lm, zm, gm = O.forward_backward(cm, pm, tok, tgt)
    assert abs(lg - lm) < 1e-13
    np.testing.assert_allclose(zg, zm, rtol=1e-12, atol=1e-13)
    # the GQA k/v gradient is the group-sum of the MHA one
    H, Hkv, d = cfg["n_head"], cfg["n_kv_head"], cfg["d_model"]
    hd, grp = d // H, H // Hkv
    lay_m = {n: (o, r, k) for n, o, r, k in O.param_layout(cm)}
    for n, o, r, k in lay:
        if not n.endswith("Wqkv"):
            continue
        G = gg[o:o + r * k].reshape(r, k)
        om, rm, km = lay_m[n]
        M = gm[om:om + rm * km].reshape(rm, km)
        np.testing.assert_allclose(G[:, :d], M[:, :d], rtol=1e-11, atol=1e-14)
        ksum = M[:, d:2 * d].reshape(d, Hkv, grp, hd).sum(2).reshape(d, Hkv * hd)
        vsum = M[:, 2 * d:].reshape(d, Hkv, grp, hd).sum(2).reshape(d, Hkv * hd)
        np.testing.assert_allclose(G[:, d:d + Hkv * hd], ksum, rtol=1e-10, atol=1e-14)
        np.testing.assert_allclose(G[:, d + Hkv * hd:], vsum, rtol=1e-10, atol=1e-14)


def test_padded_hidden_invariance():
    """Zero pad columns of W1/W3 and zero pad rows of W2 leave the loss unchanged;
    their gradients and AdamW updates stay exactly zero."""
    cfg = get_config("c1", n_layer=2, ctx=8, batch=2)
    lay, p, tok, tgt = _setup(cfg, std=0.3)
    h, hp, d = cfg["d_ff"], 64, cfg["d_model"]
    cp = dict(cfg, d_ff=hp)
    layp = {n: (o, r, k) for n, o, r, k in O.param_layout(cp)}
    pp = np.zeros(O.n_params(cp))
    for n, o, r, k in lay:
        src = p[o:o + r * k].reshape(r, k)
        op, rp, kp = layp[n]
        dst = np.zeros((rp, kp))
        if n.endswith("W13"):
            dst[:, :h] = src[:, :h]
            dst[:, hp:hp + h] = src[:, h:]
        elif n.endswith("W2"):
            dst[:h] = src
        else:
            dst = src
        pp[op:op + rp * kp] = dst.reshape(-1)
    l0, z0, g0 = O.forward_backward(cfg, p, tok, tgt)
    l1, z1, g1 = O.forward_backward(cp, pp, tok, tgt)
    assert abs(l0 - l1) < 1e-13
    np.testing.assert_allclose(z0, z1, rtol=1e-12, atol=1e-13)
    m = np.zeros_like(pp)
    p2, m2, v2 = O.adamw(pp, g1, m, m, 1, 1e-2, 0.1)
    for n, (o, r, k) in layp.items():
        G = g1[o:o + r * k].reshape(r, k)
        Pn = p2[o:o + r * k].reshape(r, k)
        if n.endswith("W13"):
            for blk in (G, Pn):
                assert np.all(blk[:, h:hp] == 0.0) and np.all(blk[:, hp + h:] == 0.0)
        if n.endswith("W2"):
            for blk in (G, Pn):
                assert np.all(blk[h:] == 0.0)


# --------------------------------------------------------------- gradcheck


def _gradcheck(cfg, p, tok, tgt, per_tensor=None, eps=1e-6, seed=0):
    loss, _, g = O.forward_backward(cfg, p, tok, tgt, want_logits=False)
    rng = np.random.default_rng(seed)
    worst = 0.0
    for name, off, r, k in O.param_layout(cfg):
        n = r * k
        idx = np.arange(n) if per_tensor is None or n <= per_tensor else \
            rng.choice(n, per_tensor, replace=False)
        num = np.zeros(len(idx))
        for e, i in enumerate(idx):
            pp = p.copy()
            pp[off + i] += eps
            lp, _, _ = O.forward_backward(cfg, pp, tok, tgt, want_logits=False, want_grads=False)
            pp[off + i] -= 2 * eps
            lm, _, _ = O.forward_backward(cfg, pp, tok, tgt, want_logits=False, want_grads=False)
            num[e] = (lp - lm) / (2 * eps)
        ana = g[off + idx]
        rel = np.linalg.norm(ana - num) / max(np.linalg.norm(num), 1e-300)
        worst = max(worst, rel)
        assert rel < 1e-6, (name, rel)
    return worst


def test_gradcheck_tiny_all_elements():
    cfg = get_config("c1")
    lay, p, tok, tgt = _setup(cfg)
    assert _gradcheck(cfg, p, tok, tgt) < 1e-6


def test_gradcheck_gqa_small():
    cfg = GQA_SMALL
    lay, p, tok, tgt = _setup(cfg, std=0.3)
    assert _gradcheck(cfg, p, tok, tgt, per_tensor=64) < 1e-6


# ------------------------------------------------- PyTorch float64 autograd


def torch_model_loss(cfg, p, tok, tgt, pairing="half", rope_scale=1.0):
    """Independent forward in PyTorch float64 (library ops: rms_norm, SDPA with
    GQA, silu, cross_entropy).  RoPE pairs dimension j with j + hd/2
    (rotate-half, the default) or 2j with 2j + 1 (pairing="interleaved"); pair
    j turns by t * base^(-2j/hd) either way."""
    V, d, L, H, Hkv, h = (cfg[k] for k in ("vocab", "d_model", "n_layer", "n_head", "n_kv_head",
                                           "d_ff"))
    T, B = cfg["ctx"], cfg["batch"]
    hd = d // H
    lay = O.param_layout(cfg)
    P = {n: p[o:o + r * k].view(r, k) if r > 1 else p[o:o + k] for n, o, r, k in lay}
    tok_t = torch.tensor(tok, dtype=torch.long)
    x = P["wte"][tok_t]  # [B,T,d]
    pos = torch.arange(T, dtype=torch.float64) / rope_scale
    inv = cfg["rope_base"] ** (-torch.arange(0, hd // 2, dtype=torch.float64) * 2 / hd)
    ang = pos[:, None] * inv[None, :]
    cos, sin = torch.cos(ang), torch.sin(ang)

    def rot(u):  # u [B, n, T, hd]
        if pairing == "interleaved":
            a, b = u[..., 0::2], u[..., 1::2]
            return torch.stack([a * cos - b * sin, b * cos + a * sin], -1).flatten(-2)
        a, b = u[..., :hd // 2], u[..., hd // 2:]
        return torch.cat([a * cos - b * sin, b * cos + a * sin], -1)

    for l in range(L):
        xn = F.rms_norm(x, (d,), P[f"l{l}.g1"], eps=cfg["rms_eps"])
        qkv = xn @ P[f"l{l}.Wqkv"]
        q = qkv[..., :d].view(B, T, H, hd).transpose(1, 2)
        k = qkv[..., d:d + Hkv * hd].view(B, T, Hkv, hd).transpose(1, 2)
        v = qkv[..., d + Hkv * hd:].view(B, T, Hkv, hd).transpose(1, 2)
        o = F.scaled_dot_product_attention(rot(q), rot(k), v, is_causal=True, enable_gqa=True)
        x = x + o.transpose(1, 2).reshape(B, T, d) @ P[f"l{l}.Wo"]
        xn2 = F.rms_norm(x, (d,), P[f"l{l}.g2"], eps=cfg["rms_eps"])
        w13 = P[f"l{l}.W13"]
        u = F.silu(xn2 @ w13[:, :h]) * (xn2 @ w13[:, h:])
        x = x + u @ P[f"l{l}.W2"]
    xf = F.rms_norm(x, (d,), P["gf"], eps=cfg["rms_eps"])
    z = xf @ P["Wlm"]
    loss = F.cross_entropy(z.reshape(-1, V), torch.tensor(tgt, dtype=torch.long).reshape(-1))
    return loss, z.reshape(-1, V)


@pytest.mark.parametrize("cfgname", ["c1", "gqa"])
def test_full_step_vs_torch_autograd_and_adamw(cfgname):
    cfg = get_config("c1") if cfgname == "c1" else GQA_SMALL
    lay, p, tok, tgt = _setup(cfg, std=0.2)
    loss, z, g = O.forward_backward(cfg, p, tok, tgt)
    pt = torch.tensor(p, requires_grad=True)
    lt, zt = torch_model_loss(cfg, pt, tok, tgt)
    lt.backward()
    assert abs(loss - lt.item()) <= 1e-12
    np.testing.assert_allclose(z, zt.detach().numpy(), rtol=1e-10, atol=1e-12)
    gt = pt.grad.numpy()
    assert np.linalg.norm(g - gt) / np.linalg.norm(gt) <= 1e-10
    # AdamW, three steps, against torch.optim.AdamW on the same gradients
    lr, wd = cfg["lr"], cfg["wd"]
    P_o, M_o, V_o = p.copy(), np.zeros_like(p), np.zeros_like(p)
    P_t = torch.tensor(p.copy(), requires_grad=True)
    opt = torch.optim.AdamW([P_t], lr=lr, betas=(0.9, 0.999), eps=1e-8, weight_decay=wd)
    rng = np.random.default_rng(3)
    for t in range(1, 4):
        grad = g * (1.0 + 0.1 * rng.standard_normal(g.size))
        P_o, M_o, V_o = O.adamw(P_o, grad, M_o, V_o, t, lr, wd)
        P_t.grad = torch.tensor(grad)
        opt.step()
        np.testing.assert_allclose(P_o, P_t.detach().numpy(), rtol=1e-12, atol=1e-15)
    st = opt.state[P_t]
    np.testing.assert_allclose(M_o, st["exp_avg"].numpy(), rtol=1e-12, atol=1e-18)
    np.testing.assert_allclose(V_o, st["exp_avg_sq"].numpy(), rtol=1e-12, atol=1e-20)


def test_rope_pairings_differ_by_a_column_permutation():
    """The pages pair RoPE dimensions two ways (rotate-half on the Llama page,
    even-odd pairs on the CodeGen page).  The oracle takes rotate-half; the
    reading rests on the two being the same model up to one fixed permutation
    of each head's q and k columns of Wqkv: rotate-half slot j takes
    interleaved dimension 2j, slot j + hd/2 takes 2j + 1."""
    cfg = GQA_SMALL
    lay, p, tok, tgt = _setup(cfg, std=0.3)
    d, H, Hkv, L = cfg["d_model"], cfg["n_head"], cfg["n_kv_head"], cfg["n_layer"]
    hd = d // H
    perm = np.concatenate([np.arange(0, hd, 2), np.arange(1, hd, 2)])
    cols = np.arange(d + 2 * Hkv * hd)
    for h in range(H + Hkv):  # q heads, then k heads; v columns keep their place
        cols[h * hd:(h + 1) * hd] = h * hd + perm
    pp = p.copy()
    spans = {n: (o, r, k) for n, o, r, k in lay}
    for l in range(L):
        o, r, k = spans[f"l{l}.Wqkv"]
        pp[o:o + r * k] = p[o:o + r * k].reshape(r, k)[:, cols].reshape(-1)
    loss_h, z_h, g_h = O.forward_backward(cfg, pp, tok, tgt)
    pt = torch.tensor(p, requires_grad=True)
    lt, zt = torch_model_loss(cfg, pt, tok, tgt, pairing="interleaved")
    lt.backward()
    assert abs(loss_h - lt.item()) <= 1e-12
    np.testing.assert_allclose(z_h, zt.detach().numpy(), rtol=1e-10, atol=1e-12)
    # gradients: the oracle's, with the columns moved back, are the interleaved model's
    g_back = g_h.copy()
    for l in range(L):
        o, r, k = spans[f"l{l}.Wqkv"]
        blk = np.empty((r, k))
        blk[:, cols] = g_h[o:o + r * k].reshape(r, k)
        g_back[o:o + r * k] = blk.reshape(-1)
    gt = pt.grad.numpy()
    assert np.linalg.norm(g_back - gt) / np.linalg.norm(gt) <= 1e-10
    # without the permutation the two pairings are different models
    loss_plain, _, _ = O.forward_backward(cfg, p, tok, tgt)
    assert abs(loss_plain - lt.item()) > 1e-6


def test_rope_position_interpolation():
    """strata, RoPE row: position interpolation folds extended positions into
    the trained range (position t / scale)."""
    rng = np.random.default_rng(12)
    hd = 16
    u, k = rng.standard_normal(hd), rng.standard_normal(hd)
    for t in (0, 1, 5, 1023):
        np.testing.assert_array_equal(O.rope(u, 2 * t, scale=2.0), O.rope(u, t))
    half = O.rope(u, 1, scale=2.0)  # two half steps make one step
    np.testing.assert_allclose(O.rope(half, 1, scale=2.0), O.rope(u, 1), atol=1e-14)
    # relative positions survive the scaling
    a = O.rope(u, 7, scale=4.0) @ O.rope(k, 3, scale=4.0)
    b = O.rope(u, 107, scale=4.0) @ O.rope(k, 103, scale=4.0)
    assert abs(a - b) < 1e-11
    # the model with a scale against PyTorch float64 autograd with scaled positions
    cfg = dict(GQA_SMALL, ctx=7, rope_scale=2.5)
    lay, p, tok, tgt = _setup(cfg, std=0.2)
    loss, z, g = O.forward_backward(cfg, p, tok, tgt)
    pt = torch.tensor(p, requires_grad=True)
    lt, zt = torch_model_loss(cfg, pt, tok, tgt, rope_scale=2.5)
    lt.backward()
    assert abs(loss - lt.item()) <= 1e-12
    np.testing.assert_allclose(z, zt.detach().numpy(), rtol=1e-10, atol=1e-12)
    assert np.linalg.norm(g - pt.grad.numpy()) / np.linalg.norm(pt.grad.numpy()) <= 1e-10
    # and scale 1 is the plain model
    l1, _, _ = O.forward_backward(dict(cfg, rope_scale=1.0), p, tok, tgt, want_grads=False)
    plain = {k_: v for k_, v in cfg.items() if k_ != "rope_scale"}
    l0, _, _ = O.forward_backward(plain, p, tok, tgt, want_grads=False)
    assert l1 == l0 and abs(l1 - loss) > 1e-9


# ------------------------------------------------------------------- AdamW


def test_adamw_closed_form_first_step():
    rng = np.random.default_rng(11)
    p = rng.standard_normal(100)
    g = rng.standard_normal(100) * 1e-3
    lr, wd, eps = 1e-2, 0.1, 1e-8
    p2, m2, v2 = O.adamw(p, g, np.zeros(100), np.zeros(100), 1, lr, wd, eps=eps)
    np.testing.assert_allclose(p2 - p, -lr * wd * p - lr * g / (np.abs(g) + eps), rtol=1e-9,
                               atol=1e-15)
    np.testing.assert_allclose(m2, 0.1 * g, rtol=1e-14)
    np.testing.assert_allclose(v2, 0.001 * g * g, rtol=1e-12)


def test_adamw_converges_on_quadratic():
    # strata, train/optim: AdamW converges on a quadratic
    target = np.array([1.5, -2.0, 0.25, 3.0])
    p, m, v = np.zeros(4), np.zeros(4), np.zeros(4)
    for t in range(1, 3001):
        g = 2.0 * (p - target)
        p, m, v = O.adamw(p, g, m, v, t, 1e-2, 0.0)
    assert np.abs(p - target).max() < 1e-3
