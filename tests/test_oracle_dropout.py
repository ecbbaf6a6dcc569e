"""Pins of the oracle's inverted dropout (Hephaistos: dropout on the
embeddings, the attention weights and the attention and MLP outputs, masks
drawn by the training forward and reused by its backward) and of its mask
generator, Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC 2011):

- the generator against the published known-answer vectors of Philox4x32-10;
- the mask of element e is output word e mod 4 of one generator call on the
  group counter (e / 4, site + 4 layer, step): four elements per call, also
  past 2^32 groups, and the four words of a group are independent;
- mask statistics (drop fraction p, unit mean of the inverted factors),
  reproducibility and independence across steps, sites and layers;
- p = 0 reduces to the training step without dropout;
- every parameter's gradient with dropout on, by central differences (the
  masks are fixed by seed and step, so the loss is a deterministic function);
- an independent PyTorch float64 autograd model with the same masks.
"""
import numpy as np
import pytest
import torch

import oracle as O
from synth import get_config, make_batch, make_params

GQA_SMALL = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                       ctx=5, batch=2, init_std=0.3, name="gqa-small", index=9)
P_DROP, SEED, STEP = 0.3, 0x1234_5678_9ABC, 7


def _setup(cfg=GQA_SMALL):
    lay = O.param_layout(cfg)
    p = make_params(cfg, lay, seed=5).astype(np.float64)
    tok, tgt = make_batch(cfg, seed=6)
    return lay, p, tok, tgt


def test_philox_known_answers():
    kat = [((0, 0, 0, 0), (0, 0), (0x6627e8d5, 0xe169c58d, 0xbc57ac4c, 0x9b00dbd8)),
           ((0xffffffff,) * 4, (0xffffffff, 0xffffffff),
            (0x408f276d, 0x41c83b0e, 0xa20bc7c6, 0x6d5451fd)),
           ((0x243f6a88, 0x85a308d3, 0x13198a2e, 0x03707344), (0xa4093822, 0x299f31d0),
            (0xd16cfe09, 0x94fdcceb, 0x5001e420, 0x24126ea1))]
    for ctr, key, want in kat:
        assert O.philox4x32_10(ctr, key) == list(want)


def test_mask_statistics_and_independence():
    n = 200_000
    f = O.dropout_factors(P_DROP, SEED, STEP, 2, 1, n)
    kept = f > 0
    assert set(np.unique(f).tolist()) == {0.0, 1.0 / (1.0 - P_DROP)}
    sd = np.sqrt(P_DROP * (1 - P_DROP) / n)
    assert abs((1 - kept.mean()) - P_DROP) < 5 * sd
    assert abs(f.mean() - 1.0) < 5 * sd / (1 - P_DROP)
    # the same (seed, step, site, layer, element) gives the same factor
    np.testing.assert_array_equal(f[1000:2000], O.dropout_factors(P_DROP, SEED, STEP, 2, 1, 1000,
                                                                  e0=1000))
    # other steps, sites, layers and seeds give unrelated masks
    for args in ((P_DROP, SEED, STEP + 1, 2, 1), (P_DROP, SEED, STEP, 3, 1),
                 (P_DROP, SEED, STEP, 2, 0), (P_DROP, SEED + 1, STEP, 2, 1)):
        g = O.dropout_factors(*args, n) > 0
        agree = (g == kept).mean()
        expect = P_DROP ** 2 + (1 - P_DROP) ** 2
        assert abs(agree - expect) < 0.01, (args, agree)
    # p = 0 keeps everything with factor 1
    np.testing.assert_array_equal(O.dropout_factors(0.0, SEED, STEP, 1, 0, 1000), np.ones(1000))


def test_mask_words_are_one_generator_call_per_four_elements():
    thr = int(np.floor(P_DROP * 2.0 ** 32))
    key = (SEED & 0xffffffff, SEED >> 32)
    site, layer = 1, 2
    for e0 in (0, 4 * 1000 + 2, (1 << 34) + 4 * 5 + 1):  # ragged starts; group high word 1
        n = 14
        f = O.dropout_factors(P_DROP, SEED, STEP, site, layer, n, e0=e0)
        for i in range(n):
            e = e0 + i
            g = e // 4
            words = O.philox4x32_10((g & 0xffffffff, g >> 32, site + 4 * layer, STEP), key)
            want = 1.0 / (1.0 - P_DROP) if words[e % 4] >= thr else 0.0
            assert f[i] == want, (e, f[i], want)
    # the four words of a group are independent: within-group pairs agree as
    # often as independent draws
    n = 400_000
    kept = (O.dropout_factors(P_DROP, SEED, STEP, 3, 0, n) > 0).reshape(-1, 4)
    expect = P_DROP ** 2 + (1 - P_DROP) ** 2
    sd = np.sqrt(expect * (1 - expect) / kept.shape[0])
    for j in range(4):
        assert abs((1 - kept[:, j].mean()) - P_DROP) < 5 * np.sqrt(P_DROP * (1 - P_DROP) / kept.shape[0])
        for k in range(j + 1, 4):
            assert abs((kept[:, j] == kept[:, k]).mean() - expect) < 5 * sd, (j, k)


def test_zero_rate_is_the_plain_step():
    lay, p, tok, tgt = _setup()
    l0, z0, g0 = O.forward_backward(GQA_SMALL, p, tok, tgt)
    l1, z1, g1 = O.forward_backward(GQA_SMALL, p, tok, tgt, dropout=(0.0, SEED, STEP))
    assert abs(l0 - l1) <= 1e-14 * abs(l0)
    np.testing.assert_allclose(z1, z0, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g1, g0, rtol=1e-10, atol=1e-14)
    # and dropout on changes the result
    l2, _, _ = O.forward_backward(GQA_SMALL, p, tok, tgt, dropout=(P_DROP, SEED, STEP))
    assert abs(l2 - l0) > 1e-6


def test_gradcheck_with_dropout_all_elements():
    lay, p, tok, tgt = _setup()
    dr = (P_DROP, SEED, STEP)
    _, _, g = O.forward_backward(GQA_SMALL, p, tok, tgt, want_logits=False, dropout=dr)
    eps = 1e-6
    for name, off, rows, cols in lay:
        n = rows * cols
        num = np.zeros(n)
        for i in range(n):
            q = p.copy()
            q[off + i] += eps
            lp, _, _ = O.forward_backward(GQA_SMALL, q, tok, tgt, want_logits=False,
                                          want_grads=False, dropout=dr)
            q[off + i] -= 2 * eps
            lm, _, _ = O.forward_backward(GQA_SMALL, q, tok, tgt, want_logits=False,
                                          want_grads=False, dropout=dr)
            num[i] = (lp - lm) / (2 * eps)
        ana = g[off:off + n]
        rel = np.linalg.norm(ana - num) / max(np.linalg.norm(num), 1e-30)
        assert rel < 1e-6, (name, rel)


def _torch_loss_dropout(cfg, p, tok, tgt, pdrop, seed, step):
    """Independent forward in PyTorch float64 with explicit attention and the
    oracle's dropout factors at the four sites."""
    import torch.nn.functional as F
    V, d, L, H, Hkv, h = (cfg[k] for k in ("vocab", "d_model", "n_layer", "n_head", "n_kv_head",
                                           "d_ff"))
    T, B = cfg["ctx"], cfg["batch"]
    hd = d // H
    P = {n: p[o:o + r * k].view(r, k) if r > 1 else p[o:o + k]
         for n, o, r, k in O.param_layout(cfg)}
    fac = lambda site, layer, shape: torch.tensor(
        O.dropout_factors(pdrop, seed, step, site, layer, int(np.prod(shape)))).view(*shape)
    x = P["wte"][torch.tensor(tok, dtype=torch.long)] * fac(0, 0, (B, T, d))
    pos = torch.arange(T, dtype=torch.float64)
    inv = cfg["rope_base"] ** (-torch.arange(0, hd // 2, dtype=torch.float64) * 2 / hd)
    ang = pos[:, None] * inv[None, :]
    cos, sin = torch.cos(ang), torch.sin(ang)

    def rot(u):
        a, b = u[..., :hd // 2], u[..., hd // 2:]
        return torch.cat([a * cos - b * sin, b * cos + a * sin], -1)

    causal = torch.ones(T, T, dtype=torch.bool).tril()
    for l in range(L):
        xn = F.rms_norm(x, (d,), P[f"l{l}.g1"], eps=cfg["rms_eps"])
        qkv = xn @ P[f"l{l}.Wqkv"]
        q = rot(qkv[..., :d].view(B, T, H, hd).transpose(1, 2))
        k = rot(qkv[..., d:d + Hkv * hd].view(B, T, Hkv, hd).transpose(1, 2))
        v = qkv[..., d + Hkv * hd:].view(B, T, Hkv, hd).transpose(1, 2)
        k = k.repeat_interleave(H // Hkv, dim=1)
        v = v.repeat_interleave(H // Hkv, dim=1)
        s = (q @ k.transpose(-1, -2)) / hd ** 0.5
        s = s.masked_fill(~causal, float("-inf"))
        att = torch.softmax(s, -1) * fac(1, l, (B, H, T, T))
        o = (att @ v).transpose(1, 2).reshape(B, T, d)
        x = x + (o @ P[f"l{l}.Wo"]) * fac(2, l, (B, T, d))
        xn2 = F.rms_norm(x, (d,), P[f"l{l}.g2"], eps=cfg["rms_eps"])
        w13 = P[f"l{l}.W13"]
        u = F.silu(xn2 @ w13[:, :h]) * (xn2 @ w13[:, h:])
        x = x + (u @ P[f"l{l}.W2"]) * fac(3, l, (B, T, d))
    xf = F.rms_norm(x, (d,), P["gf"], eps=cfg["rms_eps"])
    z = xf @ P["Wlm"]
    return F.cross_entropy(z.reshape(-1, V), torch.tensor(tgt, dtype=torch.long).reshape(-1))


@pytest.mark.parametrize("cfgname", ["c1", "gqa"])
def test_dropout_step_against_torch_autograd(cfgname):
    cfg = get_config("c1", batch=2) if cfgname == "c1" else GQA_SMALL
    lay, p, tok, tgt = _setup(cfg)
    loss, _, g = O.forward_backward(cfg, p, tok, tgt, dropout=(P_DROP, SEED, STEP))
    pt = torch.tensor(p, requires_grad=True)
    lt = _torch_loss_dropout(cfg, pt, tok, tgt, P_DROP, SEED, STEP)
    lt.backward()
    assert abs(loss - lt.item()) <= 1e-12 * abs(loss)
    gt = pt.grad.numpy()
    assert np.linalg.norm(g - gt) / np.linalg.norm(gt) <= 1e-10
