"""Pins of the float64 decode and sampler oracle (oracle/decode.py).

Decode is tied to the full forward of the C oracle (an independent code path):
strata's gate, a decoder with a key/value cache equals the full forward, checked
at every position.  The sampler is tied to closed-form cases, the greedy and
top-k limits and an empirical frequency test over 20k draws (strata, sampler
row).
"""
import math

import numpy as np
import pytest

import oracle as O
from oracle import decode as OD
from synth import get_config, make_batch, make_params

GQA_SMALL = get_config("c1", vocab=11, d_model=16, n_layer=2, n_head=4, n_kv_head=2, d_ff=42,
                       ctx=6, batch=2, init_std=0.3, name="gqa-small", index=9)


@pytest.mark.parametrize("cfgname", ["c1", "gqa", "mqa", "gqa_interp"])
def test_decode_equals_full_forward_at_every_position(cfgname):
    if cfgname == "c1":
        cfg = get_config("c1", batch=2)
    elif cfgname == "gqa":
        cfg = GQA_SMALL
    elif cfgname == "gqa_interp":  # RoPE position interpolation, scale 2
        cfg = dict(GQA_SMALL, rope_scale=2.0, name="gqa-small-interp")
    else:
        cfg = dict(GQA_SMALL, n_kv_head=1, name="mqa-small")
    c = dict(cfg, init_std=0.3)
    p = make_params(c, O.param_layout(cfg), seed=5).astype(np.float64)
    tok, _ = make_batch(cfg, seed=11)
    tok = tok.reshape(cfg["batch"], cfg["ctx"])
    _, z_full, _ = O.forward_backward(cfg, p, tok, want_grads=False)
    z_full = z_full.reshape(cfg["batch"], cfg["ctx"], cfg["vocab"])
    cache = OD.KVCache(cfg)
    for t in range(cfg["ctx"]):
        z = OD.decode_step(cfg, p, cache, tok[:, t], t)
        scale = np.abs(z_full[:, t]).max()
        assert np.abs(z - z_full[:, t]).max() <= 1e-12 * max(1.0, scale), t


def test_decode_cache_holds_rotated_keys_and_plain_values():
    cfg = GQA_SMALL
    p = make_params(dict(cfg), O.param_layout(cfg), seed=2).astype(np.float64)
    tok, _ = make_batch(cfg, seed=3)
    tok = tok.reshape(cfg["batch"], cfg["ctx"])
    cache = OD.KVCache(cfg)
    for t in range(3):
        OD.decode_step(cfg, p, cache, tok[:, t], t)
    # layer 0's key/value of position 2 from the embedding directly
    d, H, Hkv = cfg["d_model"], cfg["n_head"], cfg["n_kv_head"]
    hd = d // H
    P = OD._tensors(cfg, p)
    x = P["wte"][tok[:, 2]]
    xn, _ = O.rmsnorm_fwd(x, P["l0.g1"], cfg["rms_eps"])
    qkv = xn @ P["l0.Wqkv"]
    for b in range(cfg["batch"]):
        for g in range(Hkv):
            k = qkv[b, d + g * hd:d + (g + 1) * hd]
            v = qkv[b, d + Hkv * hd + g * hd:d + Hkv * hd + (g + 1) * hd]
            np.testing.assert_allclose(O.rope(cache.K[0][b, g, 2], 2, sign=-1), k, atol=1e-13)
            np.testing.assert_array_equal(cache.V[0][b, g, 2], v)
    # later positions are untouched
    assert not cache.K[0][:, :, 3:].any() and not cache.V[1][:, :, 3:].any()


# ------------------------------------------------------------------ sampler


def test_sampler_worked_example():
    # weights 1, 2, 3 at temperature 1: cumulative 1, 3, 6 (of 6)
    z = np.log(np.array([1.0, 2.0, 3.0]))
    assert [OD.sample(z, 1.0, 0, u) for u in (0.0, 0.1, 0.17, 0.3, 0.49, 0.51, 0.9, 0.999)] == \
        [0, 0, 1, 1, 1, 2, 2, 2]
    # top-2 keeps ids 1 and 2: cumulative 2, 5 (of 5)
    assert [OD.sample(z, 1.0, 2, u) for u in (0.0, 0.39, 0.41, 0.99)] == [1, 1, 2, 2]
    # temperature 2 takes square roots of the weights: 1, 1.414, 1.732
    w = np.sqrt([1.0, 2.0, 3.0])
    c = np.cumsum(w) / w.sum()
    assert OD.sample(z, 2.0, 0, c[0] - 1e-9) == 0 and OD.sample(z, 2.0, 0, c[0] + 1e-9) == 1
    assert OD.sample(z, 2.0, 0, c[1] - 1e-9) == 1 and OD.sample(z, 2.0, 0, c[1] + 1e-9) == 2


def test_sampler_greedy_limits_and_ties():
    z = np.array([1.0, 5.0, 5.0, 2.0], dtype=np.float32)
    for u in (0.0, 0.5, 0.99):
        assert OD.sample(z, 0.0, 0, u) == 1  # temperature 0: lowest id of the maxima
        assert OD.sample(z, 0.8, 1, u) == 1  # top-1 is greedy too
    # a tiny temperature concentrates on the maxima (split between the tied ids)
    assert OD.sample(z, 1e-4, 0, 0.2) == 1 and OD.sample(z, 1e-4, 0, 0.7) == 2
    # ties at the top-k cut go to the lower ids
    z = np.array([3.0, 1.0, 3.0, 3.0, 0.0], dtype=np.float32)
    np.testing.assert_array_equal(OD.topk_set(z, 2), [0, 2])
    got = {OD.sample(z, 1.0, 2, u) for u in np.linspace(0, 0.999, 50)}
    assert got == {0, 2}
    np.testing.assert_array_equal(OD.topk_set(z, 0), np.arange(5))
    np.testing.assert_array_equal(OD.topk_set(z, 9), np.arange(5))
    # a huge temperature makes the set uniform: u = (i + 1/2) / k picks the i-th id
    S = OD.topk_set(z, 4)
    for i in range(4):
        assert OD.sample(z, 1e9, 4, (i + 0.5) / 4) == S[i]


def test_sampler_empirical_frequencies():
    """20k draws against softmax(z / temperature) over the top-k set."""
    rng = np.random.default_rng(20)
    z = rng.standard_normal(12).astype(np.float32) * 2
    temp, k, n = 0.7, 5, 20000
    draws = np.array([OD.sample(z, temp, k, u) for u in rng.random(n)])
    S = np.argsort(-z.astype(np.float64), kind="stable")[:k]
    p = np.zeros(12)
    p[S] = np.exp(z[S].astype(np.float64) / temp)
    p /= p.sum()
    freq = np.bincount(draws, minlength=12) / n
    assert set(np.unique(draws)) <= set(S.tolist())
    sd = np.sqrt(p * (1 - p) / n)
    assert np.all(np.abs(freq - p) <= 4.5 * sd + 1e-12), (freq, p)
    # and a chi-square statistic consistent with k - 1 degrees of freedom
    chi2 = n * np.sum((freq[S] - p[S]) ** 2 / p[S])
    assert chi2 < 25.0, chi2
    assert math.isclose(freq.sum(), 1.0)


def test_sampler_top_p_worked_example():
    # probabilities 0.5, 0.3, 0.2 (ids 2, 0, 1 by logit): top_p 0.7 keeps the
    # first two by probability (0.5 + 0.3 >= 0.7), renormalised 0.625 / 0.375
    z = np.log(np.array([0.3, 0.2, 0.5]))
    S, _ = OD.nucleus(z, 1.0, 3, 0.7)
    np.testing.assert_array_equal(S, [0, 2])
    # id order: id 0 (0.375) then id 2 (0.625)
    assert [OD.sample(z, 1.0, 3, u, top_p=0.7) for u in (0.0, 0.37, 0.38, 0.99)] == [0, 0, 2, 2]
    # a prefix reaching top_p exactly stops there; top_p 1 keeps the set
    np.testing.assert_array_equal(OD.nucleus(z, 1.0, 3, 0.5)[0], [2])
    np.testing.assert_array_equal(OD.nucleus(z, 1.0, 3, 1.0)[0], [0, 1, 2])
    # a tiny top_p keeps the single most likely id (greedy-like)
    assert {OD.sample(z, 1.0, 3, u, top_p=1e-6) for u in np.linspace(0, 0.99, 20)} == {2}
    # top-p inside top-k: top-2 set {2, 0}; top_p 0.7 of its 0.8 total keeps both
    np.testing.assert_array_equal(OD.nucleus(z, 1.0, 2, 0.7)[0], [0, 2])
    np.testing.assert_array_equal(OD.nucleus(z, 1.0, 2, 0.6)[0], [2])


def test_sampler_repetition_penalty():
    z = np.array([2.0, -1.0, 0.5, 3.0], dtype=np.float32)
    pz = OD.penalise(z, 2.0, [0, 1, 1, 7, -1])
    np.testing.assert_array_equal(pz, np.array([1.0, -2.0, 0.5, 3.0], dtype=np.float32))
    np.testing.assert_array_equal(OD.penalise(z, 1.0, [0, 1]), z)
    # the penalty can move the greedy choice
    z = np.array([2.0, 1.5], dtype=np.float32)
    assert OD.sample(z, 0.0, 0, 0.5) == 0
    assert OD.sample(z, 0.0, 0, 0.5, penalty=1.5, history=[0]) == 1


def test_sampler_top_p_frequencies():
    rng = np.random.default_rng(21)
    z = (rng.standard_normal(12) * 1.5).astype(np.float32)
    temp, k, tp, n = 0.9, 8, 0.8, 20000
    S, _ = OD.nucleus(z, temp, k, tp)
    draws = np.array([OD.sample(z, temp, k, u, top_p=tp) for u in rng.random(n)])
    p = np.zeros(12)
    p[S] = np.exp(z[S].astype(np.float64) / temp)
    p /= p.sum()
    freq = np.bincount(draws, minlength=12) / n
    assert set(np.unique(draws).tolist()) <= set(S.tolist())
    assert np.all(np.abs(freq - p) <= 4.5 * np.sqrt(p * (1 - p) / n) + 1e-12)
    # the nucleus is the shortest prefix reaching top_p of the top-k weight
    w = np.sort(np.exp(z.astype(np.float64) / temp))[::-1][:k]
    m = int(np.argmax(np.cumsum(w) >= tp * w.sum())) + 1
    assert S.size == m
