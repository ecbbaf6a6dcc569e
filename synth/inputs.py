"""Seeded synthetic tokens and initial weights.

Token structure: iid draws per row.  The tiny config draws uniformly over the
vocabulary; the others draw from a Zipf law P(k) ~ (k+1)^-1.1 over [0, V),
a stand-in for the frequency structure of the pages' text corpora (none is
available here).  Each row draws T+1 tokens: tokens = row[:T], targets =
row[1:].  Weights are float64 normal draws cast to float32; RMSNorm gains are
one.  No arithmetic of the model lives here.
"""
import numpy as np


def zipf_tokens(rng, n, vocab, s=1.1):
    """n iid ids with P(k) proportional to (k+1)^-s, by inverse CDF."""
    w = (np.arange(vocab, dtype=np.float64) + 1.0) ** (-s)
    cdf = np.cumsum(w)
    cdf /= cdf[-1]
    u = rng.random(n)
    return np.minimum(np.searchsorted(cdf, u, side="right"), vocab - 1).astype(np.int32)


def make_batch(cfg, seed=None, batch=None, ctx=None):
    """(tokens [B,T], targets [B,T]) int32 for a config; seed defaults to
    1000 + the config's index."""
    B = cfg["batch"] if batch is None else batch
    T = cfg["ctx"] if ctx is None else ctx
    rng = np.random.default_rng(1000 + cfg["index"] if seed is None else seed)
    if cfg["token_dist"] == "uniform":
        rows = rng.integers(0, cfg["vocab"], size=(B, T + 1), dtype=np.int64).astype(np.int32)
    else:
        rows = zipf_tokens(rng, B * (T + 1), cfg["vocab"]).reshape(B, T + 1)
    return np.ascontiguousarray(rows[:, :T]), np.ascontiguousarray(rows[:, 1:])


def make_params(cfg, layout, seed=None):
    """Flat float32 parameters for `layout` = [(name, offset, rows, cols)].

    Matrices ~ N(0, init_std); gains (names g1, g2, gf) = 1.  When the config
    scales output projections, Wo and W2 use init_std / sqrt(2 * n_layer)
    (randyGPT, Features: GPT-2 style scaled init of output projections)."""
    rng = np.random.default_rng(1001 + cfg["index"] if seed is None else seed)
    total = max(o + r * k for _, o, r, k in layout)
    p = np.zeros(total, dtype=np.float32)
    std = cfg["init_std"]
    for name, off, rows, cols in layout:
        base = name.split(".")[-1]
        n = rows * cols
        if base in ("g1", "g2", "gf"):
            p[off:off + n] = 1.0
            continue
        s = std
        if cfg["scale_out_proj"] and base in ("Wo", "W2"):
            s = std / np.sqrt(2.0 * cfg["n_layer"])
        p[off:off + n] = (rng.standard_normal(n) * s).astype(np.float32)
    return p
