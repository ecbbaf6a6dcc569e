"""Float64 single-token decode against a key/value cache, and the token sampler.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product library.  Everything runs on
the host CPU in float64 (the sampler compares the logits as given).

Decode (Hephaistos, feature list: "True KV Cache", prefill once then one
position per call; strata, model table: KV-cache parity with pre-rotated keys):
position t of every sequence goes through the same layers as the full forward,
but its query attends only to the cached keys and values of positions 0..t.
Keys enter the cache already rotated by RoPE at their own position and are
never rotated again.  strata's gate is that decoding a sequence position by
position reproduces the full forward's logits (to ~1e-9 in float64).

Sampler (Hephaistos, Sampling: temperature + top-k; strata, sampler row:
temperature / top-k / top-p; randyGPT: top-p (nucleus) + temperature;
Transformer-In-Rust, sampling pipeline: repetition penalty, temperature,
top-k, top-p, random sample).  Readings taken where the pages are silent:
  * temperature 0 (or top_k = 1) is greedy: the largest logit, the lowest id
    among equal maxima;
  * the top-k set is the first k ids in the order (logit descending, id
    ascending), so ties at the cut go to the lower ids; top_k <= 0 or >= V
    keeps the whole vocabulary;
  * weights w_i = exp((z_i - max z) / temperature) over the set;
  * the draw is the inverse CDF in increasing id order: the smallest id i in
    the set whose cumulative weight exceeds u * sum(w), with u in [0, 1)
    supplied by the caller (random numbers are inputs, not drawn here).
The distribution is softmax(z / temperature) restricted to the set and
renormalised, whatever order the CDF walks; id order needs no sort.
  * repetition penalty r (the usual form, Keskar et al. 2019): before
    anything else, every id present in the sequence's history has its logit
    divided by r when positive and multiplied by r otherwise, in float32 (the
    logits' own precision, so both sides see the same penalised logits);
  * top-p (nucleus) applies inside the top-k set: walking the set in the
    (logit descending, id ascending) order, keep the shortest prefix whose
    weight reaches top_p of the set's total (at least one id), then draw
    from that prefix as above.
"""
import numpy as np

from .oracle import param_layout, rmsnorm_fwd, rope, swiglu_fwd


class KVCache:
    """Per layer: K and V [B, H_kv, T, hd] in float64 (K rotated)."""

    def __init__(self, cfg, batch=None):
        B = cfg["batch"] if batch is None else batch
        hd = cfg["d_model"] // cfg["n_head"]
        shape = (B, cfg["n_kv_head"], cfg["ctx"], hd)
        self.K = [np.zeros(shape) for _ in range(cfg["n_layer"])]
        self.V = [np.zeros(shape) for _ in range(cfg["n_layer"])]


def _tensors(cfg, params):
    p = np.asarray(params, dtype=np.float64)
    out = {}
    for name, off, rows, cols in param_layout(cfg):
        t = p[off:off + rows * cols]
        out[name] = t.reshape(rows, cols) if rows > 1 else t
    return out


def decode_step(cfg, params, cache, tokens, pos):
    """Logits [B, V] of position pos for tokens [B] (ids at that position);
    writes the position's rotated keys and values into cache."""
    V, d, L = cfg["vocab"], cfg["d_model"], cfg["n_layer"]
    H, Hkv, h = cfg["n_head"], cfg["n_kv_head"], cfg["d_ff"]
    hd, eps, base = d // H, cfg["rms_eps"], cfg["rope_base"]
    rs = cfg.get("rope_scale", 1.0)
    kvd, G = Hkv * hd, H // Hkv
    P = _tensors(cfg, params)
    tok = np.asarray(tokens, dtype=np.int64).reshape(-1)
    B = tok.size
    x = P["wte"][tok].copy()  # [B, d]; no position table
    for l in range(L):
        xn, _ = rmsnorm_fwd(x, P[f"l{l}.g1"], eps)
        qkv = xn @ P[f"l{l}.Wqkv"]
        q = qkv[:, :d].reshape(B, H, hd)
        k = qkv[:, d:d + kvd].reshape(B, Hkv, hd)
        v = qkv[:, d + kvd:].reshape(B, Hkv, hd)
        for b in range(B):
            for hh in range(H):
                q[b, hh] = rope(q[b, hh], pos, base, scale=rs)
            for g in range(Hkv):
                cache.K[l][b, g, pos] = rope(k[b, g], pos, base, scale=rs)
                cache.V[l][b, g, pos] = v[b, g]
        o = np.zeros((B, H, hd))
        for b in range(B):
            for hh in range(H):
                g = hh // G  # contiguous query-head groups share a key/value head
                s = cache.K[l][b, g, :pos + 1] @ q[b, hh] / np.sqrt(hd)
                w = np.exp(s - s.max())
                o[b, hh] = (w / w.sum()) @ cache.V[l][b, g, :pos + 1]
        x = x + o.reshape(B, d) @ P[f"l{l}.Wo"]
        xn2, _ = rmsnorm_fwd(x, P[f"l{l}.g2"], eps)
        w13 = P[f"l{l}.W13"]
        u = swiglu_fwd(xn2 @ w13[:, :h], xn2 @ w13[:, h:])
        x = x + u @ P[f"l{l}.W2"]
    xf, _ = rmsnorm_fwd(x, P["gf"], eps)
    return xf @ P["Wlm"]


def topk_set(z, top_k):
    """Ids of the top-k set in increasing id order (the whole vocabulary when
    top_k <= 0 or top_k >= V)."""
    z = np.asarray(z)
    V = z.size
    if top_k <= 0 or top_k >= V:
        return np.arange(V)
    order = np.lexsort((np.arange(V), -z))  # logit descending, then id ascending
    return np.sort(order[:top_k])


def sample_cdf(z, temperature, top_k):
    """(ids of the set, float64 cumulative weights over them, total)."""
    S = topk_set(z, top_k)
    zf = np.asarray(z, dtype=np.float64)
    w = np.exp((zf[S] - zf.max()) / temperature)
    C = np.cumsum(w)
    return S, C, C[-1]


def penalise(z, penalty, history):
    """Logits after the repetition penalty (float32 arithmetic)."""
    z = np.array(z, dtype=np.float32)
    if penalty == 1.0:
        return z
    r = np.float32(penalty)
    for i in sorted({int(h) for h in history if 0 <= int(h) < z.size}):
        z[i] = z[i] / r if z[i] > 0 else z[i] * r
    return z


def nucleus(z, temperature, top_k, top_p):
    """Ids of the top-p prefix of the top-k set, in increasing id order, and
    the float64 cumulative weights along the (logit desc, id asc) walk."""
    S = topk_set(z, top_k)
    zf = np.asarray(z, dtype=np.float64)
    order = S[np.lexsort((S, -zf[S]))]  # logit descending, then id ascending
    w = np.exp((zf[order] - zf.max()) / temperature)
    C = np.cumsum(w)
    n = 1 + int(np.searchsorted(C, top_p * C[-1], side="left"))
    return np.sort(order[:min(n, order.size)]), C


def sample(z, temperature, top_k, u, top_p=1.0, penalty=1.0, history=()):
    """Token id drawn from logits z [V] with uniform u in [0, 1)."""
    z = penalise(z, penalty, history) if penalty != 1.0 else np.asarray(z)
    if temperature <= 0 or top_k == 1:
        return int(np.argmax(z))  # first maximum = lowest id among ties
    if top_p < 1.0:
        S, _ = nucleus(z, temperature, top_k, top_p)
        zf = np.asarray(z, dtype=np.float64)
        C = np.cumsum(np.exp((zf[S] - zf.max()) / temperature))
        i = int(np.searchsorted(C, float(u) * C[-1], side="right"))
        return int(S[min(i, S.size - 1)])
    S, C, W = sample_cdf(z, temperature, top_k)
    i = int(np.searchsorted(C, float(u) * W, side="right"))
    return int(S[min(i, S.size - 1)])
