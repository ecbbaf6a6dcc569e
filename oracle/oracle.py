"""ctypes wrapper of the float64 oracle (llama_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product library.  Arrays in and
out are numpy float64 / int32; everything is computed on the host CPU.
"""
import ctypes as C
import os

import numpy as np

from .build import build

# LLM_ORACLE_LIB: another build of llama_oracle.c to load (the sanitizer test
# loads one built with AddressSanitizer and UBSan)
_lib = C.CDLL(os.environ.get("LLM_ORACLE_LIB") or build())

_D = C.POINTER(C.c_double)
_I32 = C.POINTER(C.c_int32)
_I64 = C.POINTER(C.c_int64)


class OrcCfg(C.Structure):
    _fields_ = [("V", C.c_int32), ("d", C.c_int32), ("L", C.c_int32), ("H", C.c_int32),
                ("Hkv", C.c_int32), ("h", C.c_int32), ("T", C.c_int32), ("B", C.c_int32),
                ("rope_base", C.c_double), ("eps", C.c_double), ("rope_scale", C.c_double)]


def _cfg(cfg) -> OrcCfg:
    """cfg: a mapping with vocab, d_model, n_layer, n_head, n_kv_head, d_ff,
    ctx, batch, rope_base, rms_eps."""
    return OrcCfg(cfg["vocab"], cfg["d_model"], cfg["n_layer"], cfg["n_head"], cfg["n_kv_head"],
                  cfg["d_ff"], cfg["ctx"], cfg["batch"], float(cfg.get("rope_base", 10000.0)),
                  float(cfg.get("rms_eps", 1e-5)), float(cfg.get("rope_scale", 1.0)))


def _dp(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(_D)


def _ip(a):
    if a is None:
        return None
    assert a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data_as(_I32)


_lib.orc_n_params.restype = C.c_int64
_lib.orc_n_params.argtypes = [C.POINTER(OrcCfg)]
_lib.orc_param_layout.restype = C.c_int
_lib.orc_param_layout.argtypes = [C.POINTER(OrcCfg), _I64, _I64, _I64]
for _n in ("orc_mm_nn", "orc_mm_tn", "orc_mm_nt"):
    getattr(_lib, _n).restype = None
    getattr(_lib, _n).argtypes = [C.c_int, C.c_int, C.c_int, _D, C.c_int64, _D, C.c_int64, _D,
                                  C.c_int64, C.c_int]
_lib.orc_rmsnorm_fwd.restype = None
_lib.orc_rmsnorm_fwd.argtypes = [C.c_int, C.c_int, _D, _D, C.c_double, _D, _D]
_lib.orc_rmsnorm_bwd.restype = None
_lib.orc_rmsnorm_bwd.argtypes = [C.c_int, C.c_int, _D, _D, _D, _D, _D, _D, C.c_int]
_lib.orc_rope.restype = None
_lib.orc_rope.argtypes = [_D, C.c_int, C.c_int, C.c_double, C.c_int]
_lib.orc_rope_pos.restype = None
_lib.orc_rope_pos.argtypes = [_D, C.c_int, C.c_double, C.c_double, C.c_int]
_lib.orc_attention_fwd.restype = None
_lib.orc_attention_fwd.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, _D, _D, _D, _D]
_lib.orc_attention_bwd.restype = None
_lib.orc_attention_bwd.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, _D, _D, _D]
_lib.orc_swiglu_fwd.restype = None
_lib.orc_swiglu_fwd.argtypes = [C.c_int64, _D, _D, _D]
_lib.orc_swiglu_bwd.restype = None
_lib.orc_swiglu_bwd.argtypes = [C.c_int64, _D, _D, _D, _D, _D]
_lib.orc_ce_fwd_bwd.restype = C.c_double
_lib.orc_ce_fwd_bwd.argtypes = [C.c_int, C.c_int, _D, _I32, C.c_double, _D]
_lib.orc_embed_bwd.restype = None
_lib.orc_embed_bwd.argtypes = [C.c_int64, C.c_int, C.c_int, _I32, _D, _D]
_lib.orc_forward_backward.restype = C.c_double
_lib.orc_forward_backward.argtypes = [C.POINTER(OrcCfg), _D, _I32, _I32, _D, _D]
_lib.orc_forward_backward_dropout.restype = C.c_double
_lib.orc_forward_backward_dropout.argtypes = [C.POINTER(OrcCfg), _D, _I32, _I32, _D, _D,
                                              C.c_double, C.c_uint64, C.c_uint32]
_lib.orc_philox4x32_10.restype = None
_lib.orc_philox4x32_10.argtypes = [C.POINTER(C.c_uint32), C.POINTER(C.c_uint32),
                                   C.POINTER(C.c_uint32)]
_lib.orc_dropout_factors.restype = None
_lib.orc_dropout_factors.argtypes = [C.c_double, C.c_uint64, C.c_uint32, C.c_int, C.c_int,
                                     C.c_uint64, C.c_int64, _D]
_lib.orc_adamw.restype = None
_lib.orc_adamw.argtypes = [C.c_int64, _D, _D, _D, _D, C.c_int64, C.c_double, C.c_double,
                           C.c_double, C.c_double, C.c_double]


def n_params(cfg) -> int:
    c = _cfg(cfg)
    return int(_lib.orc_n_params(C.byref(c)))


_NAMES_LAYER = ("g1", "Wqkv", "Wo", "g2", "W13", "W2")


def param_layout(cfg):
    """[(name, offset, rows, cols)] in flat-buffer order."""
    c = _cfg(cfg)
    n = _lib.orc_param_layout(C.byref(c), None, None, None)
    offs, rows, cols = (np.zeros(n, np.int64) for _ in range(3))
    _lib.orc_param_layout(C.byref(c), offs.ctypes.data_as(_I64), rows.ctypes.data_as(_I64),
                          cols.ctypes.data_as(_I64))
    names = ["wte"] + [f"l{l}.{nm}" for l in range(cfg["n_layer"]) for nm in _NAMES_LAYER]
    names += ["gf", "Wlm"]
    return [(nm, int(o), int(r), int(k)) for nm, o, r, k in zip(names, offs, rows, cols)]


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def mm_nn(A, B):
    A, B = _f64(A), _f64(B)
    M, K = A.shape
    N = B.shape[1]
    Cm = np.zeros((M, N))
    _lib.orc_mm_nn(M, K, N, _dp(A), K, _dp(B), N, _dp(Cm), N, 0)
    return Cm


def mm_tn(A, B):
    """A^T B with A [K,M], B [K,N]."""
    A, B = _f64(A), _f64(B)
    K, M = A.shape
    N = B.shape[1]
    Cm = np.zeros((M, N))
    _lib.orc_mm_tn(M, K, N, _dp(A), M, _dp(B), N, _dp(Cm), N, 0)
    return Cm


def mm_nt(A, B):
    """A B^T with A [M,K], B [N,K]."""
    A, B = _f64(A), _f64(B)
    M, K = A.shape
    N = B.shape[0]
    Cm = np.zeros((M, N))
    _lib.orc_mm_nt(M, K, N, _dp(A), K, _dp(B), K, _dp(Cm), N, 0)
    return Cm


def rmsnorm_fwd(x, g, eps=1e-5):
    x, g = _f64(x), _f64(g)
    n, d = x.shape
    y, r = np.zeros_like(x), np.zeros(n)
    _lib.orc_rmsnorm_fwd(n, d, _dp(x), _dp(g), eps, _dp(y), _dp(r))
    return y, r


def rmsnorm_bwd(x, rstd, g, dy):
    x, rstd, g, dy = _f64(x), _f64(rstd), _f64(g), _f64(dy)
    n, d = x.shape
    dx, dg = np.zeros_like(x), np.zeros(d)
    _lib.orc_rmsnorm_bwd(n, d, _dp(x), _dp(rstd), _dp(g), _dp(dy), _dp(dx), _dp(dg), 0)
    return dx, dg


def rope(u, t, base=10000.0, sign=1, scale=1.0):
    """RoPE of head vector u at position t (t / scale with interpolation)."""
    u = _f64(u).copy()
    if scale == 1.0:
        _lib.orc_rope(_dp(u), u.shape[0], int(t), float(base), int(sign))
    else:
        _lib.orc_rope_pos(_dp(u), u.shape[0], float(t) / float(scale), float(base), int(sign))
    return u


def attention_fwd(qkv, d, H, Hkv, want_probs=False):
    """qkv [T, d+2kvd] (RoPE applied) -> o [T,d], lse [H,T], P [H,T,T] or None."""
    qkv = _f64(qkv)
    T = qkv.shape[0]
    o, lse = np.zeros((T, d)), np.zeros((H, T))
    P = np.zeros((H, T, T)) if want_probs else None
    _lib.orc_attention_fwd(T, d, H, Hkv, _dp(qkv), _dp(o), _dp(lse), _dp(P))
    return o, lse, P


def attention_bwd(qkv, dout, d, H, Hkv):
    qkv, dout = _f64(qkv), _f64(dout)
    dqkv = np.zeros_like(qkv)
    _lib.orc_attention_bwd(qkv.shape[0], d, H, Hkv, _dp(qkv), _dp(dout), _dp(dqkv))
    return dqkv


def swiglu_fwd(a, b):
    a, b = _f64(a), _f64(b)
    u = np.zeros_like(a)
    _lib.orc_swiglu_fwd(a.size, _dp(a), _dp(b), _dp(u))
    return u


def swiglu_bwd(a, b, du):
    a, b, du = _f64(a), _f64(b), _f64(du)
    da, db = np.zeros_like(a), np.zeros_like(a)
    _lib.orc_swiglu_bwd(a.size, _dp(a), _dp(b), _dp(du), _dp(da), _dp(db))
    return da, db


def ce_fwd_bwd(z, y, inv_count=None):
    """Returns (sum of row losses, dz) with dz = (softmax - onehot) * inv_count."""
    z = _f64(z)
    y = np.ascontiguousarray(y, dtype=np.int32)
    n, V = z.shape
    if inv_count is None:
        inv_count = 1.0 / n
    dz = np.zeros_like(z)
    s = _lib.orc_ce_fwd_bwd(n, V, _dp(z), _ip(y), float(inv_count), _dp(dz))
    return s, dz


def embed_bwd(tok, dx, vocab):
    """dwte [vocab, d] = scatter-add of dx rows by token id, in position order."""
    tok = np.ascontiguousarray(tok, dtype=np.int32).reshape(-1)
    dx = _f64(dx)
    out = np.zeros((vocab, dx.shape[1]))
    _lib.orc_embed_bwd(tok.size, dx.shape[1], int(vocab), _ip(tok), _dp(dx), _dp(out))
    return out


def philox4x32_10(counter, key):
    """Philox4x32-10 of four 32-bit counter words and two key words."""
    c = (C.c_uint32 * 4)(*[int(x) & 0xffffffff for x in counter])
    k = (C.c_uint32 * 2)(*[int(x) & 0xffffffff for x in key])
    out = (C.c_uint32 * 4)()
    _lib.orc_philox4x32_10(c, k, out)
    return [int(x) for x in out]


def dropout_factors(p, seed, step, site, layer, n, e0=0):
    """Factors (0 or 1/(1-p)) of elements [e0, e0+n) of a dropout site."""
    out = np.zeros(n)
    _lib.orc_dropout_factors(float(p), int(seed), int(step), int(site), int(layer), int(e0),
                             int(n), _dp(out))
    return out


def forward_backward(cfg, params, tokens, targets=None, want_logits=True, want_grads=True,
                     dropout=None):
    """Returns (loss, logits [B*T, V] or None, grads [P] or None).  dropout:
    None or (p, seed, step) for the training forward with inverted dropout."""
    c = _cfg(cfg)
    params = _f64(params)
    tokens = np.ascontiguousarray(tokens, dtype=np.int32).reshape(-1)
    tg = None if targets is None else np.ascontiguousarray(targets, dtype=np.int32).reshape(-1)
    N = cfg["batch"] * cfg["ctx"]
    assert tokens.size == N and params.size == n_params(cfg)
    logits = np.zeros((N, cfg["vocab"])) if want_logits else None
    grads = np.zeros(params.size) if (want_grads and tg is not None) else None
    if dropout is None:
        loss = _lib.orc_forward_backward(C.byref(c), _dp(params), _ip(tokens), _ip(tg),
                                         _dp(logits), _dp(grads))
    else:
        pd, seed, stp = dropout
        loss = _lib.orc_forward_backward_dropout(C.byref(c), _dp(params), _ip(tokens), _ip(tg),
                                                 _dp(logits), _dp(grads), float(pd), int(seed),
                                                 int(stp))
    return float(loss), logits, grads


def adamw(p, g, m, v, t, lr, wd, b1=0.9, b2=0.999, eps=1e-8):
    """In-place AdamW on float64 arrays p, m, v with gradient g; returns (p, m, v)."""
    p, g, m, v = _f64(p).copy(), _f64(g), _f64(m).copy(), _f64(v).copy()
    _lib.orc_adamw(p.size, _dp(p), _dp(g), _dp(m), _dp(v), int(t), float(lr), float(wd),
                   float(b1), float(b2), float(eps))
    return p, m, v


def step(cfg, params, m, v, t, tokens, targets, lr, wd, b1=0.9, b2=0.999, eps=1e-8):
    """One full training step: (loss, logits, grads, new_params, new_m, new_v)."""
    loss, logits, grads = forward_backward(cfg, params, tokens, targets)
    p2, m2, v2 = adamw(params, grads, m, v, t, lr, wd, b1, b2, eps)
    return loss, logits, grads, p2, m2, v2
