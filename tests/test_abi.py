"""Host-side checks of the C-ABI library (no GPU needed, no compute calls).

The library must load, export every function include/llm.h declares, agree
with the oracle on the flat parameter layout, and reject invalid configs and
arguments on the host.
"""
import ctypes as C
import os
import re

import pytest

import oracle as O
from synth import CONFIGS, get_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header):
    src = open(os.path.join(ROOT, "include", header)).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(llm_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    import scratch_llama_decoder_b200 as P
    headers = [h for h in os.listdir(os.path.join(ROOT, "include")) if h.endswith(".h")]
    names = [n for h in headers for n in _declared(h)]
    assert "llm_step" in names and "llm_forward" in names and "llm_init" in names
    for n in names:
        assert hasattr(P.lib, n), n  # ctypes resolves the symbol via dlsym
        # every entry point has declared argument types: int64_t sizes must
        # never be passed as 32-bit ints
        assert n in P._lib.EXPORTS, n


def test_binding_argtypes_match_header_arity():
    import scratch_llama_decoder_b200 as P
    src = ""
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src += re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", h)).read(),
                          flags=re.S)
    for name, (_, args) in P._lib.EXPORTS.items():
        m = re.search(r"\b" + name + r"\s*\(([^)]*)\)", src)
        assert m, name
        params = [a for a in m.group(1).split(",") if a.strip() and a.strip() != "void"]
        assert len(params) == len(args), (name, len(params), len(args))
        for decl, ct in zip(params, args):
            if "*" in decl:
                continue
            if re.search(r"\buint64_t\b", decl):
                assert ct is P._lib._u64, (name, decl)
            elif re.search(r"\bint64_t\b", decl):
                assert ct is P._lib._i64, (name, decl)


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_layout_matches_oracle(name):
    from scratch_llama_decoder_b200 import llm_param_layout, llm_workspace_bytes
    cfg = get_config(name)
    lay, n = llm_param_layout(cfg)
    assert lay == O.param_layout(cfg)
    assert n == O.n_params(cfg)
    assert llm_workspace_bytes(cfg) > 0


def test_gqa_layout_matches_oracle():
    from scratch_llama_decoder_b200 import llm_param_layout
    cfg = get_config("c4", n_layer=3)
    lay, n = llm_param_layout(cfg)
    assert lay == O.param_layout(cfg) and n == O.n_params(cfg)


@pytest.mark.parametrize("bad", [dict(d_model=18, n_head=4), dict(n_head=4, n_kv_head=3),
                                 dict(d_model=12, n_head=4), dict(vocab=0), dict(compute=7),
                                 dict(batch=0)])
def test_invalid_config_rejected(bad):
    import scratch_llama_decoder_b200 as P
    cfg = get_config("c1", **bad)
    c = P.make_config(cfg)
    b = C.c_int64(0)
    assert P.lib.llm_workspace_bytes(C.byref(c), C.byref(b)) == P.LLM_ERR_CONFIG
    n, npar = C.c_int(0), C.c_int64(0)
    assert P.lib.llm_param_layout(C.byref(c), None, C.byref(n), C.byref(npar)) == P.LLM_ERR_CONFIG
    ctx = C.c_void_p()
    assert P.lib.llm_create(C.byref(c), C.c_void_p(256), 1 << 30, None, C.byref(ctx)) == \
        P.LLM_ERR_CONFIG


def test_bad_arguments_rejected_on_host():
    import scratch_llama_decoder_b200 as P
    c = P.make_config(get_config("c1"))
    ctx = C.c_void_p()
    # null / misaligned workspace, too-small workspace: rejected before any launch
    assert P.lib.llm_create(C.byref(c), None, 1 << 20, None, C.byref(ctx)) == P.LLM_ERR_ARG
    assert P.lib.llm_create(C.byref(c), C.c_void_p(0x1001), 1 << 20, None, C.byref(ctx)) == \
        P.LLM_ERR_ARG
    assert P.lib.llm_create(C.byref(c), C.c_void_p(0x10000), 16, None, C.byref(ctx)) == \
        P.LLM_ERR_ARG
    # layout with too small an output array
    n, npar = C.c_int(1), C.c_int64(0)
    arr = (P._lib.llm_tensor_info * 1)()
    assert P.lib.llm_param_layout(C.byref(c), arr, C.byref(n), C.byref(npar)) == P.LLM_ERR_ARG
    assert P.lib.llm_step(None, None, None, None, None, 1, None, None, 0.0, 0.0, None) == \
        P.LLM_ERR_ARG
    assert P.lib.llm_forward(None, None, None, None) == P.LLM_ERR_ARG
    assert P.lib.llm_status(None) == P.LLM_ERR_ARG
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert P.lib.llm_error_string(code)


def test_recompute_workspace_keeps_one_layer_of_activations():
    """recompute = 1 drops the saved activations of all but one layer: the
    workspace shrinks by (L - 1) x (x1 in float32; xn1, q|k|v, o, xn2, [a|b],
    u in the operand type; rstd1, rstd2, lse in float32), up to alignment."""
    from scratch_llama_decoder_b200 import llm_workspace_bytes
    from synth import get_config
    cfg = get_config("c5")
    w0 = llm_workspace_bytes(cfg)
    w1 = llm_workspace_bytes(dict(cfg, recompute=1))
    N, d, L, H = cfg["batch"] * cfg["ctx"], cfg["d_model"], cfg["n_layer"], cfg["n_head"]
    hp = (cfg["d_ff"] + 63) // 64 * 64
    qkvw = d + 2 * cfg["n_kv_head"] * (d // H)
    per_layer = 4 * N * d + 2 * N * (d + qkvw + d + d + 2 * hp + hp) + 4 * N * (2 + H)
    assert abs((w0 - w1) - (L - 1) * per_layer) <= 11 * 256
    assert w1 < w0 / 3  # the 350M step's workspace is mostly saved activations
    import scratch_llama_decoder_b200 as P
    with pytest.raises(P.LLMError):
        llm_workspace_bytes(dict(cfg, recompute=2))


def test_every_context_call_refuses_a_null_context():
    """Every entry point taking an llm_ctx (read from include/llm.h) returns
    LLM_ERR_ARG for a null context before touching a device; llm_destroy
    ignores it and llm_last_launch_count reports 0."""
    import re
    import scratch_llama_decoder_b200 as P
    hdr = open(os.path.join(ROOT, "include", "llm.h")).read()
    names = re.findall(r"^\w[\w ]*?\**\s*(llm_\w+)\((?:const )?llm_ctx \*", hdr, re.M)
    assert len(names) >= 20
    fill = {C.c_void_p: None, C.c_int: 1, C.c_int64: 1, C.c_uint64: 1, C.c_float: 1.0,
            C.c_double: 1.0}
    for name in names:
        fn = getattr(P.lib, name)
        args = [None] + [fill.get(t) for t in fn.argtypes[1:]]
        rc = fn(*args)
        if name == "llm_destroy":
            assert rc is None
        elif name == "llm_last_launch_count":
            assert rc == 0
        else:
            assert rc == P.LLM_ERR_ARG, name


@pytest.mark.parametrize("name,over", [("c1", {}), ("c4", {}), ("c5", {}), ("c1", dict(n_layer=0))])
def test_grad_buckets_tile_the_gradient_in_backward_order(name, over):
    """llm_grad_bucket_range: n_layer + 2 contiguous buckets covering the flat
    gradient exactly once, numbered in the order the backward finishes them
    (head, layers from the last, embedding)."""
    import scratch_llama_decoder_b200 as P
    cfg = get_config(name, **over)
    b = P.grad_buckets(cfg)
    L = cfg["n_layer"]
    assert len(b) == L + 2
    lay = {nm: (off, r * k) for nm, off, r, k in O.param_layout(cfg)}
    n = O.n_params(cfg)
    assert sorted(b) == [(o, c) for o, c in sorted(b)]
    pos = 0
    for off, cnt in sorted(b):  # a tiling of [0, n)
        assert off == pos and cnt > 0
        pos += cnt
    assert pos == n
    assert b[-1] == (0, lay["wte"][1])                    # the embedding comes last
    assert b[0] == (lay["gf"][0], n - lay["gf"][0])       # the head first
    for k in range(1, L + 1):                              # then layers L-1 .. 0
        mine = [v for nm, v in lay.items() if nm.startswith(f"l{L - k}.")]
        assert b[k] == (lay[f"l{L - k}.g1"][0], sum(c for _, c in mine))
    c = P.make_config(cfg)
    off, cnt = C.c_int64(0), C.c_int64(0)
    assert P.lib.llm_grad_bucket_range(C.byref(c), L + 2, C.byref(off), C.byref(cnt)) == \
        P.LLM_ERR_ARG
    assert P.lib.llm_grad_bucket_range(C.byref(c), -1, C.byref(off), C.byref(cnt)) == \
        P.LLM_ERR_ARG
    bad = P.make_config(get_config(name, **dict(over, n_head=3)))
    assert P.lib.llm_grad_bucket_range(C.byref(bad), 0, C.byref(off), C.byref(cnt)) == \
        P.LLM_ERR_CONFIG
