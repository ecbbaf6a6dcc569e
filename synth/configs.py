"""The five named workloads of the Llama training step.

Sizes follow the workload list of this project: a tiny fp32 decoder (the
microgpt-sized case), an fp32 8-layer decoder, a bf16 6-layer decoder, a GQA
8-layer decoder and a ~350M-parameter 20-layer decoder (CodeGen-350M's width
and depth from the Transformer-In-Rust page).  d_ff = floor(8/3 * d_model)
(Hephaistos, Architecture at a glance: SwiGLU hidden width).
"""

_BASE = dict(rope_base=10000.0, rms_eps=1e-5, beta1=0.9, beta2=0.999, adam_eps=1e-8)


def _mk(name, index, vocab, d_model, n_layer, n_head, n_kv_head, ctx, batch, compute, init_std,
        scale_out_proj, lr, wd, token_dist):
    c = dict(_BASE)
    c.update(name=name, index=index, vocab=vocab, d_model=d_model, n_layer=n_layer, n_head=n_head,
             n_kv_head=n_kv_head, d_ff=(8 * d_model) // 3, ctx=ctx, batch=batch, compute=compute,
             init_std=init_std, scale_out_proj=scale_out_proj, lr=lr, wd=wd,
             token_dist=token_dist)
    return c


CONFIGS = {
    c["name"]: c
    for c in [
        _mk("tiny-v27-d16-l1-fp32", 0, 27, 16, 1, 4, 4, 16, 1, "fp32", 0.08, False, 1e-2, 0.1,
            "uniform"),
        _mk("v500-d128-l8-fp32", 1, 500, 128, 8, 4, 4, 256, 64, "fp32", 0.02, True, 1e-4, 0.1,
            "zipf"),
        _mk("v2000-d256-l6-bf16", 2, 2000, 256, 6, 8, 8, 256, 64, "bf16", 0.02, True, 1e-4, 0.1,
            "zipf"),
        _mk("gqa-v8192-d512-l8-bf16", 3, 8192, 512, 8, 8, 2, 512, 32, "bf16", 0.02, False, 1e-4,
            0.1, "zipf"),
        _mk("350m-v32000-d1024-l20-bf16", 4, 32000, 1024, 20, 16, 16, 2048, 8, "bf16", 0.02, True,
            3e-4, 0.1, "zipf"),
    ]
}

ALIASES = {"c1": "tiny-v27-d16-l1-fp32", "c2": "v500-d128-l8-fp32", "c3": "v2000-d256-l6-bf16",
           "c4": "gqa-v8192-d512-l8-bf16", "c5": "350m-v32000-d1024-l20-bf16"}


def get_config(which: str, **overrides):
    """A copy of a named config (or alias c1..c5) with fields overridden."""
    c = dict(CONFIGS[ALIASES.get(which, which)])
    c.update(overrides)
    return c
