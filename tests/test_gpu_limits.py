"""GPU parity at the limits the configuration check accepts: the largest head
size (128: the CUDA-core attention's register rows, one GEMV block per head in
decode) on a ragged context with GQA, the smallest (2), and the widest model
(d_model 4096: the row-wise kernels' widest rows; hidden size 1024 keeps the
float64 host copies of the parameters small)."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import get_config, make_batch, make_params
from tests.gpu_util import TOL, compare, rel, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

LIMITS = [
    ("hd128_gqa_bf16", "c3", dict(batch=2, ctx=70, n_layer=1, d_model=256, n_head=2,
                                  n_kv_head=1, d_ff=682)),
    ("hd2_fp32", "c1", dict(batch=2, ctx=16, n_layer=1, d_model=8, n_head=4, n_kv_head=2,
                            d_ff=21)),
    ("d4096_bf16", "c3", dict(batch=1, ctx=16, n_layer=1, vocab=64, d_model=4096, n_head=32,
                              n_kv_head=8, d_ff=1024)),
]


@pytest.mark.parametrize("tag,name,over", LIMITS, ids=[x[0] for x in LIMITS])
def test_step_at_the_limits_matches_oracle(tag, name, over):
    cfg = get_config(name, **over)
    lay = O.param_layout(cfg)
    p = make_params(cfg, lay)
    tok, tgt = make_batch(cfg)
    gpu = run_gpu(cfg, p, tok, tgt, steps=1)
    ref = run_oracle(cfg, p, tok, tgt, steps=1)
    compare(cfg, lay, gpu, ref, prev_params=p.astype(np.float64))


def test_decode_at_head_size_128_matches_full_forward():
    from scratch_llama_decoder_b200 import LlamaStep
    cfg = get_config("c3", batch=2, ctx=70, n_layer=1, d_model=256, n_head=2, n_kv_head=1,
                     d_ff=682)
    p = make_params(cfg, O.param_layout(cfg))
    tok, _ = make_batch(cfg)
    tok = tok.reshape(2, 70)
    _, zref, _ = O.forward_backward(cfg, p, tok, want_grads=False)
    zref = zref.reshape(2, 70, -1)
    m = LlamaStep(cfg)
    P = torch.tensor(p, device="cuda")
    m.forward(P, torch.tensor(tok, device="cuda"))
    worst = 0.0
    for t in range(40, 70):
        z = m.decode(P, torch.tensor(tok[:, t], device="cuda"), t).double().cpu().numpy()
        worst = max(worst, max(rel(z[b], zref[b, t]) for b in range(2)))
    assert m.status() == 0 and worst <= TOL["bf16"]["logits"], worst
    m.close()
