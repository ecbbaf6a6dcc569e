"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
compare with the float64 oracle using norm-wise relative error per tensor."""
import numpy as np
import torch

# Tolerances of the training step (norm-wise relative error per tensor).
#   fp32 configs: loss and logits 1e-4; gradients, updated parameters and the
#   Adam moments 1e-3.
#   bf16 configs: loss 5e-3; logits, gradients and m 2e-2; v = (1-b2) g^2
#   carries twice the relative error of g, so v gets 4e-2.  The updated
#   parameters are measured but not gated: at t = 1 AdamW moves each element
#   by about lr * sign(g), so every gradient element within bf16 rounding of
#   zero can flip a whole 2*lr step (2% of W2 at the 350M workload, whose
#   scaled init is 0.003 against lr 3e-4).
# The AdamW update itself is checked in isolation for both precisions: the
# float64 oracle AdamW applied to the GPU's own gradients and previous state
# must give the GPU's update (p_new - p_old) to 1e-3 and its m, v to 1e-5
# (float32 arithmetic; the update is recovered from float32 parameters, whose
# rounding is ~1e-5 of the update).
TOL = {
    "fp32": dict(loss=1e-4, logits=1e-4, grads=1e-3, params=1e-3, m=1e-3, v=1e-3),
    "bf16": dict(loss=5e-3, logits=2e-2, grads=2e-2, params=None, m=2e-2, v=4e-2),
}
ADAMW_DP_TOL, ADAMW_MV_TOL = 1e-3, 1e-5


def rel(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    if nb == 0.0:
        return float(np.linalg.norm(a))
    return float(np.linalg.norm(a - b) / nb)


def run_gpu(cfg, params, tok, tgt, steps=1, lr=None, wd=None, clip=None):
    """Returns dict with logits (pre-step forward), and per step: loss, grads,
    params, m, v (numpy float64), and with clip (global-norm clipping
    threshold) the norm before clipping."""
    from scratch_llama_decoder_b200 import LlamaStep
    lr = cfg["lr"] if lr is None else lr
    wd = cfg["wd"] if wd is None else wd
    m = LlamaStep(cfg)
    if clip is not None:
        m.set_grad_clip(clip)
    if cfg.get("rope_scale", 1.0) != 1.0:
        m.set_rope_scale(cfg["rope_scale"])
    P = torch.tensor(params, dtype=torch.float32, device="cuda")
    G = torch.zeros_like(P)
    M = torch.zeros_like(P)
    V = torch.zeros_like(P)
    td = torch.tensor(tok, dtype=torch.int32, device="cuda").contiguous()
    yd = torch.tensor(tgt, dtype=torch.int32, device="cuda").contiguous()
    logits = m.forward(P, td)
    out = {"logits": logits.double().cpu().numpy().reshape(-1, cfg["vocab"]), "steps": []}
    assert m.status() == 0
    for t in range(1, steps + 1):
        loss = m.step(P, G, M, V, t, td, yd, lr, wd)
        st = m.status()
        out["steps"].append(dict(status=st, loss=float(loss.item()),
                                 grads=G.double().cpu().numpy(), params=P.double().cpu().numpy(),
                                 m=M.double().cpu().numpy(), v=V.double().cpu().numpy(),
                                 norm=m.read_grad_norm() if clip is not None else None))
    out["launches"] = m.last_launch_count()
    m.close()
    return out


def run_oracle(cfg, params, tok, tgt, steps=1, lr=None, wd=None, clip=None):
    import oracle as O
    from oracle import train_terms as TT
    lr = cfg["lr"] if lr is None else lr
    wd = cfg["wd"] if wd is None else wd
    p = np.asarray(params, np.float64)
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    _, logits, _ = O.forward_backward(cfg, p, tok, tgt, want_grads=False)
    out = {"logits": logits, "steps": []}
    for t in range(1, steps + 1):
        loss, _, g = O.forward_backward(cfg, p, tok, tgt, want_logits=False)
        norm = None
        if clip is not None:
            g, norm, _ = TT.clip(g, clip)
        p, m, v = O.adamw(p, g, m, v, t, lr, wd, cfg["beta1"], cfg["beta2"], cfg["adam_eps"])
        out["steps"].append(dict(loss=loss, grads=g, params=p.copy(), m=m.copy(), v=v.copy(),
                                 norm=norm))
    return out


def compare(cfg, layout, gpu, ref, prev_params=None, tol=None):
    """Asserts every gate; returns a dict of the worst errors.  prev_params:
    the parameters before the first step (float64)."""
    import oracle as O
    tol = tol or TOL[cfg["compute"]]
    worst = {"logits": rel(gpu["logits"], ref["logits"])}
    assert worst["logits"] <= tol["logits"], worst
    gp = np.asarray(prev_params, np.float64)
    gm = np.zeros_like(gp)
    gv = np.zeros_like(gp)
    # the C ABI passes lr, wd, betas and eps as float32: use those values
    f32 = lambda x: float(np.float32(x))
    hyp = [f32(cfg[k]) for k in ("lr", "wd", "beta1", "beta2", "adam_eps")]
    for k, (g, r) in enumerate(zip(gpu["steps"], ref["steps"])):
        # AdamW in isolation: oracle AdamW on the GPU's own inputs
        ep, em, ev = O.adamw(gp, g["grads"], gm, gv, k + 1, *hyp)
        for name, off, rows, cols in layout:
            sl = slice(off, off + rows * cols)
            e = rel(g["params"][sl] - gp[sl], ep[sl] - gp[sl])
            worst["adamw_dp"] = max(worst.get("adamw_dp", 0.0), e)
            assert e <= ADAMW_DP_TOL, (k, "adamw_dp", name, e)
            for key, got, want in (("m", g["m"], em), ("v", g["v"], ev)):
                e = rel(got[sl], want[sl])
                worst["adamw_" + key] = max(worst.get("adamw_" + key, 0.0), e)
                assert e <= ADAMW_MV_TOL, (k, "adamw_" + key, name, e)
        gp, gm, gv = g["params"], g["m"], g["v"]
        assert g["status"] == 0, g["status"]
        le = abs(g["loss"] - r["loss"]) / abs(r["loss"])
        worst["loss"] = max(worst.get("loss", 0.0), le)
        assert le <= tol["loss"], (k, g["loss"], r["loss"])
        for key in ("grads", "params", "m", "v"):
            for name, off, rows, cols in layout:
                sl = slice(off, off + rows * cols)
                e = rel(g[key][sl], r[key][sl])
                worst[key] = max(worst.get(key, 0.0), e)
                if tol[key] is not None:
                    assert e <= tol[key], (k, key, name, e)
    return worst
