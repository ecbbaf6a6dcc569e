"""Write sampled float64-oracle results of one full training step at full size.

Calls only the oracle (and the seeded input generators): for a named config
it runs forward + backward + AdamW (t = 1) on the default seeded inputs and
stores, in tests/golden/step_<config>.npz:
  loss                       the mean cross-entropy
  logit_idx, logit_val       4096 sampled (row*V + col) logits
  logit_rows, logit_rowvals  4 full logit rows
  g_idx, g_val, p_val, m_val, v_val
                             per parameter tensor, 256 sampled flat indices
                             (all of a smaller tensor) with the gradient and the
                             post-AdamW parameter, m and v there
  g_norm                     full L2 norm of each tensor's gradient
and, with --rows, in tests/golden/logit_rows_<config>.npz:
  rows, vals                 full logit rows (float32) from the first and the
                             last 128-row block of the [B*T, V] logits (the
                             first and last output tiles of the lm_head GEMM),
                             computed by the oracle's forward on the one
                             sequence each row belongs to (up to the row's
                             block): by causality (pinned in the oracle's
                             tests) those rows equal the whole batch's.
Usage: python tests/golden/make_golden.py [--rows] c2 [c3 ...]
"""
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle as O  # noqa: E402
from synth import get_config, make_batch, make_params  # noqa: E402

SAMPLES_PER_TENSOR = 256
LOGIT_SAMPLES = 4096


def golden(name):
    cfg = get_config(name)
    lay = O.param_layout(cfg)
    p32 = make_params(cfg, lay)
    p = p32.astype(np.float64)
    tok, tgt = make_batch(cfg)
    t0 = time.time()
    loss, logits, grads = O.forward_backward(cfg, p, tok, tgt)
    t1 = time.time()
    zeros = np.zeros_like(p)
    p2, m2, v2 = O.adamw(p, grads, zeros, zeros, 1, cfg["lr"], cfg["wd"], cfg["beta1"],
                         cfg["beta2"], cfg["adam_eps"])
    rng = np.random.default_rng(77)
    N, V = logits.shape
    li = rng.choice(N * V, size=min(LOGIT_SAMPLES, N * V), replace=False)
    rows = rng.choice(N, size=4, replace=False)
    g_idx, g_val, p_val, m_val, v_val, g_norm, t_off, t_cnt = [], [], [], [], [], [], [], []
    for _, off, r, k in lay:
        n = r * k
        idx = np.arange(n) if n <= SAMPLES_PER_TENSOR else np.sort(
            rng.choice(n, SAMPLES_PER_TENSOR, replace=False))
        gi = off + idx
        t_off.append(len(g_idx))
        t_cnt.append(len(idx))
        g_idx.extend(gi.tolist())
        g_val.append(grads[gi])
        p_val.append(p2[gi])
        m_val.append(m2[gi])
        v_val.append(v2[gi])
        g_norm.append(np.linalg.norm(grads[off:off + n]))
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), f"step_{cfg['name']}.npz")
    np.savez_compressed(
        out, loss=np.float64(loss), logit_idx=li.astype(np.int64), logit_val=logits.reshape(-1)[li],
        logit_rows=rows.astype(np.int64), logit_rowvals=logits[rows],
        g_idx=np.array(g_idx, np.int64), g_val=np.concatenate(g_val), p_val=np.concatenate(p_val),
        m_val=np.concatenate(m_val), v_val=np.concatenate(v_val), g_norm=np.array(g_norm),
        t_off=np.array(t_off, np.int64), t_cnt=np.array(t_cnt, np.int64),
        names=np.array([n for n, _, _, _ in lay]), oracle_seconds=np.float64(t1 - t0))
    print(f"{cfg['name']}: loss {loss:.6f}  oracle {t1 - t0:.1f}s -> {out}", flush=True)


def _block_rows(T, N):
    """Global row ids: four from the first 128-row block, four from the last."""
    first = [0, 1, 64, 127]
    last = [N - 128, N - 65, N - 2, N - 1]
    return [r for r in first + last if 0 <= r < N]


def logit_rows(name):
    cfg = get_config(name)
    tok, _ = make_batch(cfg)
    B, T = tok.shape
    p = make_params(cfg, O.param_layout(cfg)).astype(np.float64)
    rows = _block_rows(T, B * T)
    vals = np.zeros((len(rows), cfg["vocab"]), np.float32)
    t0 = time.time()
    for b in sorted({r // T for r in rows}):
        mine = [k for k, r in enumerate(rows) if r // T == b]
        upto = max(rows[k] % T for k in mine) + 1  # positions after the last row are not needed
        sub = dict(cfg, batch=1, ctx=upto)
        _, z, _ = O.forward_backward(sub, p, np.ascontiguousarray(tok[b:b + 1, :upto]),
                                     want_grads=False)
        for k in mine:
            vals[k] = z[rows[k] % T]
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                       f"logit_rows_{cfg['name']}.npz")
    np.savez_compressed(out, rows=np.array(rows, np.int64), vals=vals,
                        oracle_seconds=np.float64(time.time() - t0))
    print(f"{cfg['name']}: {len(rows)} logit rows in {time.time() - t0:.1f}s -> {out}", flush=True)


if __name__ == "__main__":
    args = sys.argv[1:]
    if args and args[0] == "--rows":
        for nm in args[1:]:
            logit_rows(nm)
    else:
        for nm in args:
            golden(nm)
