"""llm_lr_at and llm_plateau_* (host-only C ABI) against the oracle's
schedule and plateau rule: equal to within float32 rounding at every step,
and invalid arguments rejected.  Runs without a GPU (the library loads on the
host; the schedule launches nothing)."""
import ctypes as C

import numpy as np
import pytest

from oracle import train_terms as TT

SCHEDULES = [
    # max_lr, min_lr, warmup, decay_start, total, shape
    (3e-4, 3e-5, 100, 100, 1000, "cosine"),   # linear warm-up, then cosine
    (1e-4, 1e-5, 0, 600, 1000, "cosine"),     # randyGPT: hold, cosine over the final 40%
    (1e-3, 0.0, 10, 50, 300, "linear"),
    (2e-4, 1e-6, 7, 7, 7, "cosine"),          # total <= decay start: min_lr after warm-up
    (5e-4, 5e-5, 0, 0, 64, "constant"),
]


@pytest.mark.parametrize("sched", SCHEDULES)
def test_lr_at_matches_oracle(sched):
    import scratch_llama_decoder_b200 as P
    mx, mn, W, S, T, shape = sched
    for t in list(range(1, T + 40)):
        got = P.lr_at(t, mx, mn, W, S, T, shape)
        want = np.float32(TT.lr_at(t, float(np.float32(mx)), float(np.float32(mn)), W, S, T,
                                   shape))
        assert got == pytest.approx(float(want), rel=1.2e-7, abs=1e-30), (t, got, want)


def test_lr_at_rejects_bad_arguments():
    import scratch_llama_decoder_b200 as P
    from scratch_llama_decoder_b200._lib import llm_lr_schedule
    out = C.c_float(0.0)
    bad = [
        (llm_lr_schedule(1e-3, 1e-4, 10, 10, 100, 1), 0),       # t < 1
        (llm_lr_schedule(1e-3, 1e-4, -1, 10, 100, 1), 1),       # negative warm-up
        (llm_lr_schedule(1e-3, 1e-4, 10, 5, 100, 1), 1),        # decay before warm-up ends
        (llm_lr_schedule(1e-3, 1e-4, 10, 10, 100, 7), 1),       # unknown shape
        (llm_lr_schedule(float("nan"), 1e-4, 10, 10, 100, 1), 1),
    ]
    for sc, t in bad:
        assert P.lib.llm_lr_at(C.byref(sc), t, C.byref(out)) == P.LLM_ERR_ARG
    assert P.lib.llm_lr_at(None, 1, C.byref(out)) == P.LLM_ERR_ARG


def test_plateau_matches_oracle():
    import scratch_llama_decoder_b200 as P
    rng = np.random.default_rng(9)
    losses = np.concatenate([np.linspace(5, 3, 40), 3 + 0.01 * rng.random(200),
                             np.linspace(2.9, 2.5, 20), 2.6 + 0.01 * rng.random(150)])
    for args in ((0.5, 30, 3, 0.0), (0.3, 5, 10, 1e-3), (1.0, 0, 2, 0.0)):
        # the C ABI takes the factor as float32: the oracle gets that value
        a, b = P.Plateau(*args), TT.Plateau(float(np.float32(args[0])), *args[1:])
        for v in losses:
            assert a.update(v) == np.float32(b.update(float(v)))
    from scratch_llama_decoder_b200._lib import llm_plateau
    s = llm_plateau()
    for bad in ((0.0, 30, 3, 0.0), (1.5, 30, 3, 0.0), (0.5, -1, 3, 0.0), (0.5, 30, -1, 0.0),
                (0.5, 30, 3, 1.0)):
        assert P.lib.llm_plateau_init(C.byref(s), *bad) == P.LLM_ERR_ARG
    assert P.lib.llm_plateau_init(C.byref(s), 0.5, 30, 3, 0.0) == 0
    out = C.c_float()
    assert P.lib.llm_plateau_update(C.byref(s), float("nan"), C.byref(out)) == P.LLM_ERR_ARG
