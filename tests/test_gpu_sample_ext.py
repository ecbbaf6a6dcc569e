"""GPU parity of llm_sample_ex (repetition penalty, temperature, top-k,
top-p) against the oracle sampler on the same float32 logits.  With top_p = 1
and no penalty it returns llm_sample's ids; penalised greedy ids are exact
(both sides penalise in float32); a top-p draw must lie in the oracle's
nucleus and on its float64 cumulative-weight interval within the kernel's
float32 bound, on rows whose nucleus cut is not within 5e-5 of a boundary
(the kernel's float32 walk over at most 1024 weights);
20k draws follow the renormalised nucleus distribution."""
import ctypes as C

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _model(V):
    from scratch_llama_decoder_b200 import LlamaStep
    from synth import get_config
    return LlamaStep(get_config("c3", vocab=V, batch=1, ctx=8, n_layer=0))


def _t(a, dtype=torch.float32):
    return torch.tensor(a, dtype=dtype, device="cuda")


@pytest.mark.parametrize("V", [500, 32000])
def test_defaults_give_llm_sample_ids(V):
    m = _model(V)
    rng = np.random.default_rng(V + 1)
    z = _t((rng.standard_normal((48, V)) * 2).astype(np.float32))
    u = _t(rng.random(48).astype(np.float32))
    for temp, k in [(0.0, 0), (0.8, 40), (1.0, 0), (1.2, 7)]:
        a = m.sample(z, temp, k, u).cpu()
        b = m.sample_ex(z, temp, k, u).cpu()
        assert torch.equal(a, b), (temp, k)
    m.close()


@pytest.mark.parametrize("V", [27, 500, 32000])
def test_top_p_matches_oracle(V):
    from oracle import decode as OD
    m = _model(V)
    rng = np.random.default_rng(V + 2)
    R = 64
    z = (rng.standard_normal((R, V)) * 2).astype(np.float32)
    u = rng.random(R).astype(np.float32)
    checked = total = 0
    for temp, k, tp in [(0.8, 40, 0.9), (1.0, 5, 0.5), (1.3, 1024, 0.95), (0.7, 3, 0.99)]:
        got = m.sample_ex(_t(z), temp, k, _t(u), top_p=tp).cpu().numpy()
        again = m.sample_ex(_t(z), temp, k, _t(u), top_p=tp).cpu().numpy()
        np.testing.assert_array_equal(got, again)
        for r in range(R):
            total += 1
            S, Cw = OD.nucleus(z[r], temp, k, tp)
            if np.min(np.abs(Cw - tp * Cw[-1])) <= 5e-5 * Cw[-1]:
                continue  # the cut sits on a rounding boundary: either side is right
            checked += 1
            g = int(got[r])
            assert g in set(S.tolist()), (temp, k, tp, r, g)
            zf = z[r].astype(np.float64)
            C = np.cumsum(np.exp((zf[S] - zf.max()) / temp))
            i = int(np.searchsorted(S, g))
            lo = C[i - 1] if i > 0 else 0.0
            tol = (S.size + 1030) * 2.0 ** -23 * C[-1]
            target = float(u[r]) * C[-1]
            assert lo - tol <= target <= C[i] + tol, (r, g, lo, C[i], target)
    assert checked >= 0.8 * total
    m.close()


def test_repetition_penalty_matches_oracle():
    from oracle import decode as OD
    V, R, Hn = 500, 64, 24
    m = _model(V)
    rng = np.random.default_rng(7)
    z = (rng.standard_normal((R, V)) * 2).astype(np.float32)
    hist = rng.integers(-3, V + 3, size=(R, Hn)).astype(np.int32)  # some ids out of range
    # make the penalty matter: each row's argmax is in its history
    for r in range(R):
        hist[r, 0] = int(np.argmax(z[r]))
    for pen in (1.3, 0.8):
        got = m.sample_ex(_t(z), 0.0, 0, _t(np.zeros(R, np.float32)), penalty=pen,
                          history=_t(hist, torch.int32)).cpu().numpy()
        want = [OD.sample(z[r], 0.0, 0, 0.0, penalty=pen, history=hist[r]) for r in range(R)]
        np.testing.assert_array_equal(got, want)
    # with temperature and top-k: a valid draw from the penalised logits
    u = rng.random(R).astype(np.float32)
    got = m.sample_ex(_t(z), 0.9, 20, _t(u), penalty=1.3,
                      history=_t(hist, torch.int32)).cpu().numpy()
    for r in range(R):
        pz = OD.penalise(z[r], 1.3, hist[r])
        S, Cw, W = OD.sample_cdf(pz, 0.9, 20)
        g = int(got[r])
        assert g in set(S.tolist())
        i = int(np.searchsorted(S, g))
        lo = Cw[i - 1] if i > 0 else 0.0
        tol = (S.size + 1030) * 2.0 ** -23 * W
        assert lo - tol <= float(u[r]) * W <= Cw[i] + tol
    m.close()


def test_top_p_frequencies_over_20k_draws():
    from oracle import decode as OD
    V, n, temp, k, tp = 12, 20000, 0.9, 8, 0.8
    m = _model(V)
    rng = np.random.default_rng(21)
    z = (rng.standard_normal(V) * 1.5).astype(np.float32)
    S, _ = OD.nucleus(z, temp, k, tp)
    draws = m.sample_ex(_t(np.tile(z, (n, 1))), temp, k, _t(rng.random(n).astype(np.float32)),
                        top_p=tp).cpu().numpy()
    p = np.zeros(V)
    p[S] = np.exp(z[S].astype(np.float64) / temp)
    p /= p.sum()
    freq = np.bincount(draws, minlength=V) / n
    assert set(np.unique(draws).tolist()) <= set(S.tolist())
    assert np.all(np.abs(freq - p) <= 4.5 * np.sqrt(p * (1 - p) / n) + 1e-12), (freq, p)
    m.close()


def test_sample_ex_arguments():
    import scratch_llama_decoder_b200 as L
    m = _model(500)
    z = _t(np.zeros((2, 500), np.float32))
    u = _t(np.zeros(2, np.float32))
    o = torch.empty(2, dtype=torch.int32, device="cuda")
    h = _t(np.zeros((2, 4), np.int32), torch.int32)
    call = lambda temp, k, tp, pen, hp, hld, hl: L.lib.llm_sample_ex(
        m.ctx, z.data_ptr(), 500, 2, temp, k, tp, pen, hp, hld, hl, u.data_ptr(), o.data_ptr())
    assert call(1.0, 40, 0.0, 1.0, None, 0, 0) == L.LLM_ERR_ARG        # top_p <= 0
    assert call(1.0, 40, 1.5, 1.0, None, 0, 0) == L.LLM_ERR_ARG        # top_p > 1
    assert call(1.0, 0, 0.9, 1.0, None, 0, 0) == L.LLM_ERR_ARG         # top-p needs a top-k
    assert call(1.0, 2000, 0.9, 1.0, None, 0, 0) == L.LLM_ERR_ARG      # top-k past the sort
    assert call(1.0, 40, 1.0, 0.0, None, 0, 0) == L.LLM_ERR_ARG        # penalty <= 0
    assert call(1.0, 40, 1.0, 1.2, None, 4, 4) == L.LLM_ERR_ARG        # penalty without history
    assert call(1.0, 40, 1.0, 1.2, h.data_ptr(), 2, 4) == L.LLM_ERR_ARG  # history stride too short
    assert call(1.0, 40, 0.9, 1.2, h.data_ptr(), 4, 4) == 0
    m.close()
