"""Pins of the float64 learning-rate schedule and gradient clipping
(oracle/train_terms.py): the schedule's endpoints and midpoints (strata,
optimiser row: schedule endpoints), PyTorch's cosine-annealing and linear
schedulers on the decay phase, randyGPT's printed 1e-4 -> 1e-5 schedule, and
clipping against a closed form and torch.nn.utils.clip_grad_norm_.
"""
import math

import numpy as np
import pytest
import torch

from oracle import train_terms as TT


def test_schedule_endpoints_and_midpoints():
    mx, mn, W, T = 3e-4, 3e-5, 100, 1100
    assert TT.lr_at(1, mx, mn, W, W, T) == pytest.approx(mx / W, rel=1e-15)
    assert TT.lr_at(50, mx, mn, W, W, T) == pytest.approx(mx / 2, rel=1e-15)
    assert TT.lr_at(W, mx, mn, W, W, T) == mx
    assert TT.lr_at(T, mx, mn, W, W, T) == pytest.approx(mn, rel=1e-12)
    assert TT.lr_at(T + 500, mx, mn, W, W, T) == pytest.approx(mn, rel=1e-12)
    assert TT.lr_at(W + (T - W) // 2, mx, mn, W, W, T) == pytest.approx((mx + mn) / 2, rel=1e-12)
    # linear decay: a straight line from max to min
    assert TT.lr_at(W + (T - W) // 4, mx, mn, W, W, T, "linear") == \
        pytest.approx(mx + (mn - mx) / 4, rel=1e-12)
    # constant: max after warm-up, whatever the decay settings
    assert TT.lr_at(T, mx, mn, W, W, T, "constant") == mx
    # non-increasing after the warm-up, non-decreasing before it
    lrs = [TT.lr_at(t, mx, mn, W, W, T) for t in range(1, T + 1)]
    assert all(a <= b for a, b in zip(lrs[:W - 1], lrs[1:W]))
    assert all(a >= b for a, b in zip(lrs[W - 1:-1], lrs[W:]))


def test_randygpt_schedule():
    """randyGPT: constant 1e-4, then cosine to 1e-5 over the final 40%."""
    T = 1000
    f = lambda t: TT.lr_at(t, 1e-4, 1e-5, 0, 600, T)
    assert f(1) == 1e-4 and f(600) == 1e-4
    assert f(800) == pytest.approx(5.5e-5, rel=1e-12)
    assert f(1000) == pytest.approx(1e-5, rel=1e-12)
    assert f(601) < 1e-4


@pytest.mark.parametrize("shape", ["cosine", "linear"])
def test_decay_phase_against_torch_schedulers(shape):
    mx, mn, W, T = 1e-3, 1e-4, 20, 220
    p = torch.nn.Parameter(torch.zeros(1, dtype=torch.float64))
    opt = torch.optim.SGD([p], lr=mx)
    if shape == "cosine":
        sch = torch.optim.lr_scheduler.CosineAnnealingLR(opt, T_max=T - W, eta_min=mn)
    else:
        sch = torch.optim.lr_scheduler.LinearLR(opt, start_factor=1.0, end_factor=mn / mx,
                                                total_iters=T - W)
    for e in range(T - W + 1):
        assert TT.lr_at(W + e, mx, mn, W, W, T, shape) == \
            pytest.approx(opt.param_groups[0]["lr"], rel=1e-10, abs=1e-15), e
        opt.step()
        sch.step()


def test_clip_closed_form_and_threshold():
    g, n, s = TT.clip([3.0, 4.0], 1.0)
    assert n == 5.0 and s == pytest.approx(0.2, rel=1e-15)
    np.testing.assert_allclose(g, [0.6, 0.8], rtol=1e-15)
    g, n, s = TT.clip([0.3, 0.4], 1.0)  # norm 0.5 under the threshold: untouched
    assert s == 1.0
    np.testing.assert_array_equal(g, [0.3, 0.4])
    rng = np.random.default_rng(3)
    x = rng.standard_normal(1000)
    c, n, s = TT.clip(x, 2.0)
    assert np.linalg.norm(c) == pytest.approx(2.0, rel=1e-13)
    assert n == pytest.approx(np.sqrt(1000), rel=0.1)


def test_clip_against_torch_clip_grad_norm():
    """torch scales by max_norm / (norm + 1e-6): equal to the pages' formula up
    to that epsilon."""
    rng = np.random.default_rng(4)
    g = rng.standard_normal(5000) * 0.3
    ps = [torch.nn.Parameter(torch.zeros(2500, dtype=torch.float64)) for _ in range(2)]
    ps[0].grad = torch.tensor(g[:2500])
    ps[1].grad = torch.tensor(g[2500:])
    for max_norm in (0.5, 100.0):
        for i in range(2):
            ps[i].grad = torch.tensor(g[2500 * i:2500 * (i + 1)])
        total = torch.nn.utils.clip_grad_norm_(ps, max_norm)
        c, n, s = TT.clip(g, max_norm)
        assert float(total) == pytest.approx(n, rel=1e-12)
        got = np.concatenate([p.grad.numpy() for p in ps])
        np.testing.assert_allclose(got, c, rtol=1e-6 / max(n, 1e-30) * 10, atol=0)
        assert math.isclose(s, 1.0) == (n <= max_norm)


def test_plateau_against_torch_reduce_lr_on_plateau():
    """randyGPT's schedule: halve on stagnation (patience 30), at most 3 times;
    PyTorch's ReduceLROnPlateau (mode min, rel threshold 0, cooldown 0) with
    min_lr = lr * 0.5^3 gives the same rates."""
    rng = np.random.default_rng(9)
    losses = np.concatenate([np.linspace(5, 3, 40), 3 + 0.01 * rng.random(200),
                             np.linspace(2.9, 2.5, 20), 2.6 + 0.01 * rng.random(150)])
    pl = TT.Plateau(0.5, 30, 3, 0.0)
    p = torch.nn.Parameter(torch.zeros(1, dtype=torch.float64))
    opt = torch.optim.SGD([p], lr=1.0)
    sch = torch.optim.lr_scheduler.ReduceLROnPlateau(opt, mode="min", factor=0.5, patience=30,
                                                     threshold=0.0, threshold_mode="rel",
                                                     cooldown=0, min_lr=0.125, eps=0.0)
    scales = []
    for v in losses:
        scales.append(pl.update(float(v)))
        sch.step(float(v))
        assert scales[-1] == pytest.approx(opt.param_groups[0]["lr"], rel=1e-15)
    assert pl.reductions == 3 and scales[-1] == 0.125
    # the first reduction comes on the 31st evaluation without a better one
    first = next(i for i, x in enumerate(scales) if x < 1.0)
    best_i = int(np.argmin(losses[:first]))
    assert first - best_i == 31


def test_linf_clip_closed_form_and_torch():
    g, n, sc = TT.clip([3.0, -4.0, 0.5], 1.0, "linf")
    assert n == 4.0 and sc == 0.25
    np.testing.assert_allclose(g, [0.75, -1.0, 0.125], rtol=1e-15)
    g, n, sc = TT.clip([0.3, -0.4], 1.0, "linf")
    assert sc == 1.0 and n == 0.4
    rng = np.random.default_rng(5)
    x = rng.standard_normal(3000)
    pt = torch.nn.Parameter(torch.zeros(3000, dtype=torch.float64))
    pt.grad = torch.tensor(x)
    total = torch.nn.utils.clip_grad_norm_([pt], 1.5, norm_type=float("inf"))
    c, n, sc = TT.clip(x, 1.5, "linf")
    assert float(total) == n  # the largest |g|, exactly
    np.testing.assert_allclose(pt.grad.numpy(), c, rtol=1e-5)
    assert np.abs(c).max() == pytest.approx(1.5, rel=1e-15)


def test_nan_gradient_leaves_the_scale_at_one():
    """A NaN gradient makes either norm NaN; NaN > max_norm is false, so the
    clipping rule leaves the gradient unscaled (the step's non-finite-loss
    check is what stops such an update)."""
    for kind in ("l2", "linf"):
        n = TT.grad_norm([1.0, float("nan"), -3.0], kind)
        assert math.isnan(n)
        assert TT.clip_scale(n, 1.0) == 1.0
