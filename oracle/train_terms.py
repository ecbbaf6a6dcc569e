"""Float64 training-loop terms around the step: the learning-rate schedule and
global-norm gradient clipping.

TEST INFRASTRUCTURE ONLY: imported by the tests, never by the product library.

Schedule (Transformer-In-Rust, Features: cosine decay with linear warmup, and
its test list: cosine / linear / constant schedulers; randyGPT, Training:
constant at max_lr, then cosine decay to min_lr over the final 40%; strata,
optimiser row: cosine + warmup, pinned at its endpoints).  One shape covers
all three, with 1-based step t:
  t <= warmup (warmup > 0):      lr = max_lr * t / warmup
  t <= decay_start:              lr = max_lr
  otherwise, p = min(1, (t - decay_start) / (total - decay_start)):
    cosine:   lr = min_lr + (max_lr - min_lr) * (1 + cos(pi p)) / 2
    linear:   lr = max_lr + (min_lr - max_lr) * p
    constant: lr = max_lr
with decay_start >= warmup (Transformer-In-Rust's schedule: decay_start =
warmup; randyGPT's: warmup 0, decay_start = 0.6 total) and p = 1 whenever
total <= decay_start.

Clipping (MicroGPT in Rust, Gradient Clipping: when the gradient norm exceeds
max_norm every gradient is scaled by max_norm / norm, else left alone;
Transformer-In-Rust: by global norm).  The norm is the Euclidean norm of all
gradient elements together; randyGPT's "L-infinity norm clipped at 1.0" is
the same rule with the largest absolute gradient element as the norm.

Plateau (randyGPT, Training: ReduceLROnPlateau halves max_lr on stagnation, up
to 3 times, patience 30).  Readings: a metric counts as better when it is
below best * (1 - threshold) (threshold 0: strictly below); after more than
`patience` evaluations in a row without a better one the scale is multiplied
by `factor` (at most `max_reductions` times) and the count restarts.
"""
import math

import numpy as np

SHAPES = {"constant": 0, "cosine": 1, "linear": 2}


def lr_at(t, max_lr, min_lr, warmup, decay_start, total, shape="cosine"):
    """Learning rate of 1-based step t."""
    if warmup > 0 and t <= warmup:
        return max_lr * t / warmup
    if t <= decay_start or shape == "constant":
        return max_lr
    p = 1.0 if total <= decay_start else min(1.0, (t - decay_start) / (total - decay_start))
    if shape == "cosine":
        return min_lr + (max_lr - min_lr) * (1.0 + math.cos(math.pi * p)) / 2.0
    return max_lr + (min_lr - max_lr) * p


def grad_norm(g, kind="l2"):
    """Euclidean norm of every gradient element together ("l2"), or the
    largest absolute element ("linf")."""
    g = np.asarray(g, dtype=np.float64)
    if kind == "linf":
        return float(np.max(np.abs(g))) if g.size else 0.0
    return float(np.sqrt(np.sum(g * g)))


def clip_scale(norm, max_norm):
    return max_norm / norm if norm > max_norm else 1.0


def clip(g, max_norm, kind="l2"):
    """(clipped gradient, norm before clipping, scale)."""
    n = grad_norm(g, kind)
    s = clip_scale(n, max_norm)
    return np.asarray(g, dtype=np.float64) * s, n, s


class Plateau:
    """Learning-rate scale after each evaluation (starts at 1)."""

    def __init__(self, factor=0.5, patience=30, max_reductions=3, threshold=0.0):
        self.factor, self.patience = factor, patience
        self.max_reductions, self.threshold = max_reductions, threshold
        self.best, self.bad, self.reductions, self.scale = math.inf, 0, 0, 1.0

    def update(self, metric):
        if metric < self.best * (1.0 - self.threshold):
            self.best, self.bad = metric, 0
        else:
            self.bad += 1
            if self.bad > self.patience and self.reductions < self.max_reductions:
                self.reductions += 1
                self.scale *= self.factor
                self.bad = 0
        return self.scale
