"""Seeded synthetic inputs and named workload configurations.

This package holds no arithmetic of the method: only random draws (token ids,
initial weights) and the configuration tables.  Both the oracle tests and the
CUDA-path tests/benchmark take their inputs from here.
"""
from .configs import CONFIGS, get_config  # noqa: F401
from .inputs import make_batch, make_params, zipf_tokens  # noqa: F401
