"""Float64 CPU oracle of the Llama training step (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import
this package.  The product library never does.
"""
from .oracle import *  # noqa: F401,F403
