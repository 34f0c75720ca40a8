"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This package draws random numbers and nothing else: it holds none of the replay
method's arithmetic (no decay scan, no output route, no flush), so that a mistake in
the method cannot hide in code that both the CUDA path and the oracle use.
"""

from .gen import (  # noqa: F401
    Shape,
    SHAPES,
    sweep_shapes,
    head_decay_rates,
    step_inputs,
    verify_inputs,
    initial_state,
    accepted_lengths,
    to_numpy64,
)
