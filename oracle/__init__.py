"""CPU oracle for the pi0.5-style action-expert denoise loop (test infrastructure).

This package is the plain, slow, float64 definition that the CUDA library is
checked against.  It is test infrastructure only: the tests, the smoke check
and the benchmark's CPU-baseline leg may call it; the product path never
does, and it shares no code with the CUDA library.

Parity is unpinned only for agreement with a real trained pi0.5 policy (no
checkpoint, VLM or dataset exists here); every arithmetic step is pinned by
the tests under ``tests/test_oracle_*.py``.
"""
from .expert import (  # noqa: F401
    sinusoidal_embedding, swish, time_conditioning, modulation_tables,
    ada_rms_norm, gelu_tanh, attention, expert_layer, velocity, denoise,
    denoise_row, brute_force_denoise_row, prefix_stack_kv, prefix_stack_hidden,
    prefix_kv_from_hidden, rope, OracleParams,
    params_from_weights,
)
