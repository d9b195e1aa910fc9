"""CPU oracle for the Gemma 3 5:1 block attention (test infrastructure only).

This package is the slow, plain reference that the CUDA path is checked
against.  It is NOT part of the product: only the tests, the entry point's
smoke check and the benchmark's CPU-baseline leg may import it.  It shares no
code with the CUDA library and never imports it.

Everything is numpy float64 on the exact bf16 input values.
"""
from .attention import (  # noqa: F401
    EPS,
    LOCAL,
    GLOBAL,
    qk_rmsnorm,
    inv_frequencies,
    rope,
    allowed,
    allowed_row,
    prefill,
    prefill_rows,
    prefill_bruteforce,
    decode,
    unmasked_pairs,
)
from .projector import soft_tokens  # noqa: F401,E402
from .backward import prefill_backward, rope_backward, rmsnorm_backward  # noqa: F401,E402
