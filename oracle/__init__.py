"""CPU float64 oracle of the DSpark block verify/accept step (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and reference
arm may import this package. It shares no code with the CUDA path.
"""

from .accept_ref import (  # noqa: F401
    STATUS_BAD_DRAFT,
    STATUS_BAD_PARAM,
    STATUS_NONFINITE,
    STATUS_ZERO_RESIDUAL,
    OracleResult,
    cdf_interval,
    draw_law,
    early_exit_accept,
    greedy_accept,
    inverse_cdf,
    mixed_accept,
    row_argmax,
    softmax,
    speculative_sample_accept,
)
