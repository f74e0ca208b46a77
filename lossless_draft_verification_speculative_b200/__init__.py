"""DSpark block-draft verify/accept on B200 (sm_100a).

``greedy_accept`` and ``speculative_sample_accept`` verify a block of K drafted tokens per
sequence against the base model's [B, K+1, V] logit block and return an ``AcceptResult``;
``mixed_accept`` verifies a serving batch whose sequences have their own draft counts and
temperatures; ``early_exit_accept`` reads each sequence's rows only up to its first
rejection; ``markov_matvec`` is the drafter's Markov-head table mat-vec; ``YieldQuench`` is
the host-side policy that turns speculation off for requests whose acceptance does not pay
for the verify (``include/dspark_policy.h``).
The work runs in hand-written CUDA kernels behind a C ABI (``include/dspark_verify.h``);
this package is the thin Python binding over it plus the seeded synthetic workloads.
"""

from .binding import (  # noqa: F401
    SEQ_BAD_DRAFT,
    SEQ_BAD_PARAM,
    SEQ_NONFINITE,
    SEQ_TIMEOUT,
    SEQ_ZERO_RESIDUAL,
    AcceptResult,
    YieldQuench,
    DsparkError,
    early_exit_accept,
    greedy_accept,
    load_library,
    markov_matvec,
    mixed_accept,
    pipeline_timeouts,
    plan,
    speculative_sample_accept,
    speculative_sample_accept_static,
    workspace_bytes,
)

__all__ = [
    "AcceptResult",
    "DsparkError",
    "YieldQuench",
    "greedy_accept",
    "speculative_sample_accept",
    "speculative_sample_accept_static",
    "mixed_accept",
    "early_exit_accept",
    "markov_matvec",
    "pipeline_timeouts",
    "load_library",
    "plan",
    "workspace_bytes",
    "SEQ_BAD_DRAFT",
    "SEQ_NONFINITE",
    "SEQ_ZERO_RESIDUAL",
    "SEQ_TIMEOUT",
    "SEQ_BAD_PARAM",
]
