"""fp64 CPU oracle for gated linear attention and gated slot attention (test infrastructure only).

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may
import this package. The CUDA product path never calls it and shares no code
with it. See ``gla_oracle.c`` and ``gsa_oracle.c`` for the recurrences and their source passages.
"""
from .oracle import (  # noqa: F401
    build,
    fwd,
    bwd,
    step,
    gsa_fwd,
    gsa_bwd,
    num_threads,
    set_threads,
)
