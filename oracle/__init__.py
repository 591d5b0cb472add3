"""fp64 CPU oracle for gated linear attention (test infrastructure only).

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may
import this package. The CUDA product path never calls it and shares no code
with it. See ``gla_oracle.c`` for the recurrence and its source passages.
"""
from .oracle import (  # noqa: F401
    build,
    fwd,
    bwd,
    step,
    num_threads,
    set_threads,
)
