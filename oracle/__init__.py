"""fp64 CPU oracle for DeltaLog recurrent-state decode.

Test infrastructure only: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  Nothing here is shared
with, or called by, the CUDA path.
"""
from .oracle import (  # noqa: F401
    GDN, KDA, RWKV6, OP_NAMES, LogState, build, decay_width, eager_run,
    deltalog_run, deltalog_slots_run, materialize, merge, max_threads, rel_err,
)
