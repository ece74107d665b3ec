"""fp64 CPU oracle for TT-embedding gather -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  It shares no code with the CUDA path.
"""
from .oracle import (OracleError, backward, default_threads, digits, forward, row, segmentation,
                     sgd, workload_backward, workload_forward, workload_segmentation)

__all__ = ["OracleError", "backward", "default_threads", "digits", "forward", "row",
           "segmentation", "sgd", "workload_backward", "workload_forward",
           "workload_segmentation"]
