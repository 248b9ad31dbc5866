"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle.

This package holds no arithmetic of the training step itself: only the
workload shapes, the Zipf(s=1.1) token streams that stand in for the web-text
token shards the pages train on, and the N(0, 0.02) initial weights.  Both the
CUDA path and the CPU oracle consume the arrays produced here.
"""

from .workloads import WORKLOADS, workload, small_case  # noqa: F401
from .streams import (  # noqa: F401
    zipf_stream,
    tokens_and_targets,
    repeated_spans,
    init_params,
    round_to_bf16,
    param_shapes,
)
