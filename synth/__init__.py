"""Seeded synthetic decode-step workloads (shared by tests and the benchmark).

This package holds input generation only: shapes, value distributions, page
placement (block tables), prefix sharing and canary filling.  It contains none
of the attention arithmetic, and neither the CUDA library nor the oracle is
imported here.
"""
from .workloads import (  # noqa: F401
    CANARY_WORD,
    PAGE_TOKENS,
    Workload,
    build_workload,
    config_spec,
    named_config,
    NAMED_CONFIGS,
    step_inputs,
    to_words,
)
from .allocator import BlockAllocator  # noqa: F401
