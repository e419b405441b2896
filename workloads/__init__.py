"""Seeded synthetic inputs for the MoE token shuffle.

This package only draws inputs: routing (top-k expert ids and their weights) and
payload tensors.  It holds none of the shuffle's arithmetic (no histogram, scan,
slot assignment, copy or reduction), so both the CPU oracle and the CUDA library
can be fed from it without sharing any code with each other.
"""

from .gen import (  # noqa: F401
    CONFIGS,
    Config,
    Workload,
    ZIPF_ALPHA,
    distinct_rank_expectation,
    drop_entries,
    find_zipf_alpha,
    make_payload_x,
    make_expert_outputs,
    make_payload_y,
    make_routing,
    make_workload,
    rank_load_ratio,
)
