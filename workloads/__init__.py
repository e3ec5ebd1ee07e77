"""Seeded synthetic inputs for content-routed sparse attention.

This package draws random numbers and rounds them to the storage dtype; it
holds none of the method's arithmetic.  Both the CUDA path and the CPU oracle
consume exactly the arrays these functions return (the oracle reads host
copies).
"""
from .gen import (  # noqa: F401
    CONFIGS,
    lsh_fp32_case,
    lsh_clustered_case,
    indexer_prefill_case,
    indexer_decode_case,
    block_decode_case,
    query_subspace,
    make_config,
)
