"""Seeded synthetic inputs for the lightning-indexer workloads.

This package holds random draws only: it contains none of the indexer's
arithmetic (no scoring, no selection, no group averaging).  Both the CUDA
path and the CPU oracle receive the tensors it produces.
"""
from .workloads import (  # noqa: F401
    CONFIGS,
    DenseInputs,
    DecodeInputs,
    make_dense_inputs,
    make_decode_inputs,
    encode_e4m3,
)
