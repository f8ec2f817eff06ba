"""Seeded synthetic inputs shared by the CUDA path's tests/benchmarks and the oracle.

This package draws random numbers and lays them out; it performs none of the KDA
method's arithmetic (no gate, no sigmoid, no recurrence, no convolution, no norm of
the front or back end). Both sides compute everything from these raw draws.
"""
from .inputs import (  # noqa: F401
    CoreInputs, BlockWeights, DecodeInputs,
    core_inputs, block_weights, block_hidden, decode_inputs, t_pad, pad_rows,
)
