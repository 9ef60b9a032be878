"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

Holds no arithmetic of the Engram method: token streams, sequence bounds,
configuration constants, tables, output gradients and the PLE tail's random
activations and weights only.
"""

from . import constants
from .generate import (DTYPE_BYTES, DTYPE_CODES, PLE_SHAPES, WORKLOADS, PleShape, Workload,
                       fill_device_table, head_params, host_dout, host_table, ple_inputs,
                       random_stream, row_bounds, token_stream)

__all__ = [
    "constants", "DTYPE_BYTES", "DTYPE_CODES", "PLE_SHAPES", "WORKLOADS", "PleShape",
    "Workload", "fill_device_table", "head_params", "host_dout", "host_table", "ple_inputs",
    "random_stream", "row_bounds", "token_stream",
]
