"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

Holds no arithmetic of the Engram method: token streams, sequence bounds,
configuration constants, tables and output gradients only.
"""

from . import constants
from .generate import (DTYPE_BYTES, DTYPE_CODES, WORKLOADS, Workload,
                       fill_device_table, head_params, host_dout, host_table,
                       random_stream, token_stream)

__all__ = [
    "constants", "DTYPE_BYTES", "DTYPE_CODES", "WORKLOADS", "Workload",
    "fill_device_table", "head_params", "host_dout", "host_table",
    "random_stream", "token_stream",
]
