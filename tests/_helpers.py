"""Host-side helpers of the GPU parity tests (no GPU kernels of the library).

The expected rows of a lookup are the input table's rows at the oracle's
indices. A table that lives only on the device (the 320,001,536-row one does
not fit the host) is brought to the host in contiguous chunks by plain
device-to-host copies, and the needed rows are picked there, so no GPU gather
produces an expected value.
"""

import numpy as np
import torch

import oracle


def table_rows_to_host(table: torch.Tensor, rows_sorted: np.ndarray,
                       chunk_rows: int = 1 << 22) -> np.ndarray:
    """table[rows_sorted] on the host (rows_sorted ascending, distinct): int16
    bit patterns for 16-bit tables, float32 otherwise. Chunks holding none of
    the rows are skipped."""
    R, D = table.shape
    is16 = table.element_size() == 2
    out = np.empty((len(rows_sorted), D), dtype=np.int16 if is16 else np.float32)
    for a in range(0, R, chunk_rows):
        b = min(R, a + chunk_rows)
        i0 = int(np.searchsorted(rows_sorted, a))
        i1 = int(np.searchsorted(rows_sorted, b))
        if i1 == i0:
            continue
        blk = table[a:b].cpu()                         # one contiguous copy
        blk_np = blk.view(torch.int16).numpy() if is16 else blk.numpy()
        out[i0:i1] = blk_np[rows_sorted[i0:i1] - a]
    return out


def expected_rows(idx_rows: np.ndarray, table: torch.Tensor) -> np.ndarray:
    """oracle.gather of the table rows the flat index array names, as raw
    element bits (int16 for 16-bit tables, float32 otherwise)."""
    uniq, inv = np.unique(idx_rows.reshape(-1), return_inverse=True)
    compact = table_rows_to_host(table, uniq.astype(np.int64))
    return oracle.gather(compact, inv.reshape(-1))


def raw_bits(t: torch.Tensor) -> np.ndarray:
    """A device or host tensor's elements as int16 bits (16-bit) or float32."""
    t = t.contiguous().cpu()
    return t.view(torch.int16).numpy() if t.element_size() == 2 else t.numpy()
