"""B200-native Engram N-gram Embedding: hash, gather, compact backward, the
sparse optimizer step on the touched rows, and the PLE layer's grouped RMS
norm and causal short convolution with its backward.

Python face of the C ABI in include/engram.h (libengram_b200.so, sm_100a).
Every step runs in the library's CUDA kernels; this package only marshals
arguments and allocates buffers with torch. Importing it fails if the library
has not been built (`python hashed_gram_embedding_raw_b200/build.py`).
"""

from ._binding import (ENGRAM_BF16, ENGRAM_CONV_NORM, ENGRAM_CONV_RESIDUAL, ENGRAM_CONV_SILU,
                       ENGRAM_DEVERR_CAPACITY, ENGRAM_DEVERR_COPY_TIMEOUT,
                       ENGRAM_DEVERR_CU_SEQLENS,
                       ENGRAM_DEVERR_ROW_RANGE, ENGRAM_DEVERR_SORT_TIMEOUT,
                       ENGRAM_EINVAL, ENGRAM_ECUDA, ENGRAM_ENOSPC, ENGRAM_F16, ENGRAM_F32,
                       ENGRAM_NOALLOC_SCRATCH_BYTES, ENGRAM_OK, EXPORTED, LIB_PATH,
                       AdamParams, ConvParams, EngramError, EngramParams, engram_abi_version,
                       engram_backward, engram_backward_heads,
                       engram_backward_noalloc, engram_backward_reduce, engram_backward_sort,
                       engram_backward_sort_heads,
                       engram_backward_workspace_size, engram_gather, engram_get_device_error,
                       engram_grouped_rms_norm, engram_hash, engram_hash_gather,
                       engram_hash_gather_slice, engram_host_floor_mod, engram_ple_short_conv,
                       engram_ple_short_conv_backward,
                       engram_ple_short_conv_backward_workspace_size, engram_sparse_adam,
                       engram_owner_bucket, engram_owner_bucket_padded,
                       engram_owner_bucket_workspace_size,
                       engram_launch_count, lib, make_params, status_string)

__all__ = [
    "ENGRAM_BF16", "ENGRAM_CONV_NORM", "ENGRAM_CONV_RESIDUAL", "ENGRAM_CONV_SILU",
    "ENGRAM_DEVERR_CAPACITY", "ENGRAM_DEVERR_COPY_TIMEOUT", "ENGRAM_DEVERR_CU_SEQLENS",
    "ENGRAM_DEVERR_ROW_RANGE",
    "ENGRAM_DEVERR_SORT_TIMEOUT", "ENGRAM_EINVAL",
    "ENGRAM_ECUDA", "ENGRAM_ENOSPC", "ENGRAM_F16", "ENGRAM_F32",
    "ENGRAM_NOALLOC_SCRATCH_BYTES", "ENGRAM_OK", "EXPORTED", "LIB_PATH", "AdamParams", "ConvParams",
    "EngramError", "EngramParams", "engram_abi_version", "engram_backward",
    "engram_backward_heads", "engram_backward_noalloc",
    "engram_backward_reduce", "engram_backward_sort", "engram_backward_sort_heads",
    "engram_backward_workspace_size",
    "engram_gather", "engram_get_device_error", "engram_hash", "engram_hash_gather",
    "engram_hash_gather_slice", "engram_grouped_rms_norm", "engram_ple_short_conv",
    "engram_ple_short_conv_backward", "engram_ple_short_conv_backward_workspace_size",
    "engram_sparse_adam", "engram_owner_bucket", "engram_owner_bucket_padded",
    "engram_owner_bucket_workspace_size",
    "engram_host_floor_mod", "engram_launch_count", "lib", "make_params", "status_string",
]
