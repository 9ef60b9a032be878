"""ctypes binding of libengram_b200.so (include/engram.h).

Argument marshalling only: every function checks tensor devices, dtypes and
shapes, allocates outputs with torch when the caller passes none, and hands
raw pointers plus the current CUDA stream to the C ABI. All computation runs
in the library's sm_100a kernels; there is no fallback path. Importing this
module fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libengram_b200.so")

ENGRAM_OK, ENGRAM_EINVAL, ENGRAM_ENOSPC, ENGRAM_ECUDA = 0, 1, 2, 3
ENGRAM_F32, ENGRAM_BF16, ENGRAM_F16 = 0, 1, 2
ENGRAM_DEVERR_ROW_RANGE, ENGRAM_DEVERR_CU_SEQLENS, ENGRAM_DEVERR_SORT_TIMEOUT = 1, 2, 4
ENGRAM_DEVERR_COPY_TIMEOUT, ENGRAM_DEVERR_CAPACITY = 8, 16
ENGRAM_CONV_NORM, ENGRAM_CONV_SILU, ENGRAM_CONV_RESIDUAL = 1, 2, 4
ENGRAM_MAX_NGRAM, ENGRAM_MAX_HEADS = 4, 32

_DTYPE_CODE = {torch.float32: ENGRAM_F32, torch.bfloat16: ENGRAM_BF16,
               torch.float16: ENGRAM_F16}

EXPORTED = (
    "engram_hash", "engram_gather", "engram_hash_gather",
    "engram_backward_workspace_size", "engram_backward", "engram_backward_sort",
    "engram_backward_reduce", "engram_get_device_error", "engram_status_string",
    "engram_abi_version", "engram_params_size", "engram_launch_count",
    "engram_host_floor_mod", "engram_backward_noalloc", "engram_hash_gather_slice",
    "engram_ple_short_conv", "engram_grouped_rms_norm", "engram_sparse_adam",
    "engram_ple_short_conv_backward", "engram_ple_short_conv_backward_workspace_size",
    "engram_owner_bucket", "engram_owner_bucket_workspace_size",
    "engram_backward_heads", "engram_backward_sort_heads", "engram_owner_bucket_padded",
    "engram_ple_short_conv_save", "engram_ple_short_conv_backward_saved",
)

ENGRAM_NOALLOC_SCRATCH_BYTES = 32 << 20


class EngramError(RuntimeError):
    """A C-ABI call returned a non-zero status."""

    def __init__(self, what: str, status: int):
        super().__init__(f"{what}: {status_string(status)}")
        self.status = status


class EngramParams(ctypes.Structure):
    """Mirror of engram_params_t."""
    _fields_ = [
        ("ngram_size", ctypes.c_int32),
        ("heads_per_ngram", ctypes.c_int32),
        ("multipliers", ctypes.c_int64 * ENGRAM_MAX_NGRAM),
        ("vocab_sizes", ctypes.c_int64 * ENGRAM_MAX_HEADS),
        ("offsets", ctypes.c_int64 * ENGRAM_MAX_HEADS),
        ("fill_id", ctypes.c_int64),
        ("table_rows", ctypes.c_int64),
        ("dim", ctypes.c_int32),
        ("eos_id", ctypes.c_int32),
    ]

    @property
    def heads(self) -> int:
        return (self.ngram_size - 1) * self.heads_per_ngram


class ConvParams(ctypes.Structure):
    """Mirror of engram_conv_params_t."""
    _fields_ = [
        ("channels", ctypes.c_int32),
        ("group_size", ctypes.c_int32),
        ("kernel_size", ctypes.c_int32),
        ("dilation", ctypes.c_int32),
        ("eps", ctypes.c_float),
        ("flags", ctypes.c_uint32),
        ("weight_dtype", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


class AdamParams(ctypes.Structure):
    """Mirror of engram_adam_params_t."""
    _fields_ = [
        ("lr", ctypes.c_float),
        ("beta1", ctypes.c_float),
        ("beta2", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("weight_decay", ctypes.c_float),
        ("reserved", ctypes.c_int32),
        ("step", ctypes.c_int64),
    ]


def make_params(cfg: dict) -> EngramParams:
    """EngramParams from a dict with the NGramEmbedding constructor fields
    (ngram_size, heads_per_ngram, multipliers, vocab_sizes, offsets, eos_id,
    fill_id) and the table shape (table_rows, dim)."""
    p = EngramParams()
    p.ngram_size = int(cfg["ngram_size"])
    p.heads_per_ngram = int(cfg["heads_per_ngram"])
    for k, m in enumerate(cfg["multipliers"]):
        p.multipliers[k] = int(m)
    for h, (v, o) in enumerate(zip(cfg["vocab_sizes"], cfg["offsets"])):
        p.vocab_sizes[h] = int(v)
        p.offsets[h] = int(o)
    p.fill_id = int(cfg.get("fill_id", 0))
    p.table_rows = int(cfg["table_rows"])
    p.dim = int(cfg["dim"])
    p.eos_id = int(cfg["eos_id"])
    return p


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"Engram CUDA library not found at {LIB_PATH}; build it with "
            "`python hashed_gram_embedding_raw_b200/build.py` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "engram_hash": [P, P, P, i32, i64, P, P],
        "engram_gather": [P, i32, i64, i32, P, i64, P, P],
        "engram_hash_gather": [P, P, P, i32, i64, P, i32, P, P, P],
        "engram_backward_workspace_size": [i64, i64, i32, ctypes.POINTER(sz)],
        "engram_backward": [P, i64, i64, i32, P, i32, P, P, P, P, sz, P],
        "engram_backward_sort": [P, i64, i64, i32, P, sz, P],
        "engram_backward_reduce": [i64, i64, i32, P, i32, P, P, P, P, sz, P],
        "engram_get_device_error": [ctypes.POINTER(ctypes.c_uint32), P],
        "engram_status_string": [ctypes.c_int],
        "engram_abi_version": [],
        "engram_params_size": [],
        "engram_launch_count": [],
        "engram_host_floor_mod": [i64, i64, ctypes.POINTER(ctypes.c_int)],
        "engram_backward_noalloc": [P, i64, i64, i32, P, i32, P, P, P, P],
        "engram_hash_gather_slice": [P, P, P, i32, i64, i64, i64, i64, P, i32, P, P, P],
        "engram_ple_short_conv": [P, P, i32, P, i32, i64, P, P, P, P, i32, P],
        "engram_ple_short_conv_save": [P, P, i32, P, i32, i64, P, P, P, P, i32, P, P],
        "engram_grouped_rms_norm": [P, i32, i64, i32, i32, P, i32, ctypes.c_float, P, i32, P],
        "engram_sparse_adam": [P, P, i32, i64, i32, P, P, P, P, P, i64, P],
        "engram_ple_short_conv_backward": [P, P, i32, P, i32, i64, P, P, P, P, i32, P, P, P, P,
                                           P, sz, P],
        "engram_ple_short_conv_backward_saved": [P, P, i32, P, i32, i64, P, P, P, P, P, i32, P,
                                                 P, P, P, P, sz, P],
        "engram_ple_short_conv_backward_workspace_size": [P, i64, ctypes.POINTER(sz)],
        "engram_owner_bucket": [P, i64, i64, i32, P, P, P, P, P, sz, P],
        "engram_owner_bucket_workspace_size": [i64, i32, ctypes.POINTER(sz)],
        "engram_backward_heads": [P, P, i64, P, i32, P, P, P, P, sz, P],
        "engram_backward_sort_heads": [P, P, i64, P, sz, P],
        "engram_owner_bucket_padded": [P, i64, i64, i32, i64, P, P, P, P, P, sz, P],
    }
    for name, args in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    L.engram_status_string.restype = ctypes.c_char_p
    L.engram_params_size.restype = sz
    L.engram_launch_count.restype = ctypes.c_uint64
    L.engram_host_floor_mod.restype = i64
    if L.engram_params_size() != ctypes.sizeof(EngramParams):
        raise ImportError("engram_params_t layout differs between library and binding")
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.engram_status_string(int(status)).decode()


def _check(rc: int, what: str):
    if rc != ENGRAM_OK:
        raise EngramError(what, rc)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DTYPE_CODE[t.dtype]
    except KeyError:
        raise ValueError(f"unsupported dtype {t.dtype}") from None


def _cu_args(cu_seqlens):
    if cu_seqlens is None:
        return None, 1
    _cuda(cu_seqlens, "cu_seqlens", torch.int32)
    return cu_seqlens, cu_seqlens.numel() - 1


# ------------------------------------------------------------------ forward

def engram_hash(params: EngramParams, ids: torch.Tensor, cu_seqlens=None, out_idx=None,
                stream=None) -> torch.Tensor:
    """Row indices [T, H] int32 of every hash head for every token."""
    _cuda(ids, "ids", torch.int32)
    T = ids.numel()
    cu, nseq = _cu_args(cu_seqlens)
    if out_idx is None:
        out_idx = torch.empty((T, params.heads), dtype=torch.int32, device=ids.device)
    _cuda(out_idx, "out_idx", torch.int32)
    if out_idx.numel() != T * params.heads:
        raise ValueError("out_idx must hold T * H elements")
    _check(lib.engram_hash(ctypes.byref(params), _ptr(ids), _ptr(cu), nseq, T,
                           _ptr(out_idx), _stream(stream)), "engram_hash")
    return out_idx


def engram_gather(table: torch.Tensor, idx: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """out[i, :] = table[idx[i], :] for an int32 index tensor of any shape."""
    _cuda(table, "table")
    _cuda(idx, "idx", torch.int32)
    rows, dim = table.shape
    n = idx.numel()
    if out is None:
        out = torch.empty(tuple(idx.shape) + (dim,), dtype=table.dtype, device=table.device)
    _cuda(out, "out", table.dtype)
    if out.numel() != n * dim:
        raise ValueError("out must hold n * dim elements")
    _check(lib.engram_gather(_ptr(table), _dtype_code(table), rows, dim, _ptr(idx), n,
                             _ptr(out), _stream(stream)), "engram_gather")
    return out


def engram_hash_gather(params: EngramParams, ids: torch.Tensor, table: torch.Tensor,
                       cu_seqlens=None, out=None, out_idx=None, want_idx: bool = True,
                       stream=None):
    """Fused hash + gather: returns (out [T, H * dim], out_idx [T, H] or None)."""
    _cuda(ids, "ids", torch.int32)
    _cuda(table, "table")
    if table.shape != (params.table_rows, params.dim):
        raise ValueError("table shape must be (params.table_rows, params.dim)")
    T, H = ids.numel(), params.heads
    cu, nseq = _cu_args(cu_seqlens)
    if out is None:
        out = torch.empty((T, H * params.dim), dtype=table.dtype, device=table.device)
    _cuda(out, "out", table.dtype)
    if out.numel() != T * H * params.dim:
        raise ValueError("out must hold T * H * dim elements")
    if out_idx is None and want_idx:
        out_idx = torch.empty((T, H), dtype=torch.int32, device=ids.device)
    if out_idx is not None:
        _cuda(out_idx, "out_idx", torch.int32)
        if out_idx.numel() != T * H:
            raise ValueError("out_idx must hold T * H elements")
    _check(lib.engram_hash_gather(ctypes.byref(params), _ptr(ids), _ptr(cu), nseq, T,
                                  _ptr(table), _dtype_code(table), _ptr(out_idx), _ptr(out),
                                  _stream(stream)), "engram_hash_gather")
    return out, out_idx


def engram_hash_gather_slice(params: EngramParams, ids: torch.Tensor, table: torch.Tensor,
                             start: int, end: int, row_len: int = 0, cu_seqlens=None,
                             out=None, out_idx=None, want_idx: bool = True, stream=None):
    """_forward_global_slice: hash the whole stream, look up positions
    [start, end) of every row of row_len tokens (0: one row). Returns
    (out [rows, end - start, H * dim], out_idx [rows, end - start, H] or None)."""
    _cuda(ids, "ids", torch.int32)
    _cuda(table, "table")
    if table.shape != (params.table_rows, params.dim):
        raise ValueError("table shape must be (params.table_rows, params.dim)")
    T, H = ids.numel(), params.heads
    row = row_len or T
    if row <= 0 or T % row or not 0 <= start <= end <= row:
        raise ValueError("need 0 <= start <= end <= row_len and T divisible by row_len")
    nrows, ln = T // row, end - start
    cu, nseq = _cu_args(cu_seqlens)
    if out is None:
        out = torch.empty((nrows, ln, H * params.dim), dtype=table.dtype, device=table.device)
    _cuda(out, "out", table.dtype)
    if out.numel() != nrows * ln * H * params.dim:
        raise ValueError("out must hold rows * (end - start) * H * dim elements")
    if out_idx is None and want_idx:
        out_idx = torch.empty((nrows, ln, H), dtype=torch.int32, device=ids.device)
    if out_idx is not None:
        _cuda(out_idx, "out_idx", torch.int32)
        if out_idx.numel() != nrows * ln * H:
            raise ValueError("out_idx must hold rows * (end - start) * H elements")
    _check(lib.engram_hash_gather_slice(ctypes.byref(params), _ptr(ids), _ptr(cu), nseq, T,
                                        row_len, start, end, _ptr(table), _dtype_code(table),
                                        _ptr(out_idx), _ptr(out), _stream(stream)),
           "engram_hash_gather_slice")
    return out, out_idx


# ----------------------------------------------------------------- backward

def engram_backward_workspace_size(n: int, table_rows: int, dim: int) -> int:
    b = ctypes.c_size_t(0)
    _check(lib.engram_backward_workspace_size(n, table_rows, dim, ctypes.byref(b)),
           "engram_backward_workspace_size")
    return b.value


def _bwd_buffers(n, dim, device, uniq_rows, row_grads, num_unique, workspace, table_rows):
    if uniq_rows is None:
        uniq_rows = torch.empty(max(n, 1), dtype=torch.int32, device=device)
    if row_grads is None:
        row_grads = torch.empty((max(n, 1), dim), dtype=torch.float32, device=device)
    if num_unique is None:
        num_unique = torch.empty(1, dtype=torch.int32, device=device)
    if workspace is None:
        workspace = torch.empty(engram_backward_workspace_size(n, table_rows, dim),
                                dtype=torch.uint8, device=device)
    _cuda(uniq_rows, "uniq_rows", torch.int32)
    _cuda(row_grads, "row_grads", torch.float32)
    _cuda(num_unique, "num_unique", torch.int32)
    _cuda(workspace, "workspace", torch.uint8)
    if uniq_rows.numel() < n or row_grads.numel() < n * dim:
        raise ValueError("uniq_rows / row_grads must hold n rows")
    return uniq_rows, row_grads, num_unique, workspace


def engram_backward(idx: torch.Tensor, dout: torch.Tensor, table_rows: int, uniq_rows=None,
                    row_grads=None, num_unique=None, workspace=None, stream=None):
    """Compact table gradient: (uniq_rows [cap], row_grads [cap, dim] fp32,
    num_unique [1]); the first num_unique entries are valid."""
    _cuda(idx, "idx", torch.int32)
    _cuda(dout, "dout")
    n = idx.numel()
    dim = dout.shape[-1]
    if dout.numel() != n * dim:
        raise ValueError("dout must be [n, dim] for n = idx.numel()")
    uniq_rows, row_grads, num_unique, workspace = _bwd_buffers(
        n, dim, idx.device, uniq_rows, row_grads, num_unique, workspace, table_rows)
    _check(lib.engram_backward(_ptr(idx), n, table_rows, dim, _ptr(dout), _dtype_code(dout),
                               _ptr(uniq_rows), _ptr(row_grads), _ptr(num_unique),
                               _ptr(workspace), workspace.numel(), _stream(stream)),
           "engram_backward")
    return uniq_rows, row_grads, num_unique


def engram_backward_noalloc(idx: torch.Tensor, dout: torch.Tensor, table_rows: int,
                            uniq_rows, row_grads, num_unique, stream=None) -> None:
    """engram_backward for callers that cannot allocate device memory: the
    library uses its own fixed device scratch array (ENGRAM_NOALLOC_SCRATCH_BYTES)
    instead of a workspace, and the caller passes preallocated outputs. Calls
    that overlap on the GPU share that array and race; serialise them."""
    _cuda(idx, "idx", torch.int32)
    _cuda(dout, "dout")
    n = idx.numel()
    dim = dout.shape[-1]
    if dout.numel() != n * dim:
        raise ValueError("dout must be [n, dim] for n = idx.numel()")
    _cuda(uniq_rows, "uniq_rows", torch.int32)
    _cuda(row_grads, "row_grads", torch.float32)
    _cuda(num_unique, "num_unique", torch.int32)
    if uniq_rows.numel() < n or row_grads.numel() < n * dim:
        raise ValueError("uniq_rows / row_grads must hold n rows")
    _check(lib.engram_backward_noalloc(_ptr(idx), n, table_rows, dim, _ptr(dout),
                                       _dtype_code(dout), _ptr(uniq_rows), _ptr(row_grads),
                                       _ptr(num_unique), _stream(stream)),
           "engram_backward_noalloc")


def engram_backward_sort(idx: torch.Tensor, table_rows: int, dim: int, workspace,
                         stream=None) -> None:
    _cuda(idx, "idx", torch.int32)
    _cuda(workspace, "workspace", torch.uint8)
    _check(lib.engram_backward_sort(_ptr(idx), idx.numel(), table_rows, dim, _ptr(workspace),
                                    workspace.numel(), _stream(stream)), "engram_backward_sort")


def engram_backward_heads(params: EngramParams, idx: torch.Tensor, dout: torch.Tensor,
                          uniq_rows=None, row_grads=None, num_unique=None, workspace=None,
                          stream=None):
    """engram_backward for the hash's lookups idx [T, H] (head h's lookups in
    its own slice), sorted by head: same results, fewer radix passes."""
    _cuda(idx, "idx", torch.int32)
    _cuda(dout, "dout")
    H, dim, rows = params.heads, params.dim, params.table_rows
    n = idx.numel()
    if n % H != 0 or dout.numel() != n * dim:
        raise ValueError("idx must be [T, H] and dout [T * H, dim]")
    uniq_rows, row_grads, num_unique, workspace = _bwd_buffers(
        n, dim, idx.device, uniq_rows, row_grads, num_unique, workspace, rows)
    _check(lib.engram_backward_heads(ctypes.byref(params), _ptr(idx), n // H, _ptr(dout),
                                     _dtype_code(dout), _ptr(uniq_rows), _ptr(row_grads),
                                     _ptr(num_unique), _ptr(workspace), workspace.numel(),
                                     _stream(stream)), "engram_backward_heads")
    return uniq_rows, row_grads, num_unique


def engram_backward_sort_heads(params: EngramParams, idx: torch.Tensor, workspace,
                               stream=None) -> None:
    _cuda(idx, "idx", torch.int32)
    _cuda(workspace, "workspace", torch.uint8)
    H = params.heads
    if idx.numel() % H != 0:
        raise ValueError("idx must be [T, H]")
    _check(lib.engram_backward_sort_heads(ctypes.byref(params), _ptr(idx), idx.numel() // H,
                                          _ptr(workspace), workspace.numel(), _stream(stream)),
           "engram_backward_sort_heads")


def engram_backward_reduce(n: int, table_rows: int, dout: torch.Tensor, uniq_rows, row_grads,
                           num_unique, workspace, stream=None) -> None:
    _cuda(dout, "dout")
    dim = dout.shape[-1]
    _bwd_buffers(n, dim, dout.device, uniq_rows, row_grads, num_unique, workspace, table_rows)
    _check(lib.engram_backward_reduce(n, table_rows, dim, _ptr(dout), _dtype_code(dout),
                                      _ptr(uniq_rows), _ptr(row_grads), _ptr(num_unique),
                                      _ptr(workspace), workspace.numel(), _stream(stream)),
           "engram_backward_reduce")


# ----------------------------------------------------------- PLE layer tail

def _out_like(x: torch.Tensor, out, out_dtype):
    dt = x.dtype if out_dtype is None else out_dtype
    if out is None:
        out = torch.empty(x.shape, dtype=dt, device=x.device)
    _cuda(out, "out", dt)
    if out.shape != x.shape:
        raise ValueError("out must have the shape of x")
    return out


def engram_ple_short_conv(x: torch.Tensor, conv_weight: torch.Tensor, *, dilation: int,
                          group_size: int, cu_seqlens=None, norm_weight=None, conv_bias=None,
                          eps: float = 1e-6, norm: bool = True, silu: bool = True,
                          residual: bool = True, out=None, out_dtype=None,
                          inv_rms=None, stream=None) -> torch.Tensor:
    """PLE tail over x [T, C]: x + SiLU(causal depthwise conv(grouped RMS norm(x)))
    with each of norm, SiLU and residual optional; conv_weight is [C, K] (or
    the conv1d layout [C, 1, K]); all weights share one dtype. inv_rms, an
    fp32 [T, C / group_size] tensor (norm on), receives every branch slice's
    inverse RMS for engram_ple_short_conv_backward(..., inv_rms=...)."""
    _cuda(x, "x")
    if x.dim() != 2:
        raise ValueError("x must be [T, C]")
    T, C = x.shape
    w = conv_weight.reshape(C, -1) if conv_weight.dim() == 3 else conv_weight
    _cuda(w, "conv_weight")
    if w.shape[0] != C:
        raise ValueError("conv_weight must be [C, K]")
    for name, t in (("norm_weight", norm_weight), ("conv_bias", conv_bias)):
        if t is not None:
            _cuda(t, name, w.dtype)
            if t.numel() != C:
                raise ValueError(f"{name} must hold C elements")
    cu, nseq = _cu_args(cu_seqlens)
    out = _out_like(x, out, out_dtype)
    p = ConvParams(C, int(group_size), w.shape[1], int(dilation), float(eps),
                   (ENGRAM_CONV_NORM if norm else 0) | (ENGRAM_CONV_SILU if silu else 0)
                   | (ENGRAM_CONV_RESIDUAL if residual else 0), _dtype_code(w), 0)
    if inv_rms is None:
        _check(lib.engram_ple_short_conv(ctypes.byref(p), _ptr(x), _dtype_code(x), _ptr(cu),
                                         nseq, T, _ptr(norm_weight), _ptr(w), _ptr(conv_bias),
                                         _ptr(out), _dtype_code(out), _stream(stream)),
               "engram_ple_short_conv")
        return out
    _inv_rms_arg(inv_rms, T, C, group_size)
    _check(lib.engram_ple_short_conv_save(ctypes.byref(p), _ptr(x), _dtype_code(x), _ptr(cu),
                                          nseq, T, _ptr(norm_weight), _ptr(w), _ptr(conv_bias),
                                          _ptr(out), _dtype_code(out), _ptr(inv_rms),
                                          _stream(stream)),
           "engram_ple_short_conv_save")
    return out


def _inv_rms_arg(inv_rms, T, C, group_size):
    _cuda(inv_rms, "inv_rms", torch.float32)
    if group_size < 1 or C % group_size or inv_rms.numel() != T * (C // group_size):
        raise ValueError("inv_rms must hold T * C / group_size floats")


def _conv_params(C, group_size, w, dilation, eps, norm, silu, residual):
    return ConvParams(C, int(group_size), w.shape[1], int(dilation), float(eps),
                      (ENGRAM_CONV_NORM if norm else 0) | (ENGRAM_CONV_SILU if silu else 0)
                      | (ENGRAM_CONV_RESIDUAL if residual else 0), _dtype_code(w), 0)


def engram_ple_short_conv_backward_workspace_size(channels: int, group_size: int,
                                                  kernel_size: int, dilation: int,
                                                  tokens: int) -> int:
    """Workspace bytes of engram_ple_short_conv_backward on the current device."""
    p = ConvParams(int(channels), int(group_size), int(kernel_size), int(dilation), 1e-6,
                   ENGRAM_CONV_NORM | ENGRAM_CONV_SILU | ENGRAM_CONV_RESIDUAL, ENGRAM_F32, 0)
    n = ctypes.c_size_t(0)
    _check(lib.engram_ple_short_conv_backward_workspace_size(ctypes.byref(p), int(tokens),
                                                             ctypes.byref(n)),
           "engram_ple_short_conv_backward_workspace_size")
    return n.value


def engram_ple_short_conv_backward(x: torch.Tensor, conv_weight: torch.Tensor,
                                   dout: torch.Tensor, *, dilation: int, group_size: int,
                                   cu_seqlens=None, norm_weight=None, conv_bias=None,
                                   eps: float = 1e-6, norm: bool = True, silu: bool = True,
                                   residual: bool = True, dx=None, dnorm_weight=None,
                                   dconv_weight=None, dconv_bias=None, workspace=None,
                                   inv_rms=None, stream=None):
    """Gradients of engram_ple_short_conv's output given dout [T, C]:
    returns (dx [T, C] of dout's dtype, dnorm_weight [C], dconv_weight [C, K],
    dconv_bias [C]), the weight gradients fp32. Optional outputs and the
    workspace (uint8) may be passed in; they are allocated otherwise.
    inv_rms: the forward's saved inverse RMS (engram_ple_short_conv(...,
    inv_rms=...)) for the same x, which the backward then uses instead of
    computing it (norm on)."""
    _cuda(x, "x")
    _cuda(dout, "dout")
    if x.dim() != 2 or dout.shape != x.shape:
        raise ValueError("x and dout must both be [T, C]")
    T, C = x.shape
    w = conv_weight.reshape(C, -1) if conv_weight.dim() == 3 else conv_weight
    _cuda(w, "conv_weight")
    if w.shape[0] != C:
        raise ValueError("conv_weight must be [C, K]")
    K = w.shape[1]
    for name, t in (("norm_weight", norm_weight), ("conv_bias", conv_bias)):
        if t is not None:
            _cuda(t, name, w.dtype)
            if t.numel() != C:
                raise ValueError(f"{name} must hold C elements")
    cu, nseq = _cu_args(cu_seqlens)
    dev = x.device
    dx = _out_like(dout, dx, None)
    dnorm_weight = torch.empty(C, device=dev) if dnorm_weight is None else dnorm_weight
    dconv_weight = torch.empty((C, K), device=dev) if dconv_weight is None else dconv_weight
    dconv_bias = torch.empty(C, device=dev) if dconv_bias is None else dconv_bias
    for name, t, n in (("dnorm_weight", dnorm_weight, C), ("dconv_weight", dconv_weight, C * K),
                       ("dconv_bias", dconv_bias, C)):
        _cuda(t, name, torch.float32)
        if t.numel() != n:
            raise ValueError(f"{name} must hold {n} elements")
    p = _conv_params(C, group_size, w, dilation, eps, norm, silu, residual)
    if workspace is None:
        need = engram_ple_short_conv_backward_workspace_size(C, group_size, K, dilation, T)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _cuda(workspace, "workspace", torch.uint8)
    if inv_rms is None:
        _check(lib.engram_ple_short_conv_backward(
            ctypes.byref(p), _ptr(x), _dtype_code(x), _ptr(cu), nseq, T, _ptr(norm_weight),
            _ptr(w), _ptr(conv_bias), _ptr(dout), _dtype_code(dout), _ptr(dx),
            _ptr(dnorm_weight), _ptr(dconv_weight), _ptr(dconv_bias), _ptr(workspace),
            workspace.numel(), _stream(stream)), "engram_ple_short_conv_backward")
        return dx, dnorm_weight, dconv_weight, dconv_bias
    _inv_rms_arg(inv_rms, T, C, group_size)
    _check(lib.engram_ple_short_conv_backward_saved(
        ctypes.byref(p), _ptr(x), _dtype_code(x), _ptr(cu), nseq, T, _ptr(norm_weight), _ptr(w),
        _ptr(conv_bias), _ptr(inv_rms), _ptr(dout), _dtype_code(dout), _ptr(dx),
        _ptr(dnorm_weight), _ptr(dconv_weight), _ptr(dconv_bias), _ptr(workspace),
        workspace.numel(), _stream(stream)), "engram_ple_short_conv_backward_saved")
    return dx, dnorm_weight, dconv_weight, dconv_bias


def engram_owner_bucket_workspace_size(n: int, owners: int) -> int:
    nbytes = ctypes.c_size_t(0)
    _check(lib.engram_owner_bucket_workspace_size(int(n), int(owners), ctypes.byref(nbytes)),
           "engram_owner_bucket_workspace_size")
    return nbytes.value


def engram_owner_bucket(rows: torch.Tensor, rows_per_owner: int, owners: int, send_rows=None,
                        src_pos=None, dst_pos=None, counts=None, workspace=None, stream=None):
    """Stable grouping of lookups by owner rank (rows // rows_per_owner):
    returns (send_rows [n] owner-local rows in owner order, src_pos [n] the
    lookup of each grouped position, dst_pos [n] the grouped position of each
    lookup, counts [owners] int32 on the device)."""
    _cuda(rows, "rows", torch.int32)
    n = rows.numel()
    dev = rows.device

    def buf(t, name, size):
        t = torch.empty(size, dtype=torch.int32, device=dev) if t is None else t
        _cuda(t, name, torch.int32)
        if t.numel() != size:
            raise ValueError(f"{name} must hold {size} elements")
        return t

    send_rows, src_pos, dst_pos = (buf(send_rows, "send_rows", n), buf(src_pos, "src_pos", n),
                                   buf(dst_pos, "dst_pos", n))
    counts = buf(counts, "counts", int(owners))
    if workspace is None:
        workspace = torch.empty(max(16, engram_owner_bucket_workspace_size(n, owners)),
                                dtype=torch.uint8, device=dev)
    _cuda(workspace, "workspace", torch.uint8)
    _check(lib.engram_owner_bucket(_ptr(rows), n, int(rows_per_owner), int(owners),
                                   _ptr(send_rows), _ptr(src_pos), _ptr(dst_pos), _ptr(counts),
                                   _ptr(workspace), workspace.numel(), _stream(stream)),
           "engram_owner_bucket")
    return send_rows, src_pos, dst_pos, counts


def engram_owner_bucket_padded(rows: torch.Tensor, rows_per_owner: int, owners: int,
                               capacity: int, send_rows=None, src_pos=None, dst_pos=None,
                               counts=None, workspace=None, stream=None):
    """engram_owner_bucket into fixed-capacity segments: (send_rows
    [owners * capacity], src_pos [owners * capacity] with -1 padding, dst_pos
    [n] (-1 for a lookup dropped past the capacity), counts [owners])."""
    _cuda(rows, "rows", torch.int32)
    n = rows.numel()
    dev = rows.device
    slots = int(owners) * int(capacity)

    def buf(t, name, size):
        t = torch.empty(size, dtype=torch.int32, device=dev) if t is None else t
        _cuda(t, name, torch.int32)
        if t.numel() != size:
            raise ValueError(f"{name} must hold {size} elements")
        return t

    send_rows, src_pos = buf(send_rows, "send_rows", slots), buf(src_pos, "src_pos", slots)
    dst_pos, counts = buf(dst_pos, "dst_pos", n), buf(counts, "counts", int(owners))
    if workspace is None:
        workspace = torch.empty(max(16, engram_owner_bucket_workspace_size(n, owners)),
                                dtype=torch.uint8, device=dev)
    _cuda(workspace, "workspace", torch.uint8)
    _check(lib.engram_owner_bucket_padded(_ptr(rows), n, int(rows_per_owner), int(owners),
                                          int(capacity), _ptr(send_rows), _ptr(src_pos),
                                          _ptr(dst_pos), _ptr(counts), _ptr(workspace),
                                          workspace.numel(), _stream(stream)),
           "engram_owner_bucket_padded")
    return send_rows, src_pos, dst_pos, counts


def engram_grouped_rms_norm(x: torch.Tensor, group_size: int, weight=None, eps: float = 1e-6,
                            out=None, out_dtype=None, stream=None) -> torch.Tensor:
    """Branch-local Gemma RMS norm of x [..., C] over groups of group_size
    features, scale (1 + weight); out may be x itself (in place)."""
    _cuda(x, "x")
    C = x.shape[-1]
    rows = x.numel() // C if C else 0
    wdt = ENGRAM_F32
    if weight is not None:
        _cuda(weight, "weight")
        if weight.numel() != C:
            raise ValueError("weight must hold C elements")
        wdt = _dtype_code(weight)
    out = _out_like(x, out, out_dtype)
    _check(lib.engram_grouped_rms_norm(_ptr(x), _dtype_code(x), rows, C, int(group_size),
                                       _ptr(weight), wdt, float(eps), _ptr(out),
                                       _dtype_code(out), _stream(stream)),
           "engram_grouped_rms_norm")
    return out


# ---------------------------------------------------------- optimizer step

def engram_sparse_adam(table: torch.Tensor, exp_avg: torch.Tensor, exp_avg_sq: torch.Tensor,
                       uniq_rows: torch.Tensor, row_grads: torch.Tensor, num_unique: torch.Tensor,
                       *, lr: float, betas=(0.9, 0.999), eps: float = 1e-8,
                       weight_decay: float = 0.0, step: int, stream=None) -> None:
    """Lazy AdamW step, in place, on the rows uniq_rows[:num_unique] of
    `table` [R, D] (fp32 / bf16 / fp16) with fp32 moments [R, D];
    num_unique is the device scalar the backward wrote."""
    _cuda(table, "table")
    _cuda(exp_avg, "exp_avg", torch.float32)
    _cuda(exp_avg_sq, "exp_avg_sq", torch.float32)
    _cuda(uniq_rows, "uniq_rows", torch.int32)
    _cuda(row_grads, "row_grads", torch.float32)
    _cuda(num_unique, "num_unique", torch.int32)
    R, D = table.shape
    if exp_avg.shape != table.shape or exp_avg_sq.shape != table.shape:
        raise ValueError("moments must have the table's shape")
    cap = uniq_rows.numel()
    if row_grads.numel() < cap * D:
        raise ValueError("row_grads must hold capacity x D values")
    p = AdamParams(float(lr), float(betas[0]), float(betas[1]), float(eps), float(weight_decay),
                   0, int(step))
    _check(lib.engram_sparse_adam(ctypes.byref(p), _ptr(table), _dtype_code(table), R, D,
                                  _ptr(exp_avg), _ptr(exp_avg_sq), _ptr(uniq_rows),
                                  _ptr(row_grads), _ptr(num_unique), cap, _stream(stream)),
           "engram_sparse_adam")


# -------------------------------------------------------------------- misc

def engram_get_device_error(stream=None) -> int:
    """ENGRAM_DEVERR_* bits set since the last call (synchronises the stream)."""
    v = ctypes.c_uint32(0)
    _check(lib.engram_get_device_error(ctypes.byref(v), _stream(stream)),
           "engram_get_device_error")
    return int(v.value)


def engram_launch_count() -> int:
    return int(lib.engram_launch_count())


def engram_abi_version() -> int:
    return int(lib.engram_abi_version())


def engram_host_floor_mod(a: int, m: int) -> int:
    st = ctypes.c_int(0)
    r = lib.engram_host_floor_mod(int(a), int(m), ctypes.byref(st))
    _check(st.value, "engram_host_floor_mod")
    return int(r)
