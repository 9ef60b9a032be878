"""CPU oracle of the Engram N-gram Embedding path (hash, gather, backward,
the PLE layer's grouped RMS norm and causal short convolution with its
backward, and the sparse optimizer step on the touched rows).

TEST INFRASTRUCTURE ONLY. Only `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline / reference legs of `bench.py` may import this package. The
product path (`hashed_gram_embedding_raw_b200`) never imports it and shares no
code with it.

`engram_oracle.c` is the oracle proper (scalar C, fp64 accumulation);
`bruteforce.py` is an independent exact-integer statement of the hash that
pins it on tiny inputs. This module compiles the C file with gcc (`build()`)
and wraps it with ctypes over NumPy arrays.

Parity of the hash against the released checkpoint is unpinned: the engram
page prints no worked example. What pins each function is listed in the
oracle tests.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "engram_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

F32, BF16, F16 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into oracle/liboracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-shared",
                               "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def build_mutant(mutant: int, outdir: str):
    """Build a copy of the oracle with one planted mistake (tests only) and
    return it loaded; see ORACLE_MUTANT in engram_oracle.c."""
    path = os.path.join(outdir, f"liboracle_mutant{mutant}.so")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC",
                           f"-DORACLE_MUTANT={int(mutant)}", "-o", path, _SRC, "-lm"])
    return _declare(ctypes.CDLL(path))


def _declare(L):
    P = ctypes.c_void_p
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    L.oracle_hash.argtypes = [i32, i32, P, P, P, i64, i32, P, P, i32, i64, P]
    L.oracle_hash.restype = ctypes.c_int
    L.oracle_gather.argtypes = [P, i64, i64, P, i64, P]
    L.oracle_gather.restype = ctypes.c_int
    L.oracle_backward.argtypes = [P, i64, P, ctypes.c_int, i32, P, P, P]
    L.oracle_backward.restype = ctypes.c_int
    L.oracle_grouped_rms_norm.argtypes = [P, ctypes.c_int, i64, i32, i32, P, ctypes.c_int,
                                          ctypes.c_double, P]
    L.oracle_grouped_rms_norm.restype = ctypes.c_int
    L.oracle_short_conv.argtypes = [P, ctypes.c_int, P, i32, i64, i32, i32, P, ctypes.c_double,
                                    P, P, ctypes.c_int, i32, i32, ctypes.c_int, ctypes.c_int,
                                    ctypes.c_int, P]
    L.oracle_short_conv.restype = ctypes.c_int
    d = ctypes.c_double
    L.oracle_sparse_adam.argtypes = [P, P, P, i64, i32, P, P, i64, d, d, d, d, d, i64]
    L.oracle_sparse_adam.restype = ctypes.c_int
    L.oracle_short_conv_backward.argtypes = [P, ctypes.c_int, P, i32, i64, i32, i32, P, d, P, P,
                                             ctypes.c_int, i32, i32, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, P, P, P, P, P]
    L.oracle_short_conv_backward.restype = ctypes.c_int
    return L


def lib():
    global _lib
    if _lib is None:
        build()
        _lib = _declare(ctypes.CDLL(_LIB))
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def hash_ids(ids, cu, params) -> np.ndarray:
    """Global row IDs [T, H] (int64) of every head for every token."""
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    T = ids.shape[0]
    N, K = params["ngram_size"], params["heads_per_ngram"]
    H = (N - 1) * K
    mult = np.asarray(params["multipliers"], dtype=np.int64)
    vocab = np.asarray(params["vocab_sizes"], dtype=np.int64)
    off = np.asarray(params["offsets"], dtype=np.int64)
    out = np.empty((T, H), dtype=np.int64)
    if cu is None:
        cu_arr, nseq, cu_p = None, 1, None
    else:
        cu_arr = np.ascontiguousarray(cu, dtype=np.int32)
        nseq, cu_p = cu_arr.shape[0] - 1, _ptr(cu_arr)
    rc = lib().oracle_hash(N, K, _ptr(mult), _ptr(vocab), _ptr(off),
                           int(params["fill_id"]), int(params["eos_id"]),
                           _ptr(ids), cu_p, nseq, T, _ptr(out))
    if rc != 0:
        raise ValueError("oracle_hash: invalid arguments")
    return out


def gather(table: np.ndarray, idx) -> np.ndarray:
    """out[i, :] = table[idx[i], :] bit for bit; table is any [R, D] array."""
    table = np.ascontiguousarray(table)
    idx = np.ascontiguousarray(np.asarray(idx).reshape(-1), dtype=np.int64)
    out = np.empty((idx.shape[0],) + table.shape[1:], dtype=table.dtype)
    row_bytes = table.strides[0] if table.ndim > 1 else table.itemsize
    rc = lib().oracle_gather(_ptr(table), table.shape[0], row_bytes, _ptr(idx),
                             idx.shape[0], _ptr(out))
    if rc != 0:
        raise IndexError("oracle_gather: row index out of range")
    return out


def backward(idx, dout: np.ndarray, dtype: int):
    """(uniq_rows int64 [U], row_grads fp32 [U, D]) of the row-gradient sum.

    `dout` holds raw values of `dtype` (F32: float32 array; BF16/F16: uint16
    bit patterns), shape [n, D].
    """
    idx = np.ascontiguousarray(np.asarray(idx).reshape(-1), dtype=np.int64)
    dout = np.ascontiguousarray(dout)
    n, D = dout.shape
    assert n == idx.shape[0]
    uniq = np.empty(max(n, 1), dtype=np.int64)
    grads = np.empty((max(n, 1), D), dtype=np.float32)
    nu = np.zeros(1, dtype=np.int64)
    rc = lib().oracle_backward(_ptr(idx), n, _ptr(dout), dtype, D, _ptr(uniq),
                               _ptr(grads), _ptr(nu))
    if rc != 0:
        raise ValueError("oracle_backward: invalid arguments")
    U = int(nu[0])
    return uniq[:U].copy(), grads[:U].copy()


def _raw(a, dtype):
    """Contiguous raw buffer of `dtype` (F32: float32 values; BF16/F16: uint16
    bit patterns, or float16 values for F16)."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if dtype == F32:
        return np.ascontiguousarray(a, dtype=np.float32)
    if a.dtype == np.float16:
        return a.view(np.uint16)
    assert a.dtype == np.uint16, "BF16/F16 buffers are passed as uint16 bit patterns"
    return a


def grouped_rms_norm(x, dtype, group, weight=None, wdtype=F32, eps=1e-6) -> np.ndarray:
    """fp64 [rows, C] Gemma-style norm of every group of `group` features."""
    xr = _raw(x, dtype)
    rows, C = xr.shape
    wr = _raw(weight, wdtype)
    out = np.empty((rows, C), dtype=np.float64)
    rc = lib().oracle_grouped_rms_norm(_ptr(xr), dtype, rows, C, group,
                                       None if wr is None else _ptr(wr), wdtype, float(eps),
                                       _ptr(out))
    if rc != 0:
        raise ValueError("oracle_grouped_rms_norm: invalid arguments")
    return out


def short_conv(x, dtype, cu, conv_w, *, dilation, group=None, norm_w=None, eps=1e-6,
               bias=None, wdtype=F32, norm=True, silu=True, residual=True) -> np.ndarray:
    """fp64 [T, C] output of the PLE tail x + SiLU(conv(norm(x))) (each of
    norm, SiLU and residual optional); conv_w is [C, K]."""
    xr = _raw(x, dtype)
    T, C = xr.shape
    wr = _raw(conv_w, wdtype)
    K = wr.shape[1]
    nw, br = _raw(norm_w, wdtype), _raw(bias, wdtype)
    if cu is None:
        cu_arr, nseq, cu_p = None, 1, None
    else:
        cu_arr = np.ascontiguousarray(cu, dtype=np.int32)
        nseq, cu_p = cu_arr.shape[0] - 1, _ptr(cu_arr)
    out = np.empty((T, C), dtype=np.float64)
    rc = lib().oracle_short_conv(_ptr(xr), dtype, cu_p, nseq, T, C,
                                 int(group if group else C),
                                 None if nw is None else _ptr(nw), float(eps), _ptr(wr),
                                 None if br is None else _ptr(br), wdtype, K, int(dilation),
                                 int(bool(norm)), int(bool(silu)), int(bool(residual)),
                                 _ptr(out))
    if rc != 0:
        raise ValueError("oracle_short_conv: invalid arguments")
    return out


def sparse_adam(p, m, v, rows, grads, *, lr, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0,
                step=1):
    """One lazy AdamW step on `rows` (int64 [U]) with row gradients `grads`
    (fp32 [U, D]); p, m, v are fp64 [R, D] arrays, returned updated copies."""
    p = np.array(p, dtype=np.float64, order="C")
    m = np.array(m, dtype=np.float64, order="C")
    v = np.array(v, dtype=np.float64, order="C")
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1)
    grads = np.ascontiguousarray(grads, dtype=np.float32)
    R, D = p.shape
    U = rows.shape[0]
    assert grads.shape == (U, D)
    rc = lib().oracle_sparse_adam(_ptr(p), _ptr(m), _ptr(v), R, D, _ptr(rows),
                                  _ptr(grads) if U else None, U, float(lr), float(betas[0]),
                                  float(betas[1]), float(eps), float(weight_decay), int(step))
    if rc != 0:
        raise ValueError("oracle_sparse_adam: invalid arguments")
    return p, m, v


def short_conv_backward(x, dtype, cu, conv_w, dout, *, dilation, group=None, norm_w=None,
                        eps=1e-6, bias=None, wdtype=F32, norm=True, silu=True, residual=True):
    """Gradients of short_conv's output given dout (fp64 [T, C]): returns
    (dx [T, C], dnorm_w [C], dconv_w [C, K], dbias [C]), all fp64."""
    xr = _raw(x, dtype)
    T, C = xr.shape
    wr = _raw(conv_w, wdtype)
    K = wr.shape[1]
    nw, br = _raw(norm_w, wdtype), _raw(bias, wdtype)
    if cu is None:
        cu_arr, nseq, cu_p = None, 1, None
    else:
        cu_arr = np.ascontiguousarray(cu, dtype=np.int32)
        nseq, cu_p = cu_arr.shape[0] - 1, _ptr(cu_arr)
    g = np.ascontiguousarray(dout, dtype=np.float64)
    dx = np.empty((T, C)); dnw = np.empty(C); dw = np.empty((C, K)); db = np.empty(C)
    rc = lib().oracle_short_conv_backward(
        _ptr(xr), dtype, cu_p, nseq, T, C, int(group if group else C),
        None if nw is None else _ptr(nw), float(eps), _ptr(wr), None if br is None else _ptr(br),
        wdtype, K, int(dilation), int(bool(norm)), int(bool(silu)), int(bool(residual)),
        _ptr(g), _ptr(dx), _ptr(dnw), _ptr(dw), _ptr(db))
    if rc != 0:
        raise ValueError("oracle_short_conv_backward: invalid arguments")
    return dx, dnw, dw, db
