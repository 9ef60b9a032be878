"""The C-ABI library loads and exports what include/engram.h declares (CPU only).

No kernel runs here: these checks cover symbol export, the parameter layout,
status strings, host-side argument rejection (which returns before any CUDA
call), and the Barrett modular reduction the kernels use, run on the host.
"""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "engram.h")


@pytest.fixture(scope="session")
def E():
    import __graft_entry__
    __graft_entry__._build_module().build()
    import hashed_gram_embedding_raw_b200 as E
    return E


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^ENGRAM_API\s+[\w\s\*]*?\b(engram_\w+)\(", src, re.M)))


def test_header_declares_expected_entry_points():
    names = declared_functions()
    for must in ("engram_hash", "engram_gather", "engram_hash_gather", "engram_backward",
                 "engram_backward_workspace_size", "engram_get_device_error"):
        assert must in names


def test_library_exports_every_declared_symbol(E):
    out = subprocess.check_output(["nm", "-D", "--defined-only", E.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    # and nothing else of ours leaks out of the library
    assert sorted(n for n in exported if n.startswith("engram")) == declared_functions()
    assert set(E.EXPORTED) == set(declared_functions())


def test_params_layout_and_version(E):
    assert E.lib.engram_params_size() == ctypes.sizeof(E.EngramParams) == 576
    assert E.engram_abi_version() == 2
    for rc in range(4):
        assert E.status_string(rc).startswith("ENGRAM_")
    assert "unknown" in E.status_string(99)


def test_host_floor_mod_matches_python(E):
    rng = np.random.Generator(np.random.PCG64(0))
    mods = [1, 2, 3, 7, 1000003, 20000003, 20000171, 2 ** 31 - 1, 2 ** 32 - 1]
    vals = [0, 1, -1, 2 ** 63 - 1, -(2 ** 63), -(2 ** 63) + 1, 2 ** 62, -(2 ** 62)]
    vals += [int(v) for v in rng.integers(-(2 ** 63), 2 ** 63 - 1, size=400, dtype=np.int64)]
    for m in mods:
        for a in vals:
            assert E.engram_host_floor_mod(a, m) == a % m, (a, m)
        # values next to multiples of m, where a one-off quotient would show
        for k in (1, 2, 12345, 2 ** 31):
            for d in (-1, 0, 1):
                a = k * m + d
                if a < 2 ** 63:
                    assert E.engram_host_floor_mod(a, m) == a % m
                    assert E.engram_host_floor_mod(-a, m) == (-a) % m
    with pytest.raises(E.EngramError):
        E.engram_host_floor_mod(5, 0)


def _page_params(E):
    from workloads import head_params
    return E.make_params(head_params("full"))


def test_host_rejects_bad_params(E):
    L = E.lib
    bad = []
    p = _page_params(E)
    p.ngram_size = 5
    bad.append(p)
    p = _page_params(E)
    p.heads_per_ngram = 0
    bad.append(p)
    p = _page_params(E)
    p.vocab_sizes[3] = 0
    bad.append(p)
    p = _page_params(E)
    p.offsets[15] = p.table_rows - p.vocab_sizes[15] + 1    # slice past the table end
    bad.append(p)
    p = _page_params(E)
    p.table_rows = 2 ** 31 + 1
    bad.append(p)
    dummy = ctypes.c_void_p(16)
    for p in bad:
        assert L.engram_hash(ctypes.byref(p), dummy, None, 1, 10, dummy, None) == E.ENGRAM_EINVAL
        assert L.engram_hash_gather(ctypes.byref(p), dummy, None, 1, 10, dummy, 1, None, dummy,
                                    None) == E.ENGRAM_EINVAL
    assert L.engram_hash(None, dummy, None, 1, 10, dummy, None) == E.ENGRAM_EINVAL
    p = _page_params(E)
    assert L.engram_hash(ctypes.byref(p), dummy, None, 1, -1, dummy, None) == E.ENGRAM_EINVAL
    assert L.engram_hash(ctypes.byref(p), dummy, dummy, 0, 10, dummy, None) == E.ENGRAM_EINVAL
    assert L.engram_hash(ctypes.byref(p), None, None, 1, 10, dummy, None) == E.ENGRAM_EINVAL
    # T = 0 is a no-op
    assert L.engram_hash(ctypes.byref(p), None, None, 1, 0, None, None) == E.ENGRAM_OK
    # slices: start > end, end past the row, T not a multiple of the row length
    for row_len, start, end in [(64, 10, 5), (64, 0, 65), (60, 0, 10), (-5, 0, 1)]:
        assert L.engram_hash_gather_slice(ctypes.byref(p), dummy, None, 1, 128, row_len, start,
                                          end, dummy, 1, None, dummy, None) == E.ENGRAM_EINVAL
    # an empty slice is a no-op
    assert L.engram_hash_gather_slice(ctypes.byref(p), dummy, None, 1, 128, 64, 7, 7, dummy,
                                      1, None, dummy, None) == E.ENGRAM_OK


def test_host_rejects_bad_gather_and_backward_args(E):
    L = E.lib
    al = ctypes.c_void_p(256)
    mis = ctypes.c_void_p(264)
    # row bytes not a multiple of 16, bad dtype, misaligned table or output
    assert L.engram_gather(al, 1, 100, 12, al, 5, al, None) == E.ENGRAM_EINVAL
    assert L.engram_gather(al, 7, 100, 160, al, 5, al, None) == E.ENGRAM_EINVAL
    assert L.engram_gather(mis, 1, 100, 160, al, 5, al, None) == E.ENGRAM_EINVAL
    assert L.engram_gather(al, 1, 100, 160, al, 5, mis, None) == E.ENGRAM_EINVAL
    assert L.engram_gather(al, 1, 100, 160, al, 0, al, None) == E.ENGRAM_OK
    # backward: dim must be a multiple of 8 up to 512; n below 2^31
    size = ctypes.c_size_t(0)
    assert L.engram_backward_workspace_size(10, 100, 12, ctypes.byref(size)) == E.ENGRAM_EINVAL
    assert L.engram_backward_workspace_size(10, 100, 520, ctypes.byref(size)) == E.ENGRAM_EINVAL
    assert L.engram_backward_workspace_size(2 ** 31, 100, 160,
                                            ctypes.byref(size)) == E.ENGRAM_EINVAL
    assert L.engram_backward_workspace_size(10, 0, 160, ctypes.byref(size)) == E.ENGRAM_EINVAL
    assert L.engram_backward_workspace_size(10, 100, 160, None) == E.ENGRAM_EINVAL


def test_host_rejects_bad_conv_args(E):
    L = E.lib
    al, al2, mis = ctypes.c_void_p(256), ctypes.c_void_p(1 << 30), ctypes.c_void_p(264)

    def params(**kw):
        base = dict(channels=10240, group_size=2560, kernel_size=4, dilation=3, eps=1e-6,
                    flags=7, weight_dtype=1, reserved=0)
        base.update(kw)
        return E.ConvParams(**base)

    def conv(p, x=al, dtype=1, cu=None, nseq=1, T=100, out=al2, out_dtype=1):
        return L.engram_ple_short_conv(ctypes.byref(p), x, dtype, cu, nseq, T, None, al, None,
                                       out, out_dtype, None)

    for bad in (dict(group_size=12), dict(group_size=3000), dict(channels=7680 + 100),
                dict(group_size=8192, channels=8192), dict(kernel_size=0),
                dict(kernel_size=9), dict(dilation=0), dict(eps=-1.0),
                dict(eps=float("nan")), dict(flags=8), dict(weight_dtype=5), dict(reserved=1),
                dict(kernel_size=8, dilation=4096)):
        assert conv(params(**bad)) == E.ENGRAM_EINVAL, bad
    p = params()
    assert L.engram_ple_short_conv(None, al, 1, None, 1, 100, None, al, None, al2, 1,
                                   None) == E.ENGRAM_EINVAL
    assert conv(p, dtype=7) == E.ENGRAM_EINVAL
    assert conv(p, out_dtype=2) == E.ENGRAM_EINVAL          # bf16 in, f16 out
    assert conv(p, dtype=0, out_dtype=1) == E.ENGRAM_EINVAL  # f32 in, bf16 out
    assert conv(p, T=-1) == E.ENGRAM_EINVAL
    assert conv(p, cu=al, nseq=0) == E.ENGRAM_EINVAL
    assert conv(p, x=mis) == E.ENGRAM_EINVAL
    assert conv(p, out=mis) == E.ENGRAM_EINVAL
    assert conv(p, x=None) == E.ENGRAM_EINVAL
    assert conv(p, out=ctypes.c_void_p(256 + 4096)) == E.ENGRAM_EINVAL  # overlaps x
    assert conv(p, T=0, x=None, out=None) == E.ENGRAM_OK                # empty: no-op
    # the norm alone: groups must divide the row, in place needs one dtype
    N = L.engram_grouped_rms_norm
    assert N(al, 1, 10, 100, 30, None, 0, 1e-6, al2, 1, None) == E.ENGRAM_EINVAL
    assert N(al, 1, 10, 96, 0, None, 0, 1e-6, al2, 1, None) == E.ENGRAM_EINVAL
    assert N(al, 1, 10, 96, 32, None, 0, 1e-6, al, 0, None) == E.ENGRAM_EINVAL
    assert N(al, 1, 0, 96, 32, None, 0, 1e-6, al, 1, None) == E.ENGRAM_OK


def test_host_rejects_bad_conv_backward_args(E):
    L = E.lib
    al, al2, al3 = ctypes.c_void_p(256), ctypes.c_void_p(1 << 30), ctypes.c_void_p(1 << 31)
    mis = ctypes.c_void_p(264)
    ws = ctypes.c_void_p(1 << 32)

    def params(**kw):
        base = dict(channels=10240, group_size=2560, kernel_size=4, dilation=3, eps=1e-6,
                    flags=7, weight_dtype=1, reserved=0)
        base.update(kw)
        return E.ConvParams(**base)

    def bwd(p, x=al, dtype=1, cu=None, nseq=1, T=100, dout=al2, gdt=1, dx=al3, dw=al,
            work=ws):
        return L.engram_ple_short_conv_backward(ctypes.byref(p), x, dtype, cu, nseq, T, None,
                                                al, None, dout, gdt, dx, None, dw, None, work,
                                                1 << 30, None)

    for bad in (dict(group_size=12), dict(group_size=2568, channels=2568),
                dict(channels=7680 + 100), dict(kernel_size=0), dict(kernel_size=5),
                dict(dilation=0), dict(eps=-1.0), dict(eps=float("nan")), dict(flags=8),
                dict(weight_dtype=5), dict(reserved=1)):
        assert bwd(params(**bad)) == E.ENGRAM_EINVAL, bad
    p = params()
    assert bwd(p, dtype=7) == E.ENGRAM_EINVAL
    assert bwd(p, gdt=7) == E.ENGRAM_EINVAL
    assert bwd(p, T=-1) == E.ENGRAM_EINVAL
    assert bwd(p, cu=al, nseq=0) == E.ENGRAM_EINVAL
    assert bwd(p, x=mis) == E.ENGRAM_EINVAL
    assert bwd(p, dout=mis) == E.ENGRAM_EINVAL
    assert bwd(p, dx=mis) == E.ENGRAM_EINVAL
    assert bwd(p, x=None) == E.ENGRAM_EINVAL
    assert bwd(p, dw=None) == E.ENGRAM_EINVAL
    assert bwd(p, work=None) == E.ENGRAM_EINVAL
    assert bwd(p, dx=ctypes.c_void_p((1 << 30) + 4096)) == E.ENGRAM_EINVAL  # overlaps dout
    assert bwd(p, dx=ctypes.c_void_p(256 + 4096)) == E.ENGRAM_EINVAL        # overlaps x
    assert L.engram_ple_short_conv_backward_workspace_size(
        ctypes.byref(params(kernel_size=5)), 100, ctypes.byref(ctypes.c_size_t())) == \
        E.ENGRAM_EINVAL


def test_host_rejects_bad_adam_args(E):
    L = E.lib
    a16, a8 = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 21) + 8)

    def adam(dtype=1, rows=100, dim=160, table=a16, m=a16, cap=10, **kw):
        base = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, reserved=0,
                    step=1)
        base.update(kw)
        p = E.AdamParams(**base)
        return L.engram_sparse_adam(ctypes.byref(p), table, dtype, rows, dim, m, a16, a16, a16,
                                    a16, cap, None)

    for kw in (dict(dim=6), dict(dim=0), dict(dtype=9), dict(rows=0), dict(step=0),
               dict(lr=-1.0), dict(beta1=1.0), dict(beta2=-0.1), dict(eps=-1e-8),
               dict(weight_decay=float("inf")), dict(reserved=3), dict(cap=-1),
               dict(m=a8), dict(dtype=0, table=a8)):
        assert adam(**kw) == E.ENGRAM_EINVAL, kw
    assert adam(cap=0) == E.ENGRAM_OK                            # nothing to update
    assert L.engram_sparse_adam(None, a16, 1, 100, 160, a16, a16, a16, a16, a16, 10,
                                None) == E.ENGRAM_EINVAL


def test_package_import_fails_loudly_without_library(tmp_path):
    # a copy of the binding pointed at a directory with no library must raise
    import importlib.util
    src = os.path.join(ROOT, "hashed_gram_embedding_raw_b200", "_binding.py")
    pkg = tmp_path / "fakepkg"
    pkg.mkdir()
    (pkg / "_binding.py").write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("fake_binding", pkg / "_binding.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="not found"):
        spec.loader.exec_module(mod)


def test_host_rejects_bad_owner_bucket_args(E):
    L = E.lib
    a, b, c, d, e = (ctypes.c_void_p(v << 20) for v in (1, 2, 3, 4, 5))
    ws = ctypes.c_void_p(6 << 20)
    sz = ctypes.c_size_t(0)

    def call(rows=a, n=100, rpo=10, owners=4, send=b, src=c, dst=d, counts=e, work=ws,
             nbytes=1 << 20):
        return L.engram_owner_bucket(rows, n, rpo, owners, send, src, dst, counts, work,
                                     nbytes, None)

    assert L.engram_owner_bucket_workspace_size(100, 0, ctypes.byref(sz)) == E.ENGRAM_EINVAL
    assert L.engram_owner_bucket_workspace_size(100, 257, ctypes.byref(sz)) == E.ENGRAM_EINVAL
    assert L.engram_owner_bucket_workspace_size(-1, 4, ctypes.byref(sz)) == E.ENGRAM_EINVAL
    assert L.engram_owner_bucket_workspace_size(4096, 4, ctypes.byref(sz)) == E.ENGRAM_OK
    assert sz.value == 2 * 2 * 4 * 4
    assert call(owners=0) == E.ENGRAM_EINVAL
    assert call(rpo=0) == E.ENGRAM_EINVAL
    assert call(n=-1) == E.ENGRAM_EINVAL
    assert call(counts=None) == E.ENGRAM_EINVAL
    assert call(rows=None) == E.ENGRAM_EINVAL
    assert call(work=None) == E.ENGRAM_EINVAL
    assert call(send=ctypes.c_void_p((1 << 20) + 64)) == E.ENGRAM_EINVAL   # overlaps rows
    assert call(dst=c) == E.ENGRAM_EINVAL                                  # src = dst
    assert call(nbytes=8) == E.ENGRAM_ENOSPC
