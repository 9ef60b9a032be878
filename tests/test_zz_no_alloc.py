"""engram_backward_noalloc against engram_backward, on a GPU.

engram_backward_noalloc serves callers that cannot allocate device memory
(a plugin inside an application that owns all device memory and offers no
workspace, or a path that must not call cudaMalloc because it can synchronise
the device). It keeps its scratch in one fixed array inside the library, so
these tests call it through the C ABI twice in a row -- the second call
starts from whatever the first left in that array -- and compare each result
with the workspace-based entry point on the same input and with the CPU
oracle, within the tolerance the other backward tests use. This file is
collected last so that a run stopping at the first failure has run every
other test already.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

RTOL, ATOL = 1e-5, 1e-6


@pytest.fixture(scope="module")
def E():
    import hashed_gram_embedding_raw_b200 as E
    torch.cuda.set_device(0)
    E.engram_get_device_error()
    return E


def _case(seed, n, rows, dim, dtype):
    g = torch.Generator().manual_seed(seed)
    # a mix of hot and cold rows, so some segments cross warp ranges
    hot = torch.randint(0, 7, (n,), generator=g)
    cold = torch.randint(0, rows, (n,), generator=g)
    idx = torch.where(torch.rand(n, generator=g) < 0.2, hot, cold).to(torch.int32).cuda()
    dout = torch.randn(n, dim, generator=g).to(dtype).cuda()
    return idx, dout


def _noalloc_via_abi(E, idx, dout, rows):
    n, dim = idx.numel(), dout.shape[-1]
    uniq = torch.full((n,), -1, dtype=torch.int32, device="cuda")
    grads = torch.full((n, dim), float("nan"), dtype=torch.float32, device="cuda")
    nu = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    code = {torch.float32: E.ENGRAM_F32, torch.bfloat16: E.ENGRAM_BF16,
            torch.float16: E.ENGRAM_F16}[dout.dtype]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = E.lib.engram_backward_noalloc(
        ctypes.c_void_p(idx.data_ptr()), n, rows, dim, ctypes.c_void_p(dout.data_ptr()), code,
        ctypes.c_void_p(uniq.data_ptr()), ctypes.c_void_p(grads.data_ptr()),
        ctypes.c_void_p(nu.data_ptr()), stream)
    assert rc == E.ENGRAM_OK, E.status_string(rc)
    return uniq, grads, nu


def _close(got, want):
    err = (got.double() - want.double()).abs()
    return bool((err <= ATOL + RTOL * want.double().abs()).all())


def _compare(E, idx, dout, rows):
    ref_u, ref_g, ref_nu = E.engram_backward(idx, dout, rows)
    u, g, nu = _noalloc_via_abi(E, idx, dout, rows)
    torch.cuda.synchronize()
    U = int(ref_nu.item())
    assert int(nu.item()) == U
    assert torch.equal(u[:U], ref_u[:U])
    assert _close(g[:U], ref_g[:U])
    assert E.engram_get_device_error() == 0
    # and against the oracle
    d = dout.cpu()
    raw = d.numpy() if d.dtype == torch.float32 else \
        d.view(torch.int16).numpy().view(np.uint16)
    code = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16,
            torch.float16: oracle.F16}[d.dtype]
    want_u, want_g = oracle.backward(idx.cpu().numpy(), raw, code)
    assert len(want_u) == U
    np.testing.assert_array_equal(u[:U].cpu().numpy(), want_u)
    assert _close(g[:U].cpu(), torch.from_numpy(want_g))


def test_noalloc_two_calls_in_a_row_match_workspace_entry(E):
    # first call: page-sized rows (bf16, 160 wide) on a 320,001,536-row table
    idx, dout = _case(1, 200_003, 320_001_536, 160, torch.bfloat16)
    _compare(E, idx, dout, 320_001_536)
    # second call, different shape and dtype, on top of the first's leftovers
    idx, dout = _case(2, 70_001, 5_000, 96, torch.float32)
    _compare(E, idx, dout, 5_000)


def test_noalloc_wide_rows_small_batch(E):
    # 512-wide rows: the scratch the reduction needs grows with the lookups,
    # so a small batch fits the array
    idx, dout = _case(3, 5_000, 70_000, 512, torch.bfloat16)
    _compare(E, idx, dout, 70_000)
    idx, dout = _case(4, 1, 10, 512, torch.float32)
    _compare(E, idx, dout, 10)


def test_noalloc_rejects_sizes_beyond_its_array(E):
    n, rows, dim = 4_000_000, 320_001_536, 160
    assert E.engram_backward_workspace_size(n, rows, dim) > E.ENGRAM_NOALLOC_SCRATCH_BYTES
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    dummy = ctypes.c_void_p(256)
    rc = E.lib.engram_backward_noalloc(dummy, n, rows, dim, dummy, E.ENGRAM_BF16, dummy,
                                       dummy, dummy, stream)
    assert rc == E.ENGRAM_ENOSPC
