"""Pins of the PLE-layer oracle (grouped RMS norm + causal short convolution).

CPU only. The oracle functions are checked against library routines the
operations reduce to (torch.nn.functional.rms_norm, conv1d, silu, all in
fp64), against closed forms (constant rows, impulse responses) and against
properties the pages fix: the convolution is causal with zero history before a
sequence start (engram page, Qwen3_8_FlashNextPLELayer._causal_short_conv),
the norm is local to each HyperConnection branch (layers page,
Qwen3_8_FlashNextGroupedRMSNorm), and a zero-start convolution
(Qwen3_8_FlashNextPLELayer.init_weights) leaves only the residual.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

F32 = oracle.F32


def _data(seed, T=40, C=16, K=4):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, C)).astype(np.float32)
    w = (0.5 * rng.standard_normal((C, K))).astype(np.float32)
    nw = (0.3 * rng.standard_normal(C)).astype(np.float32)
    b = (0.2 * rng.standard_normal(C)).astype(np.float32)
    return x, w, nw, b


def _bounds(cu, T):
    return [(0, T)] if cu is None else list(zip(cu[:-1], cu[1:]))


# ------------------------------------------------------------------- norm

@pytest.mark.parametrize("G", [4, 8, 16])
def test_norm_matches_torch_rms_norm(G):
    x, _, nw, _ = _data(1)
    got = oracle.grouped_rms_norm(x, F32, G, nw, eps=1e-6)
    xt = torch.from_numpy(x).double().reshape(x.shape[0], -1, G)
    ref = F.rms_norm(xt, [G], eps=1e-6).reshape(x.shape) * (1.0 + torch.from_numpy(nw).double())
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-13, atol=1e-13)


def test_norm_constant_group_closed_form():
    # a group holding one value a everywhere normalises to a / sqrt(a^2 + eps)
    x = np.full((3, 8), 1.0, dtype=np.float32)
    x[1] = -2.0
    x[2, 4:] = 0.25
    got = oracle.grouped_rms_norm(x, F32, 4, None, eps=0.5)
    for a, row in ((1.0, 0), (-2.0, 1), (0.25, 2)):
        want = a / np.sqrt(a * a + 0.5)
        cols = slice(4, 8) if row == 2 else slice(0, 8)
        np.testing.assert_allclose(got[row, cols], want, rtol=1e-15)


def test_norm_unit_rms_and_branch_scale_invariance():
    x, _, _, _ = _data(2)
    n0 = oracle.grouped_rms_norm(x, F32, 4, None, eps=0.0)
    np.testing.assert_allclose((n0.reshape(40, 4, 4) ** 2).mean(-1), 1.0, rtol=1e-13)
    # scaling one branch of one row by a power of two changes nothing anywhere
    xs = x.copy()
    xs[5, 4:8] *= 8.0
    xs[9, 12:16] *= 0.125
    n1 = oracle.grouped_rms_norm(xs, F32, 4, None, eps=0.0)
    np.testing.assert_allclose(n1, n0, rtol=1e-14, atol=1e-15)


def test_norm_zero_scale_is_plain_rms_norm():
    x, _, _, _ = _data(3)
    a = oracle.grouped_rms_norm(x, F32, 8, np.zeros(16, np.float32), eps=1e-6)
    b = oracle.grouped_rms_norm(x, F32, 8, None, eps=1e-6)
    np.testing.assert_array_equal(a, b)
    ref = F.rms_norm(torch.from_numpy(x).double().reshape(40, 2, 8), [8], eps=1e-6)
    np.testing.assert_allclose(a, ref.reshape(40, 16).numpy(), rtol=1e-13)


# ------------------------------------------------------------ convolution

def _torch_conv(x, w, b, cu, d):
    """Depthwise causal conv per sequence through torch's conv1d (fp64)."""
    T, C = x.shape
    K = w.shape[1]
    out = np.zeros((T, C))
    wt = torch.from_numpy(w).double()[:, None, :]
    bt = None if b is None else torch.from_numpy(b).double()
    for s, e in _bounds(cu, T):
        if e <= s:
            continue
        seg = torch.from_numpy(x[s:e]).double().T[None]
        y = F.conv1d(seg, wt, bt, padding=(K - 1) * d, dilation=d, groups=C)
        out[s:e] = y[0, :, : e - s].T.numpy()
    return out


@pytest.mark.parametrize("K,d", [(4, 3), (1, 1), (2, 1), (3, 5), (8, 2)])
@pytest.mark.parametrize("cu", [None, [0, 13, 13, 40], [0, 1, 2, 3, 40]])
def test_conv_matches_torch_conv1d(K, d, cu):
    x, w, _, b = _data(4 + K + d, K=K)
    got = oracle.short_conv(x, F32, cu, w, dilation=d, bias=b, norm=False, silu=False,
                            residual=False)
    np.testing.assert_allclose(got, _torch_conv(x, w, b, cu, d), rtol=1e-12, atol=1e-12)


def test_conv_impulse_response():
    T, C, K, d = 30, 4, 4, 3
    w = np.arange(1, C * K + 1, dtype=np.float32).reshape(C, K)
    x = np.zeros((T, C), np.float32)
    x[7, 2] = 1.0
    got = oracle.short_conv(x, F32, None, w, dilation=d, norm=False, silu=False, residual=False)
    want = np.zeros((T, C))
    for k in range(K):  # the token k*d after the impulse sees it through tap K-1-k
        want[7 + k * d, 2] = w[2, K - 1 - k]
    np.testing.assert_array_equal(got, want)


def test_silu_and_residual_match_torch():
    x, _, _, _ = _data(5)
    one = np.ones((16, 1), np.float32)
    xt = torch.from_numpy(x).double()
    s = oracle.short_conv(x, F32, None, one, dilation=1, norm=False, silu=True, residual=False)
    np.testing.assert_allclose(s, F.silu(xt).numpy(), rtol=1e-14, atol=1e-15)
    r = oracle.short_conv(x, F32, None, one, dilation=1, norm=False, silu=True, residual=True)
    np.testing.assert_allclose(r, (F.silu(xt) + xt).numpy(), rtol=1e-14, atol=1e-15)


def test_full_tail_matches_torch_chain():
    x, w, nw, b = _data(6)
    cu = [0, 17, 40]
    got = oracle.short_conv(x, F32, cu, w, dilation=3, group=8, norm_w=nw, bias=b, eps=1e-6)
    n = F.rms_norm(torch.from_numpy(x).double().reshape(40, 2, 8), [8], eps=1e-6)
    n = (n.reshape(40, 16) * (1.0 + torch.from_numpy(nw).double())).numpy()
    y = torch.from_numpy(_torch_conv(n, w, b, cu, 3))
    want = (F.silu(y) + torch.from_numpy(x).double()).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_zero_start_convolution_leaves_the_residual():
    x, _, nw, _ = _data(7)
    got = oracle.short_conv(x, F32, [0, 9, 40], np.zeros((16, 4), np.float32), dilation=3,
                            group=4, norm_w=nw)
    np.testing.assert_array_equal(got, x.astype(np.float64))


def test_causal_branch_local_and_sequence_local():
    x, w, nw, b = _data(8)
    cu = [0, 20, 40]
    base = oracle.short_conv(x, F32, cu, w, dilation=3, group=4, norm_w=nw, bias=b)
    for t0, c0 in ((5, 1), (18, 9), (20, 14), (39, 3)):
        xp = x.copy()
        xp[t0, c0] += 1.0
        got = oracle.short_conv(xp, F32, cu, w, dilation=3, group=4, norm_w=nw, bias=b)
        seq_end = 20 if t0 < 20 else 40
        g0 = c0 // 4 * 4
        may = np.zeros_like(got, dtype=bool)
        for k in range(4):
            if t0 + 3 * k < seq_end:
                may[t0 + 3 * k, g0:g0 + 4] = True
        np.testing.assert_array_equal(got[~may], base[~may])
        assert np.all(got[t0, g0:g0 + 4] != base[t0, g0:g0 + 4])


def test_sequences_are_independent():
    x, w, nw, b = _data(9)
    cu = [0, 11, 11, 26, 40]
    whole = oracle.short_conv(x, F32, cu, w, dilation=3, group=8, norm_w=nw, bias=b)
    for s, e in _bounds(cu, 40):
        if e > s:
            part = oracle.short_conv(x[s:e], F32, None, w, dilation=3, group=8, norm_w=nw,
                                     bias=b)
            np.testing.assert_array_equal(whole[s:e], part)


def test_bf16_input_and_weights_decode():
    # values exactly representable in bf16 give the fp32 result bit for bit
    x, w, nw, b = _data(10)

    def bf(a):
        return (np.ascontiguousarray(a, np.float32).view(np.uint32) >> 16).astype(np.uint16)

    def unbf(u):
        return (u.astype(np.uint32) << 16).view(np.float32)

    xb, wb, nwb, bb = bf(x), bf(w), bf(nw), bf(b)
    got = oracle.short_conv(xb, oracle.BF16, None, wb, dilation=3, group=8, norm_w=nwb,
                            bias=bb, wdtype=oracle.BF16)
    ref = oracle.short_conv(unbf(xb), F32, None, unbf(wb), dilation=3, group=8,
                            norm_w=unbf(nwb), bias=unbf(bb))
    np.testing.assert_array_equal(got, ref)


def test_rejects_bad_arguments():
    x, w, _, _ = _data(11)
    with pytest.raises(ValueError):
        oracle.short_conv(x, F32, [0, 20, 39], w, dilation=3, group=8)
    with pytest.raises(ValueError):
        oracle.short_conv(x, F32, None, w, dilation=0, group=8)
    with pytest.raises(ValueError):
        oracle.grouped_rms_norm(x, F32, 5)
