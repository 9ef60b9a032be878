"""Pins of the PLE-tail backward in the oracle (CPU only).

oracle.short_conv_backward returns the gradients of L = sum(dout * out), with
out the PLE tail x + SiLU(conv(norm(x))) of oracle.short_conv, with respect to
x, the norm scale, the convolution weights and the bias. It is pinned against
torch.autograd over the same chain written with library routines (rms_norm,
conv1d, silu, in fp64), against central finite differences of the forward
oracle (Richardson-extrapolated, on inputs whose perturbations are exact in
fp32), and against identities the chain fixes: the adjoint of the linear
convolution, the bilinear form in the weights, the impulse response of the
transposed convolution, and the norm's invariance to the scale of each
HyperConnection branch (layers page, Qwen3_8_FlashNextGroupedRMSNorm), which
makes the input gradient of every group orthogonal to the group's input.
"""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

F32 = oracle.F32


def _grid(a, step=2.0 ** -10):
    """Values on a grid of 2^-10 in fp32, so x + h v stays exact for h = 2^-8, 2^-9."""
    return (np.round(np.asarray(a, np.float64) / step) * step).astype(np.float32)


def _data(seed, T=30, C=16, K=4):
    rng = np.random.default_rng(100 + seed)
    x = _grid(rng.standard_normal((T, C)))
    w = _grid(0.5 * rng.standard_normal((C, K)))
    nw = _grid(0.3 * rng.standard_normal(C))
    b = _grid(0.2 * rng.standard_normal(C))
    dout = rng.standard_normal((T, C))
    return x, w, nw, b, dout


def _bounds(cu, T):
    return [(0, T)] if cu is None else list(zip(cu[:-1], cu[1:]))


def _torch_grads(x, w, nw, b, dout, cu, d, G, eps, norm, silu, residual):
    """The same chain through torch library routines, differentiated by autograd."""
    T, C = x.shape
    K = w.shape[1]
    xt = torch.tensor(x, dtype=torch.float64, requires_grad=True)
    wt = torch.tensor(w, dtype=torch.float64, requires_grad=True)
    nwt = torch.tensor(nw, dtype=torch.float64, requires_grad=True)
    bt = torch.tensor(b, dtype=torch.float64, requires_grad=True)
    if norm:
        n = F.rms_norm(xt.reshape(T, C // G, G), [G], eps=eps).reshape(T, C) * (1.0 + nwt)
    else:
        n = xt
    parts = []
    for s, e in _bounds(cu, T):
        if e <= s:
            continue
        y = F.conv1d(n[s:e].T[None], wt[:, None, :], bt, padding=(K - 1) * d, dilation=d,
                     groups=C)
        parts.append(y[0, :, : e - s].T)
    y = torch.cat(parts) if parts else torch.zeros((0, C), dtype=torch.float64)
    out = F.silu(y) if silu else y
    if residual:
        out = out + xt
    (out * torch.from_numpy(dout)).sum().backward()
    g = lambda t: np.zeros(t.shape) if t.grad is None else t.grad.numpy()  # noqa: E731
    return g(xt), g(nwt), g(wt), g(bt)


CASES = [
    # K, d, G, cu, norm, silu, residual
    (4, 3, 8, [0, 17, 30], True, True, True),
    (4, 3, 4, [0, 1, 1, 9, 30], True, True, True),
    (4, 3, 16, None, True, True, False),
    (3, 5, 8, [0, 12, 30], False, True, True),
    (2, 1, 4, [0, 30], True, False, True),
    (1, 1, 8, None, True, True, True),
    (8, 2, 4, [0, 3, 30], False, False, False),
]


@pytest.mark.parametrize("K,d,G,cu,norm,silu,residual", CASES)
def test_matches_torch_autograd(K, d, G, cu, norm, silu, residual):
    x, w, nw, b, dout = _data(K * 10 + d, K=K)
    got = oracle.short_conv_backward(x, F32, cu, w, dout, dilation=d, group=G, norm_w=nw,
                                     bias=b, eps=1e-6, norm=norm, silu=silu, residual=residual)
    want = _torch_grads(x, w, nw, b, dout, cu, d, G, 1e-6, norm, silu, residual)
    for name, g_, w_ in zip(("dx", "dnorm_w", "dconv_w", "dbias"), got, want):
        np.testing.assert_allclose(g_, w_, rtol=1e-11, atol=1e-11, err_msg=name)


def _loss(x, w, nw, b, dout, cu, d, G):
    out = oracle.short_conv(x, F32, cu, w, dilation=d, group=G, norm_w=nw, bias=b, eps=1e-6)
    return float((out * dout).sum())


def _fd(f, base, v):
    """<grad f, v> by central differences at h = 2^-8 and 2^-9, Richardson-combined
    (error O(h^4)); base + h v is exact in fp32 for grid values and integer v."""
    def central(h):
        return (f(base + np.float32(h) * v) - f(base - np.float32(h) * v)) / (2 * h)
    d1, d2 = central(2.0 ** -8), central(2.0 ** -9)
    return (4 * d2 - d1) / 3


@pytest.mark.parametrize("seed", range(3))
def test_finite_differences(seed):
    x, w, nw, b, dout = _data(seed, T=24, C=8)
    cu, d, G = [0, 10, 24], 3, 4
    dx, dnw, dw, db = oracle.short_conv_backward(x, F32, cu, w, dout, dilation=d, group=G,
                                                 norm_w=nw, bias=b, eps=1e-6)
    rng = np.random.default_rng(seed)
    checks = [
        (lambda t: _loss(t, w, nw, b, dout, cu, d, G), x, dx),
        (lambda t: _loss(x, t, nw, b, dout, cu, d, G), w, dw),
        (lambda t: _loss(x, w, t, b, dout, cu, d, G), nw, dnw),
        (lambda t: _loss(x, w, nw, t, dout, cu, d, G), b, db),
    ]
    for f, base, grad in checks:
        v = rng.integers(-1, 2, size=base.shape).astype(np.float32)
        fd = _fd(f, base, v)
        an = float((grad * v).sum())
        assert abs(fd - an) <= 1e-7 * (1 + abs(an)), (fd, an)
    # single entries: a tap's own weight, an input right after a sequence start
    for (t, c) in ((10, 2), (13, 5), (0, 7), (23, 0)):
        v = np.zeros_like(x)
        v[t, c] = 1.0
        fd = _fd(lambda z: _loss(z, w, nw, b, dout, cu, d, G), x, v)
        assert abs(fd - dx[t, c]) <= 1e-7 * (1 + abs(dx[t, c])), (t, c, fd, dx[t, c])


def test_linear_convolution_adjoint_and_bilinear_form():
    # norm, SiLU, residual off: out = conv_w * x + bias is linear in x and in conv_w
    x, w, _, b, dout = _data(20, T=40)
    cu = [0, 7, 7, 40]
    kw = dict(dilation=3, norm=False, silu=False, residual=False)
    dx, _, dw, db = oracle.short_conv_backward(x, F32, cu, w, dout, bias=b, **kw)
    conv = oracle.short_conv(x, F32, cu, w, bias=None, **kw)
    lhs = float((dout * conv).sum())
    np.testing.assert_allclose(float((dx * x).sum()), lhs, rtol=1e-13)
    np.testing.assert_allclose(float((dw * w).sum()), lhs, rtol=1e-13)
    np.testing.assert_allclose(db, dout.sum(0), rtol=1e-13, atol=1e-13)


def test_transposed_impulse_response():
    T, C, K, d = 30, 4, 4, 3
    w = np.arange(1, C * K + 1, dtype=np.float32).reshape(C, K)
    x = np.zeros((T, C), np.float32)
    dout = np.zeros((T, C))
    dout[20, 1] = 1.0
    cu = [0, 14, 30]
    dx, _, dw, _ = oracle.short_conv_backward(x, F32, cu, w, dout, dilation=d, norm=False,
                                              silu=False, residual=False)
    want = np.zeros((T, C))
    for k in range(K):  # output row 20 read row 20 - k d through tap K-1-k, not before 14
        if 20 - k * d >= 14:
            want[20 - k * d, 1] = w[1, K - 1 - k]
    np.testing.assert_array_equal(dx, want)
    np.testing.assert_array_equal(dw, np.zeros((C, K)))   # the input was zero


def test_norm_input_gradient_orthogonal_to_each_group():
    # with eps = 0 the norm is invariant to scaling one group of one row, so
    # d/da L(a x_g) = <dx_g, x_g> = 0 for the non-residual part
    x, w, nw, b, dout = _data(21, T=20)
    dx, _, _, _ = oracle.short_conv_backward(x, F32, [0, 20], w, dout, dilation=3, group=4,
                                             norm_w=nw, bias=b, eps=0.0, residual=False)
    dots = (dx * x).reshape(20, 4, 4).sum(-1)
    scale = np.abs(dx * x).reshape(20, 4, 4).sum(-1)
    assert (np.abs(dots) <= 1e-13 * (1 + scale)).all()
    dxr, _, _, _ = oracle.short_conv_backward(x, F32, [0, 20], w, dout, dilation=3, group=4,
                                              norm_w=nw, bias=b, eps=0.0, residual=True)
    np.testing.assert_allclose(dxr - dx, dout, rtol=1e-14, atol=1e-14)


def test_empty_and_rejects():
    w = np.ones((8, 4), np.float32)
    got = oracle.short_conv_backward(np.zeros((0, 8), np.float32), F32, [0, 0], w,
                                     np.zeros((0, 8)), dilation=3, group=4)
    assert got[0].shape == (0, 8)
    for g in got[1:]:
        assert not g.any()
    x, w, nw, b, dout = _data(22)
    with pytest.raises(ValueError):
        oracle.short_conv_backward(x, F32, [0, 10, 29], w, dout, dilation=3, group=8)
    with pytest.raises(ValueError):
        oracle.short_conv_backward(x, F32, None, w, dout, dilation=3, group=5)
