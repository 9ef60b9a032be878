"""Pins of the sparse optimizer-step oracle (lazy AdamW on the touched rows).

CPU only. The pages name no optimizer formula (the owner updates each row's
gradient and the table carries optimizer tensors, model card). The oracle's
reading, AdamW updated only on the rows a backward produced with a global
step count, is pinned against library routines it reduces to:
  - torch.optim.AdamW (fp64) when every row is present at every step;
  - torch.optim.SparseAdam (fp64) over steps touching different row sets, with
    eps = 1e-30, where SparseAdam's and AdamW's placements of eps (after or
    before the bias correction of v) agree to far below the tolerance;
plus the first-step closed form and untouched rows left bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle


def _state(seed, R=12, D=8):
    rng = np.random.default_rng(seed)
    p = rng.standard_normal((R, D))
    return p, np.zeros((R, D)), np.zeros((R, D)), rng


def test_first_step_closed_form():
    # m = (1-b1) g, v = (1-b2) g^2, so the bias-corrected step is -lr g / (|g| + eps)
    p, m, v, rng = _state(0)
    rows = np.array([1, 4, 7])
    g = rng.standard_normal((3, 8)).astype(np.float32)
    lr, eps = 0.01, 1e-3
    P, M, V = oracle.sparse_adam(p, m, v, rows, g, lr=lr, eps=eps)
    g64 = g.astype(np.float64)
    np.testing.assert_allclose(M[rows], 0.1 * g64, rtol=1e-13)
    np.testing.assert_allclose(V[rows], 0.001 * g64 ** 2, rtol=1e-13)
    np.testing.assert_allclose(P[rows], p[rows] - lr * g64 / (np.abs(g64) + eps), rtol=1e-13,
                               atol=1e-15)


def test_untouched_rows_keep_everything():
    p, m, v, rng = _state(1)
    m += rng.standard_normal(m.shape)
    v += rng.random(v.shape)
    rows = np.array([0, 5, 11])
    g = rng.standard_normal((3, 8)).astype(np.float32)
    P, M, V = oracle.sparse_adam(p, m, v, rows, g, lr=0.05, weight_decay=0.1, step=4)
    others = np.setdiff1d(np.arange(12), rows)
    for new, old in ((P, p), (M, m), (V, v)):
        np.testing.assert_array_equal(new[others], old[others])
    P0, M0, V0 = oracle.sparse_adam(p, m, v, np.zeros(0, np.int64),
                                    np.zeros((0, 8), np.float32), lr=0.05, step=4)
    np.testing.assert_array_equal(P0, p)


@pytest.mark.parametrize("wd", [0.0, 0.05])
def test_matches_torch_adamw_when_all_rows_present(wd):
    p, m, v, rng = _state(2)
    lr, betas, eps = 0.02, (0.85, 0.995), 1e-6
    tp = torch.nn.Parameter(torch.from_numpy(p.copy()))
    opt = torch.optim.AdamW([tp], lr=lr, betas=betas, eps=eps, weight_decay=wd)
    rows = np.arange(12)
    for step in range(1, 5):
        g = rng.standard_normal((12, 8)).astype(np.float32)
        tp.grad = torch.from_numpy(g.astype(np.float64))
        opt.step()
        p, m, v = oracle.sparse_adam(p, m, v, rows, g, lr=lr, betas=betas, eps=eps,
                                     weight_decay=wd, step=step)
        st = opt.state[tp]
        np.testing.assert_allclose(p, tp.detach().numpy(), rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-12, atol=1e-15)


def test_matches_torch_sparse_adam_over_changing_rows():
    p, m, v, rng = _state(3)
    lr, betas = 0.03, (0.9, 0.99)
    tp = torch.nn.Parameter(torch.from_numpy(p.copy()))
    opt = torch.optim.SparseAdam([tp], lr=lr, betas=betas, eps=1e-30)
    for step, rows in enumerate(([0, 3, 4], [3, 9], [1, 3, 4, 10, 11], [9]), start=1):
        rows = np.array(rows)
        g = rng.standard_normal((len(rows), 8)).astype(np.float32)
        tp.grad = torch.sparse_coo_tensor(torch.from_numpy(rows)[None],
                                          torch.from_numpy(g.astype(np.float64)), (12, 8))
        opt.step()
        p, m, v = oracle.sparse_adam(p, m, v, rows, g, lr=lr, betas=betas, eps=1e-30,
                                     step=step)
        np.testing.assert_allclose(p, tp.detach().numpy(), rtol=1e-12, atol=1e-14)
        st = opt.state[tp]
        np.testing.assert_allclose(m, st["exp_avg"].to_dense().numpy(), rtol=1e-12,
                                   atol=1e-15)
        np.testing.assert_allclose(v, st["exp_avg_sq"].to_dense().numpy(), rtol=1e-12,
                                   atol=1e-15)


def test_rejects_bad_arguments():
    p, m, v, _ = _state(4)
    g = np.zeros((1, 8), np.float32)
    with pytest.raises(ValueError):
        oracle.sparse_adam(p, m, v, [12], g, lr=0.1)
    with pytest.raises(ValueError):
        oracle.sparse_adam(p, m, v, [0], g, lr=0.1, step=0)
