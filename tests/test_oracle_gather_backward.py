"""Pins of the oracle gather and backward (CPU only).

Gather: `_lookup_ngram_ids` on a single-rank table is plain row indexing;
pinned bit for bit against NumPy fancy indexing (a library routine).

Backward: the owner-side row-gradient accumulation of the page's
OwnerShardedEmbedding. Pinned by
  * a library routine: np.add.at into an fp64 dense table, then the non-zero
    rows in ascending order (same summation order, so exact after rounding);
  * the adjoint identity <gather(W), dY> = <W, scatter(dY)> in fp64;
  * per-head mass: the sum of row gradients over head h's slice equals the
    sum of dout over head h's lookups;
  * counts: with dout = 1 every gradient is the row's multiplicity, summing
    to the number of lookups.
"""

import numpy as np
import pytest
import torch

import oracle
from workloads import head_params, host_dout, host_table, token_stream


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def test_gather_matches_fancy_indexing_fp32_and_bf16():
    p = head_params("tiny")
    tab = host_table("tiny")
    ids, cu = token_stream("tiny")
    idx = oracle.hash_ids(ids, cu, p).reshape(-1)
    out = oracle.gather(tab, idx)
    assert out.tobytes() == tab[idx].tobytes()
    tab16 = bf16_bits(torch.from_numpy(tab).to(torch.bfloat16))
    out16 = oracle.gather(tab16, idx)
    assert out16.tobytes() == tab16[idx].tobytes()


def test_gather_rejects_out_of_range():
    tab = np.zeros((10, 4), np.float32)
    with pytest.raises(IndexError):
        oracle.gather(tab, np.array([3, 10]))
    with pytest.raises(IndexError):
        oracle.gather(tab, np.array([-1]))


def _dense_scatter_fp64(idx, dout64, rows):
    dense = np.zeros((rows, dout64.shape[1]), np.float64)
    np.add.at(dense, idx, dout64)
    hit = np.zeros(rows, bool)
    hit[idx] = True
    return np.nonzero(hit)[0], dense[hit]


@pytest.mark.parametrize("seed", range(4))
def test_backward_matches_add_at(seed):
    rng = np.random.Generator(np.random.PCG64(seed))
    rows, n, D = 300, 2000, 24
    # skewed rows: some hot rows, many cold ones
    idx = np.where(rng.random(n) < 0.3, rng.integers(0, 5, n), rng.integers(0, rows, n))
    dout = rng.standard_normal((n, D)).astype(np.float32)
    uniq, grads = oracle.backward(idx, dout, oracle.F32)
    want_rows, want = _dense_scatter_fp64(idx, dout.astype(np.float64), rows)
    np.testing.assert_array_equal(uniq, want_rows)
    np.testing.assert_array_equal(grads, want.astype(np.float32))


def test_backward_bf16_and_f16_decode():
    rng = np.random.Generator(np.random.PCG64(5))
    n, D = 500, 16
    idx = rng.integers(0, 40, n)
    vals = torch.from_numpy(rng.standard_normal((n, D)).astype(np.float32))
    vals[0, :4] = torch.tensor([6.1e-5, -3.0e-7, 65504.0, 0.0])  # f16 subnormal/max
    for dt, code in [(torch.bfloat16, oracle.BF16), (torch.float16, oracle.F16)]:
        q = vals.to(dt)
        uniq, grads = oracle.backward(idx, bf16_bits(q), code)
        want_rows, want = _dense_scatter_fp64(idx, q.double().numpy(), 40)
        np.testing.assert_array_equal(uniq, want_rows)
        np.testing.assert_array_equal(grads, want.astype(np.float32))


def test_backward_adjoint_identity():
    p = head_params("tiny")
    ids, cu = token_stream("tiny")
    idx = oracle.hash_ids(ids, cu, p).reshape(-1)
    rng = np.random.Generator(np.random.PCG64(7))
    W = rng.standard_normal((p["table_rows"], p["dim"]))
    dY = rng.standard_normal((idx.shape[0], p["dim"])).astype(np.float32)
    lhs = float(np.sum(oracle.gather(W, idx) * dY.astype(np.float64)))
    uniq, grads = oracle.backward(idx, dY, oracle.F32)
    rhs = float(np.sum(W[uniq] * grads.astype(np.float64)))
    # grads are fp32 roundings of exact fp64 sums: relative error <= 2**-24 each
    bound = np.sum(np.abs(W[uniq]) * np.abs(grads)) * 2.0 ** -23
    assert abs(lhs - rhs) <= bound


@pytest.mark.parametrize("name", ["tiny", "b4x4096"])
def test_backward_per_head_mass_and_counts(name):
    p = head_params(name)
    ids, cu = token_stream(name)
    if name != "tiny":
        ids, cu = ids[:2048], np.array([0, 2048], np.int32)
    idx = oracle.hash_ids(ids, cu, p)
    T, H = idx.shape
    D = 8
    dout = host_dout(name, T * H, D, "f32").numpy()
    uniq, grads = oracle.backward(idx.reshape(-1), dout, oracle.F32)
    assert np.all(np.diff(uniq) > 0)
    per_lookup = dout.reshape(T, H, D).astype(np.float64)
    for h in range(H):
        lo, hi = p["offsets"][h], p["offsets"][h] + p["vocab_sizes"][h]
        sel = (uniq >= lo) & (uniq < hi)
        got = grads[sel].astype(np.float64).sum(0)
        want = per_lookup[:, h].sum(0)
        tol = 1e-6 * (np.abs(per_lookup[:, h]).sum(0) + 1)
        assert np.all(np.abs(got - want) <= tol)
    ones = np.ones((T * H, 1), np.float32)
    u2, counts = oracle.backward(idx.reshape(-1), ones, oracle.F32)
    np.testing.assert_array_equal(u2, uniq)
    assert counts.sum() == T * H and counts.min() >= 1
    # brute-force multiplicity of a few rows
    flat = idx.reshape(-1)
    for r in uniq[:: max(1, len(uniq) // 17)]:
        assert counts[np.searchsorted(uniq, r), 0] == np.count_nonzero(flat == r)


def test_backward_empty_and_single():
    u, g = oracle.backward(np.zeros(0, np.int64), np.zeros((0, 4), np.float32), oracle.F32)
    assert u.shape == (0,) and g.shape == (0, 4)
    u, g = oracle.backward(np.array([7]), np.full((1, 4), 2.5, np.float32), oracle.F32)
    assert u.tolist() == [7] and g.tolist() == [[2.5] * 4]
