"""Parity of the sparse optimizer step (through the C ABI) with the oracle, on a B200.

engram_sparse_adam updates only the rows uniq_rows[:num_unique] (num_unique
read on the device). The kernel computes in fp32 from the stored fp32
moments and the fp32 hyperparameters of the ABI; the oracle computes in fp64
from the same values (hyperparameters rounded to fp32 first). Bar, per
element, scaled by the terms, not the result (b1 m + (1 - b1) g can cancel):
  m:  |g - o| <= 1e-6 (b1 |m0| + (1 - b1) |grad|) + 1e-12, v likewise with g^2;
  p:  |g - o| <= 1e-6 |p0| + 1e-5 lr, plus half an ulp of the table dtype
      (2^-8 |o| for bf16, 2^-11 |o| for f16) for the final rounding;
rows not listed are compared bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
HALF_ULP = {"f32": 0.0, "bf16": 2.0 ** -8, "f16": 2.0 ** -11}


@pytest.fixture(scope="module")
def E():
    import hashed_gram_embedding_raw_b200 as E
    torch.cuda.set_device(0)
    E.engram_get_device_error()
    return E


def make_state(R, D, U, cap, dt, seed):
    g = torch.Generator().manual_seed(7000 + seed)
    p = torch.randn((R, D), generator=g).to(TORCH_DT[dt])
    m = 0.01 * torch.randn((R, D), generator=g)
    v = 1e-4 * torch.rand((R, D), generator=g)
    rows = torch.randperm(R, generator=g)[:U].sort().values.to(torch.int32)
    rows_cap = torch.full((cap,), -5, dtype=torch.int32)   # entries past U must be ignored
    rows_cap[:U] = rows
    grads = torch.randn((cap, D), generator=g)
    return p, m, v, rows_cap, grads


def run(E, p, m, v, rows, grads, U, **kw):
    pd, md, vd = p.cuda(), m.cuda(), v.cuda()
    nu = torch.tensor([U], dtype=torch.int32, device="cuda")
    E.engram_sparse_adam(pd, md, vd, rows.cuda(), grads.cuda(), nu, **kw)
    torch.cuda.synchronize()
    return pd.cpu(), md.cpu(), vd.cpu()


def f32(x):
    return float(np.float32(x))


def oracle_step(p, m, v, rows, grads, lr, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.0,
                step=1):
    """The oracle with the hyperparameters the kernel sees (fp32)."""
    return oracle.sparse_adam(p, m, v, rows, grads, lr=f32(lr),
                              betas=(f32(betas[0]), f32(betas[1])), eps=f32(eps),
                              weight_decay=f32(weight_decay), step=step)


def check(p, m, v, rows, grads, U, dt, got, lr, betas=(0.9, 0.999), **kw):
    p0, m0, v0 = p.double().numpy(), m.double().numpy(), v.double().numpy()
    g0 = grads[:U].double().numpy()
    P, M, V = oracle_step(p0, m0, v0, rows[:U].numpy(), grads[:U].numpy(), lr, betas, **kw)
    gp, gm, gv = (t.double().numpy() for t in got)
    r = rows[:U].long().numpy()
    b1, b2 = betas
    scale_m = b1 * np.abs(m0[r]) + (1 - b1) * np.abs(g0)
    scale_v = b2 * np.abs(v0[r]) + (1 - b2) * g0 ** 2
    for name, g_, o_, sc in (("m", gm[r], M[r], scale_m), ("v", gv[r], V[r], scale_v)):
        err = np.abs(g_ - o_)
        assert (err <= 1e-6 * sc + 1e-12).all(), (name, err.max())
    err = np.abs(gp[r] - P[r])
    bound = 1e-6 * np.abs(p0[r]) + 1e-5 * lr + HALF_ULP[dt] * np.abs(P[r]) * (1 + 1e-3)
    assert (err <= bound).all(), ("p", err.max(), (err - bound).max())
    others = np.setdiff1d(np.arange(p.shape[0]), r)
    assert torch.equal(got[0][others], p[others])
    assert torch.equal(got[1][others], m[others]) and torch.equal(got[2][others], v[others])


@pytest.mark.parametrize("dt", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("wd,step", [(0.0, 1), (0.01, 7), (0.1, 1000)])
def test_matches_oracle(E, dt, wd, step):
    R, D, U, cap = 1000, 160, 300, 400
    p, m, v, rows, grads = make_state(R, D, U, cap, dt, seed=step)
    kw = dict(betas=(0.9, 0.999), eps=1e-8, weight_decay=wd, step=step)
    got = run(E, p, m, v, rows, grads, U, lr=1e-3, **kw)
    check(p, m, v, rows, grads, U, dt, got, 1e-3, **kw)
    assert E.engram_get_device_error() == 0


@pytest.mark.parametrize("D", [4, 8, 96, 512])
def test_other_widths(E, D):
    R, U = 257, 100
    p, m, v, rows, grads = make_state(R, D, U, U, "f32", seed=D)
    kw = dict(betas=(0.8, 0.99), eps=1e-6, weight_decay=0.0, step=3)
    got = run(E, p, m, v, rows, grads, U, lr=0.01, **kw)
    check(p, m, v, rows, grads, U, "f32", got, 0.01, **kw)


def test_zero_unique_changes_nothing(E):
    p, m, v, rows, grads = make_state(100, 160, 10, 10, "bf16", seed=1)
    got = run(E, p, m, v, rows, grads, 0, lr=0.1, step=1)
    assert torch.equal(got[0], p) and torch.equal(got[1], m) and torch.equal(got[2], v)


def test_out_of_range_row_is_flagged_and_skipped(E):
    R, D, U = 100, 160, 5
    p, m, v, rows, grads = make_state(R, D, U, U, "f32", seed=2)
    rows[2] = R          # outside the table
    got = run(E, p, m, v, rows, grads, U, lr=0.1, step=1)
    assert E.engram_get_device_error() & E.ENGRAM_DEVERR_ROW_RANGE
    keep = torch.tensor([0, 1, 3, 4])
    check(p, m, v, rows[keep], grads[keep], 4, "f32",
          tuple(t for t in got), 0.1, step=1)


def test_backward_then_step_end_to_end(E):
    """engram_hash_gather -> engram_backward -> engram_sparse_adam on the tiny
    workload, against oracle hash + backward + optimizer step."""
    from workloads import head_params, host_dout, host_table, token_stream
    cfg = head_params("tiny")
    params = E.make_params(cfg)
    ids, cu = token_stream("tiny")
    table = host_table("tiny")
    R, D = table.shape
    n = len(ids) * params.heads
    dout = host_dout("tiny", n, D, "f32")
    tab_d = torch.from_numpy(table.copy()).cuda()
    ids_d, cu_d = torch.from_numpy(ids.copy()).cuda(), torch.from_numpy(cu.copy()).cuda()
    _, idx = E.engram_hash_gather(params, ids_d, tab_d, cu_seqlens=cu_d)
    uniq, grads, nu = E.engram_backward(idx.view(-1), dout.cuda(), R)
    m = torch.zeros((R, D), device="cuda")
    v = torch.zeros((R, D), device="cuda")
    E.engram_sparse_adam(tab_d, m, v, uniq, grads, nu, lr=0.05, weight_decay=0.01, step=1)
    torch.cuda.synchronize()
    o_idx = oracle.hash_ids(ids, cu, cfg)
    o_rows, o_grads = oracle.backward(o_idx.reshape(-1), dout.numpy(), oracle.F32)
    P, M, V = oracle_step(table.astype(np.float64), np.zeros((R, D)), np.zeros((R, D)),
                          o_rows, o_grads, 0.05, weight_decay=0.01, step=1)
    np.testing.assert_allclose(tab_d.cpu().double().numpy(), P, rtol=2e-6, atol=2e-7)
    np.testing.assert_allclose(m.cpu().double().numpy(), M, rtol=1e-5, atol=1e-9)


def test_large_table_sampled(E):
    """4,194,304 x 160 bf16 table, 262,144 touched rows; 3,000 rows sampled
    against the oracle run on exactly those rows."""
    R, D, U = 1 << 22, 160, 1 << 18
    g = torch.Generator(device="cuda").manual_seed(11)
    p = torch.randn((R, D), generator=g, device="cuda").to(torch.bfloat16)
    m = 0.01 * torch.randn((R, D), generator=g, device="cuda")
    v = 1e-4 * torch.rand((R, D), generator=g, device="cuda")
    rows = torch.randperm(R, generator=g, device="cuda")[:U].sort().values.to(torch.int32)
    grads = torch.randn((U, D), generator=g, device="cuda")
    pick = torch.randperm(U, generator=g, device="cuda")[:3000].sort().values
    prow = rows[pick].long()
    p0, m0, v0 = p[prow].cpu(), m[prow].cpu(), v[prow].cpu()
    untouched = torch.tensor([0, 1, R - 1], device="cuda")
    untouched = untouched[~torch.isin(untouched, rows.long())]
    pu = p[untouched].clone()
    nu = torch.tensor([U], dtype=torch.int32, device="cuda")
    kw = dict(betas=(0.9, 0.999), eps=1e-8, weight_decay=0.01, step=5)
    E.engram_sparse_adam(p, m, v, rows, grads, nu, lr=1e-3, **kw)
    torch.cuda.synchronize()
    local = torch.arange(3000, dtype=torch.int32)
    P, M, V = oracle_step(p0.double().numpy(), m0.double().numpy(), v0.double().numpy(),
                          local.numpy(), grads[pick].cpu().numpy(), 1e-3, **kw)
    gp = p[prow].cpu().double().numpy()
    err = np.abs(gp - P)
    bound = 1e-6 * np.abs(p0.double().numpy()) + 1e-8 + 2.0 ** -8 * np.abs(P) * 1.001
    assert (err <= bound).all()
    scale = 0.9 * np.abs(m0.double().numpy()) + 0.1 * np.abs(grads[pick].cpu().double().numpy())
    assert (np.abs(m[prow].cpu().double().numpy() - M) <= 1e-6 * scale + 1e-12).all()
    assert torch.equal(p[untouched], pu)
