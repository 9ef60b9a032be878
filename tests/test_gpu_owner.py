"""Owner-sharded table on a B200 (hashed_gram_embedding_raw_b200.owner with the
library's kernels).

engram_owner_bucket is checked against a stable argsort by owner (exact:
grouped rows, positions, counts), including an empty input, ragged tiles and
rows no owner holds. The routing then runs as 1, 2, 4 and 8 owner ranks
emulated on one GPU (the all-to-alls become device copies): on the tiny
workload every rank's output must equal the oracle's lookup in the whole table
bit for bit and every owner's row gradients the oracle's backward over all
ranks' lookups restricted to its rows; on b4x4096 (a 16.8M-row bf16 table)
the outputs must equal engram_hash_gather on the unsharded table and the
owners' gradients engram_backward over the concatenated lookups. A real NCCL
process group of one rank runs the same routing through all_to_all_single.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from workloads import fill_device_table, head_params, host_dout, host_table, token_stream

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    import hashed_gram_embedding_raw_b200 as E
    torch.cuda.set_device(0)
    E.engram_get_device_error()
    return E


def stable_bucket(rows, rpo, owners):
    r = rows.astype(np.int64)
    o = np.where(r < 0, owners - 1, np.minimum(r // rpo, owners - 1))
    bad = (r < 0) | (r // rpo >= owners)
    order = np.argsort(o, kind="stable")
    local = np.where(bad, -1, r - o * rpo)[order]
    dst = np.empty_like(order)
    dst[order] = np.arange(len(order))
    return local, order, dst, np.bincount(o, minlength=owners)


@pytest.mark.parametrize("n,owners,rpo", [(0, 4, 10), (1, 1, 5), (2047, 3, 1000),
                                          (2048, 8, 512), (2049, 8, 700),
                                          (100_000, 256, 400), (300_000, 8, 40_000_192)])
def test_bucket_matches_stable_argsort(E, n, owners, rpo):
    rng = np.random.default_rng(n + owners)
    rows = rng.integers(0, owners * rpo, size=n).astype(np.int32)
    if n > 10:
        rows[:5] = rows[5]            # runs of one row
    send, src, dst, counts = E.engram_owner_bucket(torch.from_numpy(rows).cuda(), rpo, owners)
    torch.cuda.synchronize()
    want = stable_bucket(rows, rpo, owners)
    assert np.array_equal(send.cpu().numpy(), want[0])
    assert np.array_equal(src.cpu().numpy(), want[1])
    assert np.array_equal(dst.cpu().numpy(), want[2])
    assert np.array_equal(counts.cpu().numpy(), want[3])
    assert E.engram_get_device_error() == 0


def test_bucket_flags_rows_no_owner_holds(E):
    rows = np.array([5, -3, 40, 39, 0, 41, 17], dtype=np.int32)
    send, src, dst, counts = E.engram_owner_bucket(torch.from_numpy(rows).cuda(), 10, 4)
    torch.cuda.synchronize()
    assert E.engram_get_device_error() & E.ENGRAM_DEVERR_ROW_RANGE
    want = stable_bucket(rows, 10, 4)
    assert np.array_equal(send.cpu().numpy(), want[0])
    assert np.array_equal(counts.cpu().numpy(), want[3])


def split(ids, W):
    T = len(ids) // W
    return [(torch.from_numpy(ids[r * T:(r + 1) * T].copy()).cuda(),
             torch.tensor([0, T], dtype=torch.int32, device="cuda")) for r in range(W)]


def run_group(E, params, table, W, parts, douts):
    from hashed_gram_embedding_raw_b200 import owner
    rpo = params.table_rows // W
    shards = [table[r * rpo:(r + 1) * rpo] for r in range(W)]
    fwd = owner.run_lockstep([owner.forward_steps(params, shards[r], W, *parts[r])
                              for r in range(W)])
    bwd = owner.run_lockstep([owner.backward_steps(params, W, fwd[r][1], douts[r])
                              for r in range(W)])
    torch.cuda.synchronize()
    return fwd, bwd


@pytest.mark.parametrize("W", [1, 2, 4, 8])
def test_emulated_group_tiny_vs_oracle(E, W):
    cfg = head_params("tiny")
    params = E.make_params(cfg)
    table_h = host_table("tiny")
    ids, _ = token_stream("tiny")
    parts = split(ids, W)
    H, D = params.heads, cfg["dim"]
    douts = [host_dout("tiny", len(p[0]) * H, D, "f32", seed_offset=r) for r, p in
             enumerate(parts)]
    fwd, bwd = run_group(E, params, torch.from_numpy(table_h).cuda(), W, parts,
                         [d.cuda() for d in douts])
    rpo = cfg["table_rows"] // W
    all_idx = []
    for r, (ids_r, cu_r) in enumerate(parts):
        idx = oracle.hash_ids(ids_r.cpu().numpy(), cu_r.cpu().numpy(), cfg)
        want = oracle.gather(table_h, idx).reshape(len(ids_r), -1)
        assert np.array_equal(fwd[r][0].cpu().numpy(), want)
        all_idx.append(idx.reshape(-1))
    idx = np.concatenate(all_idx)
    dout = np.concatenate([d.numpy() for d in douts])
    for r in range(W):
        keep = (idx // rpo) == r
        u, g = oracle.backward(idx[keep] - r * rpo, dout[keep], oracle.F32)
        gu, gg, gn = bwd[r]
        U = int(gn.item())
        assert U == len(u)
        assert np.array_equal(gu[:U].cpu().numpy(), u)
        np.testing.assert_allclose(gg[:U].cpu().numpy(), g, rtol=1e-5, atol=1e-6)
    assert E.engram_get_device_error() == 0


@pytest.mark.parametrize("name,W", [("b4x4096", 2), ("b4x4096", 8), ("thd64k", 8)])
def test_emulated_group_vs_unsharded(E, name, W):
    # thd64k: Zipf IDs, so hot rows load some owners far more than others
    cfg = head_params(name)
    params = E.make_params(cfg)
    R, D, H = cfg["table_rows"], cfg["dim"], params.heads
    table = torch.empty((R, D), dtype=torch.bfloat16, device="cuda")
    fill_device_table(table, 1)
    ids, _ = token_stream(name)
    parts = split(ids, W)
    douts = [host_dout(name, len(p[0]) * H, D, "bf16", seed_offset=r).cuda()
             for r, p in enumerate(parts)]
    fwd, bwd = run_group(E, params, table, W, parts, douts)
    idx_all = []
    counts = []
    for r, (ids_r, cu_r) in enumerate(parts):
        out, idx = E.engram_hash_gather(params, ids_r, table, cu_seqlens=cu_r)
        assert torch.equal(fwd[r][0], out)
        idx_all.append(idx.view(-1))
        counts.append(fwd[r][1].send_counts)
    idx = torch.cat(idx_all)
    dout = torch.cat(douts)
    u, g, nu = E.engram_backward(idx, dout, R)
    torch.cuda.synchronize()
    U = int(nu.item())
    u, g = u[:U].long(), g[:U]
    rpo = R // W
    for r in range(W):
        keep = (u // rpo) == r
        gu, gg, gn = bwd[r]
        Ur = int(gn.item())
        assert Ur == int(keep.sum())
        assert torch.equal(gu[:Ur].long(), u[keep] - r * rpo)
        torch.testing.assert_close(gg[:Ur], g[keep], rtol=1e-6, atol=1e-6)
    assert E.engram_get_device_error() == 0
    per_owner = np.asarray(counts).sum(0)
    assert per_owner.sum() == idx.numel()
    if name == "thd64k":
        assert per_owner.max() > 1.5 * per_owner.min()   # the splits really are uneven


def test_nccl_group_of_one(E):
    import torch.distributed as dist
    from hashed_gram_embedding_raw_b200 import owner
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True, timeout=datetime.timedelta(seconds=60))
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        cfg = head_params("tiny")
        params = E.make_params(cfg)
        table = torch.from_numpy(host_table("tiny")).cuda()
        ids, cu = token_stream("tiny")
        ids_d, cu_d = torch.from_numpy(ids.copy()).cuda(), torch.from_numpy(cu.copy()).cuda()
        dout = host_dout("tiny", len(ids) * params.heads, cfg["dim"], "f32").cuda()
        out, routing = owner.run_collective(owner.forward_steps(params, table, 1, ids_d, cu_d))
        u, g, nu = owner.run_collective(owner.backward_steps(params, 1, routing, dout))
        want_out, idx = E.engram_hash_gather(params, ids_d, table, cu_seqlens=cu_d)
        wu, wg, wn = E.engram_backward(idx.view(-1), dout, cfg["table_rows"])
        torch.cuda.synchronize()
        assert torch.equal(out, want_out)
        U = int(nu.item())
        assert U == int(wn.item())
        assert torch.equal(u[:U], wu[:U]) and torch.equal(g[:U], wg[:U])
    finally:
        dist.destroy_process_group()
