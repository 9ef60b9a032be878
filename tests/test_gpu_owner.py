"""Owner-sharded table on a B200 (hashed_gram_embedding_raw_b200.owner with the
library's kernels).

engram_owner_bucket is checked against a stable argsort by owner (exact:
grouped rows, positions, counts), including an empty input, ragged tiles and
rows no owner holds; engram_owner_bucket_padded against the same grouping
laid out in fixed-capacity segments (padding, overflow). The routing then
runs as 1, 2, 4 and 8 owner ranks emulated on one GPU (the all-to-alls become
device copies): on the tiny workload every rank's output must equal the
oracle's lookup in the whole table bit for bit and every owner's row
gradients the oracle's backward over all ranks' lookups restricted to its
rows; on b4x4096 and thd64k (Zipf traffic) the same against the oracle, with
the table's rows brought to the host by plain copies. The fixed-capacity
exchange needs no host synchronisation, so one step of 1 and of 2 emulated
ranks is captured in a CUDA graph and replayed. A real NCCL process group of
one rank runs the same routing through all_to_all_single.
"""

import datetime
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from tests._helpers import expected_rows, raw_bits
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


def padded_bucket(rows, rpo, owners, cap):
    local, order, dst, counts = stable_bucket(rows, rpo, owners)
    send = np.full(owners * cap, -1, np.int64)
    src = np.full(owners * cap, -1, np.int64)
    dst_p = np.full(len(rows), -1, np.int64)
    start = np.concatenate([[0], np.cumsum(counts)])
    for p in range(len(order)):
        o = np.searchsorted(start, p, side="right") - 1
        k = p - start[o]
        if k < cap:
            send[o * cap + k], src[o * cap + k] = local[p], order[p]
            dst_p[order[p]] = o * cap + k
    return send, src, dst_p, np.minimum(counts, cap)


@pytest.mark.parametrize("n,owners,rpo,cap", [(0, 4, 10, 3), (1, 1, 5, 1), (2049, 3, 1000, 2049),
                                              (5000, 8, 512, 700), (5000, 8, 512, 400),
                                              (100_000, 256, 400, 500)])
def test_padded_bucket_matches_host_layout(E, n, owners, rpo, cap):
    rng = np.random.default_rng(n + cap)
    rows = rng.integers(0, owners * rpo, size=n).astype(np.int32)
    send, src, dst, counts = E.engram_owner_bucket_padded(torch.from_numpy(rows).cuda(), rpo,
                                                          owners, cap)
    torch.cuda.synchronize()
    want = padded_bucket(rows, rpo, owners, cap)
    assert np.array_equal(send.cpu().numpy(), want[0])
    assert np.array_equal(src.cpu().numpy(), want[1])
    assert np.array_equal(dst.cpu().numpy(), want[2])
    assert np.array_equal(counts.cpu().numpy(), want[3])
    overflow = n > 0 and np.bincount(rows // rpo, minlength=owners).max() > cap
    assert bool(E.engram_get_device_error() & E.ENGRAM_DEVERR_CAPACITY) == bool(overflow)


def test_gather_and_backward_skip_negative_rows(E):
    """-1 marks an absent lookup: a zero row in the gather, left out of the
    backward; neither raises an error."""
    table = torch.randn(50, 32, device="cuda")
    idx = torch.tensor([3, -1, 7, -1, 3, 49], dtype=torch.int32, device="cuda")
    out = E.engram_gather(table, idx)
    assert torch.equal(out[[0, 2, 4, 5]], table[[3, 7, 3, 49]].contiguous())
    assert not out[[1, 3]].any()
    dout = torch.randn(6, 32, device="cuda")
    u, g, nu = E.engram_backward(idx, dout, 50)
    U = int(nu.item())
    assert U == 3 and u[:3].tolist() == [3, 7, 49]
    want = np.stack([dout[0].cpu().double().numpy() + dout[4].cpu().double().numpy(),
                     dout[2].cpu().numpy(), dout[5].cpu().numpy()])
    np.testing.assert_allclose(g[:3].cpu().numpy(), want, rtol=1e-6, atol=1e-6)
    assert E.engram_get_device_error() == 0


def split(ids, W):
    T = len(ids) // W
    return [(torch.from_numpy(ids[r * T:(r + 1) * T].copy()).cuda(),
             torch.tensor([0, T], dtype=torch.int32, device="cuda")) for r in range(W)]


def run_group(E, params, table, W, parts, douts, capacity=None):
    from hashed_gram_embedding_raw_b200 import owner
    rpo = params.table_rows // W
    shards = [table[r * rpo:(r + 1) * rpo] for r in range(W)]
    fwd = owner.run_lockstep([owner.forward_steps(params, shards[r], W, *parts[r],
                                                  capacity=capacity) for r in range(W)])
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


@pytest.mark.parametrize("name,W,tight", [("b4x4096", 4, False), ("thd64k", 8, False),
                                          ("thd64k", 8, True)])
def test_emulated_group_vs_oracle(E, name, W, tight):
    """Larger tables (16.8M and 67M bf16 rows) against the oracle: outputs row
    for row, every owner's gradients over all ranks' lookups. thd64k's Zipf
    IDs load some owners far more than others. `tight`: the capacity is the
    busiest (requester, owner) pair's count, the smallest that drops nothing."""
    cfg = head_params(name)
    params = E.make_params(cfg)
    R, D, H = cfg["table_rows"], cfg["dim"], params.heads
    table = torch.empty((R, D), dtype=torch.bfloat16, device="cuda")
    fill_device_table(table, 1)
    ids, _ = token_stream(name)
    parts = split(ids, W)
    rpo = R // W
    cap = None
    if tight:
        cap = max(int(np.bincount(oracle.hash_ids(p[0].cpu().numpy(), p[1].cpu().numpy(),
                                                  cfg).reshape(-1) // rpo, minlength=W).max())
                  for p in parts)
        assert cap < len(parts[0][0]) * H
    douts = [host_dout(name, len(p[0]) * H, D, "bf16", seed_offset=r)
             for r, p in enumerate(parts)]
    fwd, bwd = run_group(E, params, table, W, parts, [d.cuda() for d in douts], capacity=cap)
    all_idx = []
    for r, (ids_r, cu_r) in enumerate(parts):
        idx = oracle.hash_ids(ids_r.cpu().numpy(), cu_r.cpu().numpy(), cfg)
        want = expected_rows(idx, table).reshape(len(ids_r), -1)
        assert raw_bits(fwd[r][0]).tobytes() == want.tobytes()
        all_idx.append(idx.reshape(-1))
    idx = np.concatenate(all_idx)
    dout = np.concatenate([d.view(torch.int16).numpy().view(np.uint16) for d in douts])
    per_owner = np.bincount(idx // rpo, minlength=W)
    for r in range(W):
        keep = (idx // rpo) == r
        u, g = oracle.backward(idx[keep] - r * rpo, dout[keep], oracle.BF16)
        gu, gg, gn = bwd[r]
        U = int(gn.item())
        assert U == len(u)
        assert np.array_equal(gu[:U].cpu().numpy(), u)
        err = np.abs(gg[:U].cpu().numpy().astype(np.float64) - g)
        assert (err <= 1e-6 + 1e-5 * np.abs(g)).all()
    assert E.engram_get_device_error() == 0
    if name == "thd64k":
        assert per_owner.max() > 1.5 * per_owner.min()   # the splits really are uneven


@pytest.mark.parametrize("W", [1, 2])
def test_step_captured_in_cuda_graph(E, W):
    """The fixed-capacity step has static shapes and no host round trip: the
    whole forward and backward of W emulated ranks is captured once and
    replayed, with the same results as the eager step on new inputs."""
    from hashed_gram_embedding_raw_b200 import owner
    cfg = head_params("tiny")
    params = E.make_params(cfg)
    table = torch.from_numpy(host_table("tiny")).cuda()
    ids, _ = token_stream("tiny")
    H, D = params.heads, cfg["dim"]
    rpo = params.table_rows // W
    shards = [table[r * rpo:(r + 1) * rpo] for r in range(W)]
    parts = split(ids, W)
    T = len(parts[0][0])
    douts = [torch.zeros(T * H, D, device="cuda") for _ in range(W)]

    def step():
        fwd = owner.run_lockstep([owner.forward_steps(params, shards[r], W, *parts[r])
                                  for r in range(W)])
        bwd = owner.run_lockstep([owner.backward_steps(params, W, fwd[r][1], douts[r])
                                  for r in range(W)])
        return fwd, bwd

    step()                                   # warm-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            fwd_g, bwd_g = step()
    torch.cuda.current_stream().wait_stream(s)
    # new inputs in the captured buffers, then replay
    rng = np.random.default_rng(W)
    for r in range(W):
        new_ids = rng.integers(0, 1000, T).astype(np.int32)
        new_ids[rng.random(T) < 0.05] = cfg["eos_id"]
        parts[r][0].copy_(torch.from_numpy(new_ids))
        douts[r].copy_(torch.randn(T * H, D, generator=torch.Generator().manual_seed(r)))
    graph.replay()
    torch.cuda.synchronize()
    fwd_e, bwd_e = step()
    torch.cuda.synchronize()
    for r in range(W):
        assert torch.equal(fwd_g[r][0], fwd_e[r][0])
        U = int(bwd_e[r][2].item())
        assert int(bwd_g[r][2].item()) == U
        assert torch.equal(bwd_g[r][0][:U], bwd_e[r][0][:U])
        assert torch.equal(bwd_g[r][1][:U], bwd_e[r][1][:U])
        # and against the oracle
        idx = oracle.hash_ids(parts[r][0].cpu().numpy(), parts[r][1].cpu().numpy(), cfg)
        want = oracle.gather(host_table("tiny"), idx).reshape(T, -1)
        assert np.array_equal(fwd_g[r][0].cpu().numpy(), want)
    del graph
    assert E.engram_get_device_error() == 0


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
