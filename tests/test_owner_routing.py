"""Owner-sharded routing (hashed_gram_embedding_raw_b200.owner) on the CPU.

The routing generators run with host stand-ins for the device steps (defined
here: the oracle's hash, gather and backward, and a stable argsort for the
grouping), first as ranks emulated in one process, then as two gloo ranks with
real all-to-alls. What they pin is the exchange logic of the page's
Qwen3_8_FlashNextOwnerShardedEmbedding with its fixed-capacity exchange: the
grouping by owner into padded segments, putting values back in request order
and sending gradients back to the owner, which alone accumulates its rows.
Every rank's output must equal the oracle's lookup in the whole table, and
every owner's row gradients the oracle's backward over all ranks' lookups
restricted to its rows -- at the default capacity and at tight ones.
"""

import os
import socket

import numpy as np
import pytest
import torch

import oracle
from workloads import head_params, host_dout, host_table, token_stream


class HostOps:
    """Host stand-ins for the device steps (test only)."""

    def __init__(self, cfg):
        self.cfg = cfg

    def hash(self, params, ids, cu):
        idx = oracle.hash_ids(ids.numpy(), None if cu is None else cu.numpy(), self.cfg)
        return torch.from_numpy(idx.astype(np.int32))

    def bucket(self, rows, rpo, owners, cap):
        r = rows.numpy().astype(np.int64)
        o = r // rpo
        order = np.argsort(o, kind="stable")
        counts = np.bincount(o, minlength=owners)
        send = np.full(owners * cap, -1, np.int32)
        src = np.full(owners * cap, -1, np.int32)
        dst = np.full(len(r), -1, np.int32)
        start = np.concatenate([[0], np.cumsum(counts)])
        for p, i in enumerate(order):
            k = p - start[o[i]]
            if k < cap:
                slot = o[i] * cap + k
                send[slot], src[slot], dst[i] = r[i] - o[i] * rpo, i, slot
        return (torch.from_numpy(send), torch.from_numpy(src), torch.from_numpy(dst),
                torch.from_numpy(np.minimum(counts, cap).astype(np.int32)))

    def gather(self, table, idx):
        i = idx.long()
        out = table[i.clamp(min=0)]
        out[i < 0] = 0
        return out

    def backward(self, idx, dout, table_rows):
        keep = idx.numpy() >= 0
        u, g = oracle.backward(idx.numpy()[keep], dout.numpy()[keep], oracle.F32)
        return torch.from_numpy(u), torch.from_numpy(g), torch.tensor([len(u)], dtype=torch.int32)


def split_stream(ids, W):
    """W equal token chunks of the tiny stream, one sequence each."""
    T = len(ids) // W
    return [(torch.from_numpy(ids[r * T:(r + 1) * T].copy()),
             torch.tensor([0, T], dtype=torch.int32)) for r in range(W)]


def expected(cfg, table, parts, douts, W):
    rpo = cfg["table_rows"] // W
    outs, all_idx = [], []
    for ids, cu in parts:
        idx = oracle.hash_ids(ids.numpy(), cu.numpy(), cfg)
        outs.append(oracle.gather(table, idx).reshape(len(ids), -1))
        all_idx.append(idx.reshape(-1))
    idx = np.concatenate(all_idx)
    dout = np.concatenate([d.numpy() for d in douts])
    owners = []
    for r in range(W):
        keep = (idx // rpo) == r
        u, g = oracle.backward(idx[keep] - r * rpo, dout[keep], oracle.F32)
        owners.append((u, g))
    return outs, owners


def run_rank(E_owner, params, cfg, table, W, r, ids, cu, dout, runner, capacity=None):
    rpo = cfg["table_rows"] // W
    shard = torch.from_numpy(table[r * rpo:(r + 1) * rpo].copy())
    ops = HostOps(cfg)
    out, routing = runner(E_owner.forward_steps(params, shard, W, ids, cu, capacity=capacity,
                                                ops=ops))
    u, g, nu = runner(E_owner.backward_steps(params, W, routing, dout, ops=ops))
    return out, u, g, nu


@pytest.mark.parametrize("W,cap", [(1, None), (2, None), (4, None), (2, 1100), (4, 600)])
def test_lockstep_emulated_ranks(W, cap):
    from hashed_gram_embedding_raw_b200 import make_params, owner
    cfg = head_params("tiny")
    params = make_params(cfg)
    table = host_table("tiny")
    ids, _ = token_stream("tiny")
    parts = split_stream(ids, W)
    H, D = params.heads, cfg["dim"]
    douts = [host_dout("tiny", len(p[0]) * H, D, "f32", seed_offset=r) for r, p in
             enumerate(parts)]
    rpo = cfg["table_rows"] // W
    ops = HostOps(cfg)
    shards = [torch.from_numpy(table[r * rpo:(r + 1) * rpo].copy()) for r in range(W)]
    fwd = owner.run_lockstep([owner.forward_steps(params, shards[r], W, *parts[r],
                                                  capacity=cap, ops=ops) for r in range(W)])
    bwd = owner.run_lockstep([owner.backward_steps(params, W, fwd[r][1], douts[r], ops=ops)
                              for r in range(W)])
    outs, owners = expected(cfg, table, parts, douts, W)
    for r in range(W):
        assert np.array_equal(fwd[r][0].numpy(), outs[r])
        u, g, nu = bwd[r]
        assert int(nu[0]) == len(owners[r][0])
        assert np.array_equal(u.numpy(), owners[r][0]) and np.array_equal(g.numpy(), owners[r][1])


def test_lockstep_capacity_overflow_drops_lookups():
    """A capacity below some owner's lookups drops the excess: their rows come
    back zero and their gradients are left out, nothing else changes."""
    from hashed_gram_embedding_raw_b200 import make_params, owner
    cfg = head_params("tiny")
    params = make_params(cfg)
    table = host_table("tiny")
    ids, _ = token_stream("tiny")
    W, cap = 2, 300
    parts = split_stream(ids, W)
    ops = HostOps(cfg)
    rpo = cfg["table_rows"] // W
    shards = [torch.from_numpy(table[r * rpo:(r + 1) * rpo].copy()) for r in range(W)]
    fwd = owner.run_lockstep([owner.forward_steps(params, shards[r], W, *parts[r],
                                                  capacity=cap, ops=ops) for r in range(W)])
    for r in range(W):
        idx = oracle.hash_ids(parts[r][0].numpy(), parts[r][1].numpy(), cfg).reshape(-1)
        got = fwd[r][0].numpy().reshape(len(idx), -1)
        # lookups kept: each owner's first `cap` lookups in request order
        o = idx // rpo
        kept = np.zeros(len(idx), bool)
        for w in range(W):
            kept[np.nonzero(o == w)[0][:cap]] = True
        assert (~kept).any()
        want = oracle.gather(table, idx)
        assert np.array_equal(got[kept], want[kept]) and not got[~kept].any()


def test_rows_must_divide_among_owners():
    from hashed_gram_embedding_raw_b200 import make_params, owner
    cfg = dict(head_params("tiny"))
    cfg["table_rows"] += 1
    with pytest.raises(ValueError):
        owner.rows_per_owner(make_params(cfg), 2)


def _gloo_rank(rank, world, port, result_dir):
    import datetime
    import torch.distributed as dist
    from hashed_gram_embedding_raw_b200 import make_params, owner
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cfg = head_params("tiny")
        params = make_params(cfg)
        table = host_table("tiny")
        ids, _ = token_stream("tiny")
        parts = split_stream(ids, world)
        H, D = params.heads, cfg["dim"]
        douts = [host_dout("tiny", len(p[0]) * H, D, "f32", seed_offset=r)
                 for r, p in enumerate(parts)]
        # the capacity agreed over both ranks: the largest owner segment of
        # either rank's lookups, rounded up to 16
        cap = owner.agree_capacity(params, world, *parts[rank], multiple=16, ops=HostOps(cfg))
        rpo = cfg["table_rows"] // world
        top = max(np.bincount(oracle.hash_ids(i.numpy(), c.numpy(), cfg).reshape(-1) // rpo,
                              minlength=world).max() for i, c in parts)
        out, u, g, nu = run_rank(owner, params, cfg, table, world, rank, *parts[rank],
                                 douts[rank], lambda gen: owner.run_collective(gen),
                                 capacity=cap)
        outs, owners = expected(cfg, table, parts, douts, world)
        ok = (cap == -(-top // 16) * 16 and cap < len(parts[rank][0]) * params.heads
              and np.array_equal(out.numpy(), outs[rank]) and int(nu[0]) == len(owners[rank][0])
              and np.array_equal(u.numpy(), owners[rank][0])
              and np.array_equal(g.numpy(), owners[rank][1]))
        with open(os.path.join(result_dir, f"rank{rank}"), "w") as f:
            f.write("ok" if ok else "mismatch")
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    """Two gloo ranks with real all-to-alls at the capacity they agree on
    (agree_capacity's all-reduce), below the default, with nothing dropped."""
    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mp.start_processes(_gloo_rank, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    for r in range(2):
        assert (tmp_path / f"rank{r}").read_text() == "ok"
