"""Owner-sharded Engram table over an owner group of ranks (engram page,
Qwen3_8_FlashNextOwnerShardedEmbedding with _FixedCapacityAllToAll).

Rank r of W owners holds rows [r * R / W, (r + 1) * R / W) of the packed
table (R divisible by W, as the page requires). A requesting rank hashes its
tokens, groups the row lookups by owner (engram_owner_bucket), and

  1. exchanges the per-owner counts (a W-element all-to-all),
  2. sends the owner-local rows to their owners (all-to-all of int32),
  3. each owner gathers the rows from its shard (engram_gather),
  4. the rows come back in the same grouping (all-to-all of rows) and are
     put back in request order (engram_gather by each lookup's position).

The backward sends each lookup's gradient to the owner the row came from
(engram_gather by grouped position, then the reverse all-to-all), and the
owner reduces them into compact per-row gradients of its shard
(engram_backward), ready for engram_sparse_adam on that shard: only the owner
accumulates and updates a row's gradient.

Every step on the device runs in the library's kernels; the exchanges are
NCCL all-to-alls through torch.distributed (uneven splits, so no padding to a
common capacity is needed). The routing is written as generators that yield
at each exchange, so one code path serves a real process group
(`run_collective`) and a group of ranks emulated in one process on one device
(`run_lockstep`), where the exchange is a set of device copies.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _binding as B


@dataclass
class Counts:
    """Exchange request: every rank's per-owner counts [W] (int32, device)."""
    counts: torch.Tensor


@dataclass
class AllToAll:
    """Exchange request: send[sum(send_counts)] grouped by destination rank,
    receive sum(recv_counts) rows grouped by source rank."""
    send: torch.Tensor
    send_counts: list
    recv_counts: list


@dataclass
class Routing:
    """What the backward needs from a forward."""
    src_pos: torch.Tensor     # [n] lookup index of each grouped position
    recv_rows: torch.Tensor   # [sum recv] owner-local rows this rank serves
    send_counts: list
    recv_counts: list


class CudaOps:
    """The device steps, one library call each."""

    @staticmethod
    def hash(params, ids, cu_seqlens):
        return B.engram_hash(params, ids, cu_seqlens)

    @staticmethod
    def bucket(rows, rows_per_owner, owners):
        send, src_pos, dst_pos, counts = B.engram_owner_bucket(rows, rows_per_owner, owners)
        return send, src_pos, dst_pos, counts

    @staticmethod
    def gather(table, idx):
        return B.engram_gather(table, idx)

    @staticmethod
    def backward(idx, dout, table_rows):
        return B.engram_backward(idx, dout, table_rows)


def rows_per_owner(params, owners: int) -> int:
    if params.table_rows % owners:
        raise ValueError("the table's rows must divide evenly among the owners")
    return params.table_rows // owners


def forward_steps(params, shard: torch.Tensor, owners: int, ids: torch.Tensor,
                  cu_seqlens=None, ops=CudaOps):
    """Generator: the owner-sharded forward of one rank. Yields Counts and
    AllToAll requests and receives their results; returns (out [T, H * dim],
    Routing)."""
    rpo = rows_per_owner(params, owners)
    if shard.shape[0] != rpo:
        raise ValueError("shard must hold table_rows / owners rows")
    idx = ops.hash(params, ids, cu_seqlens)                  # [T, H] global rows
    T, H = idx.shape
    send, src_pos, dst_pos, counts = ops.bucket(idx.reshape(-1), rpo, owners)
    recv_counts = yield Counts(counts)
    sc, rc = [int(v) for v in counts.tolist()], [int(v) for v in recv_counts.tolist()]
    recv_rows = yield AllToAll(send, sc, rc)                 # rows this rank serves
    vals = ops.gather(shard, recv_rows)                      # [sum rc, dim]
    back = yield AllToAll(vals, rc, sc)                      # [n, dim], grouped by owner
    out = ops.gather(back, dst_pos)                          # request order
    return out.reshape(T, H * shard.shape[1]), Routing(src_pos, recv_rows, sc, rc)


def backward_steps(params, owners: int, routing: Routing, dout: torch.Tensor, ops=CudaOps):
    """Generator: the backward of one rank given dout [T, H * dim] (or
    [n, dim]). Returns (uniq_rows, row_grads, num_unique) of this rank's shard
    (owner-local rows)."""
    rpo = rows_per_owner(params, owners)
    dim = params.dim
    grouped = ops.gather(dout.reshape(-1, dim), routing.src_pos)   # grouped by owner
    owner_dout = yield AllToAll(grouped, routing.send_counts, routing.recv_counts)
    return ops.backward(routing.recv_rows, owner_dout, rpo)


def run_collective(gen, group=None):
    """Runs one rank's generator over a torch.distributed process group."""
    import torch.distributed as dist
    try:
        req = next(gen)
        while True:
            if isinstance(req, Counts):
                out = torch.empty_like(req.counts)
                dist.all_to_all_single(out, req.counts, group=group)
            else:
                rows = sum(req.recv_counts)
                out = torch.empty((rows,) + tuple(req.send.shape[1:]), dtype=req.send.dtype,
                                  device=req.send.device)
                dist.all_to_all_single(out, req.send, output_split_sizes=req.recv_counts,
                                       input_split_sizes=req.send_counts, group=group)
            req = gen.send(out)
    except StopIteration as stop:
        return stop.value


def run_lockstep(gens):
    """Runs the generators of W ranks emulated in one process: every exchange
    is performed as copies once all ranks have reached it."""
    W = len(gens)
    reqs = [next(g) for g in gens]
    results = [None] * W
    done = [False] * W
    while not all(done):
        kinds = {type(r) for r in reqs}
        if len(kinds) != 1:
            raise RuntimeError("ranks reached different exchanges")
        if isinstance(reqs[0], Counts):
            table = torch.stack([r.counts for r in reqs])            # [src, dst]
            outs = [table[:, r].contiguous() for r in range(W)]
        else:
            starts = []
            for r in reqs:
                offs, o = [], 0
                for c in r.send_counts:
                    offs.append(o)
                    o += c
                starts.append(offs)
            outs = []
            for dst in range(W):
                parts = [reqs[src].send[starts[src][dst]:starts[src][dst] +
                                        reqs[src].send_counts[dst]] for src in range(W)]
                got = torch.cat(parts) if parts else reqs[dst].send[:0]
                if got.shape[0] != sum(reqs[dst].recv_counts):
                    raise RuntimeError("receive counts disagree with the senders")
                outs.append(got)
        for r, g in enumerate(gens):
            try:
                reqs[r] = g.send(outs[r])
            except StopIteration as stop:
                results[r] = stop.value
                done[r] = True
        if any(done) and not all(done):
            raise RuntimeError("ranks finished at different exchanges")
    return results
