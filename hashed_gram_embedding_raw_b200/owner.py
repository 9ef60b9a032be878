"""Owner-sharded Engram table over an owner group of ranks (engram API page,
Qwen3_8_FlashNextOwnerShardedEmbedding with _FixedCapacityAllToAll /
_fixed_capacity_all_to_all).

Rank r of W owners holds rows [r * R / W, (r + 1) * R / W) of the packed
table (R divisible by W, as the page requires). A requesting rank hashes its
tokens and groups the row lookups by owner into fixed-capacity segments
(engram_owner_bucket_padded: W segments of `capacity` slots, the unused
slots marked -1), then

  1. sends every owner its segment (an equal-split all-to-all of int32 rows),
  2. each owner gathers the rows from its shard (engram_gather; padding
     slots give zero rows),
  3. the rows come back in the same layout (an equal-split all-to-all) and
     are put back in request order (engram_gather by each lookup's slot).

The backward sends each lookup's gradient to the owner the row came from
(engram_gather by grouped slot, then the same exchange), and the owner
reduces them into compact per-row gradients of its shard (engram_backward,
which leaves the padding slots out), ready for engram_sparse_adam on that
shard: only the owner accumulates and updates a row's gradient.

The capacity is agreed ahead of time, as the page's capacity is, so every
exchange has the same size whatever the data: no counts cross to the host,
nothing synchronises with it, and a whole step can be captured in a CUDA
graph. capacity = n (the default) can never overflow; a smaller one that
an owner's lookups exceed drops the excess and sets ENGRAM_DEVERR_CAPACITY.

Every step on the device runs in the library's kernels; the exchanges are
NCCL all-to-alls through torch.distributed. The routing is written as
generators that yield at each exchange, so one code path serves a real
process group (`run_collective`) and a group of ranks emulated in one process
on one device (`run_lockstep`), where the exchange is a set of device copies.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _binding as B


@dataclass
class AllToAll:
    """Exchange request: send [W * capacity, ...] holds one segment of
    `capacity` rows per destination rank; the result holds one such segment
    per source rank."""
    send: torch.Tensor


@dataclass
class Routing:
    """What the backward needs from a forward."""
    src_pos: torch.Tensor     # [W * capacity] lookup of each grouped slot, -1: padding
    recv_rows: torch.Tensor   # [W * capacity] owner-local rows this rank serves, -1: padding


class CudaOps:
    """The device steps, one library call each."""

    @staticmethod
    def hash(params, ids, cu_seqlens):
        return B.engram_hash(params, ids, cu_seqlens)

    @staticmethod
    def bucket(rows, rows_per_owner, owners, capacity):
        return B.engram_owner_bucket_padded(rows, rows_per_owner, owners, capacity)

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
                  cu_seqlens=None, capacity=None, ops=CudaOps):
    """Generator: the owner-sharded forward of one rank. Yields AllToAll
    requests and receives their results; returns (out [T, H * dim], Routing).
    `capacity` (slots per owner and requesting rank, the same on every rank)
    defaults to this rank's lookups, T * H."""
    rpo = rows_per_owner(params, owners)
    if shard.shape[0] != rpo:
        raise ValueError("shard must hold table_rows / owners rows")
    idx = ops.hash(params, ids, cu_seqlens)                  # [T, H] global rows
    T, H = idx.shape
    cap = T * H if capacity is None else int(capacity)
    if cap < 1:
        raise ValueError("capacity must be at least 1")
    send, src_pos, dst_pos, _ = ops.bucket(idx.reshape(-1), rpo, owners, cap)
    recv_rows = yield AllToAll(send)                         # rows this rank serves
    vals = ops.gather(shard, recv_rows)                      # [W * cap, dim]
    back = yield AllToAll(vals)                              # grouped by owner
    out = ops.gather(back, dst_pos)                          # request order
    return out.reshape(T, H * shard.shape[1]), Routing(src_pos, recv_rows)


def backward_steps(params, owners: int, routing: Routing, dout: torch.Tensor, ops=CudaOps):
    """Generator: the backward of one rank given dout [T, H * dim] (or
    [n, dim]). Returns (uniq_rows, row_grads, num_unique) of this rank's shard
    (owner-local rows)."""
    rpo = rows_per_owner(params, owners)
    dim = params.dim
    grouped = ops.gather(dout.reshape(-1, dim), routing.src_pos)   # grouped by owner
    owner_dout = yield AllToAll(grouped)
    return ops.backward(routing.recv_rows, owner_dout, rpo)


def agree_capacity(params, owners: int, ids: torch.Tensor, cu_seqlens=None, group=None,
                   multiple: int = 256, ops=CudaOps) -> int:
    """A capacity for batches like this one, agreed once ahead of the steps:
    the largest number of lookups any rank sends any owner (the page's global
    maximum peer-segment row count), rounded up to `multiple`. This setup
    call reads the counts on the host and, in a process group, takes their
    maximum over the ranks with an all-reduce; the steps that then use the
    capacity do neither."""
    rpo = rows_per_owner(params, owners)
    idx = ops.hash(params, ids, cu_seqlens).reshape(-1)
    n = idx.numel()
    _, _, _, counts = ops.bucket(idx, rpo, owners, max(n, 1))
    top = counts.max().reshape(1).to(torch.int64)
    if group is not None or owners > 1:
        import torch.distributed as dist
        dist.all_reduce(top, op=dist.ReduceOp.MAX, group=group)
    cap = int(top.item())
    return max(multiple, -(-cap // multiple) * multiple)


def run_collective(gen, group=None):
    """Runs one rank's generator over a torch.distributed process group; every
    exchange is an equal-split all_to_all_single."""
    import torch.distributed as dist
    try:
        req = next(gen)
        while True:
            out = torch.empty_like(req.send)
            dist.all_to_all_single(out, req.send, group=group)
            req = gen.send(out)
    except StopIteration as stop:
        return stop.value


def run_lockstep(gens):
    """Runs the generators of W ranks emulated in one process: every exchange
    is performed as device copies once all ranks have reached it."""
    W = len(gens)
    reqs = [next(g) for g in gens]
    results = [None] * W
    done = [False] * W
    while not all(done):
        shape = reqs[0].send.shape
        if any(r.send.shape != shape for r in reqs) or shape[0] % W:
            raise RuntimeError("ranks disagree on the exchange's capacity")
        cap = shape[0] // W
        outs = [torch.cat([reqs[src].send[dst * cap:(dst + 1) * cap] for src in range(W)])
                for dst in range(W)]
        for r, g in enumerate(gens):
            try:
                reqs[r] = g.send(outs[r])
            except StopIteration as stop:
                results[r] = stop.value
                done[r] = True
        if any(done) and not all(done):
            raise RuntimeError("ranks finished at different exchanges")
    return results
