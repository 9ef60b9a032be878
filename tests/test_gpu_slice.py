"""engram_hash_gather_slice (the page's NGramEmbedding._forward_global_slice)
against the oracle, on a B200.

A slice [start, end) of every row must equal the whole-stream hash and lookup
restricted to those positions: the two tokens before `start` and any EOS or
sequence reset before it still shape the slice's first tokens (the engram
page's two-rank tests check exactly this across an EOS/shard boundary).
Indices and rows are compared bit for bit.
"""

import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle_hash import small_params
from workloads import (WORKLOADS, fill_device_table, head_params, host_table, random_stream,
                       token_stream)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    import hashed_gram_embedding_raw_b200 as E
    torch.cuda.set_device(0)
    E.engram_get_device_error()
    return E


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def check_slice(E, cfg, ids, cu, table, row_len, start, end):
    out, idx = E.engram_hash_gather_slice(E.make_params(cfg), dev(ids), table, start, end,
                                          row_len=row_len,
                                          cu_seqlens=None if cu is None else dev(cu))
    row = row_len or len(ids)
    want_idx = oracle.hash_ids(ids, cu, cfg).reshape(len(ids) // row, row, -1)[:, start:end]
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
    rows = want_idx.reshape(-1)
    uniq, inv = np.unique(rows, return_inverse=True)
    compact = table[torch.from_numpy(uniq).cuda()].cpu()
    view = torch.int32 if compact.dtype == torch.float32 else torch.int16
    want = oracle.gather(compact.view(view).numpy(), inv)
    assert out.cpu().view(view).numpy().reshape(-1).tobytes() == want.reshape(-1).tobytes()
    assert E.engram_get_device_error() == 0


def test_slice_tiny_every_window(E):
    cfg = head_params("tiny")
    ids, cu = token_stream("tiny")
    table = dev(host_table("tiny"))
    for start, end in [(0, 64), (0, 1), (1, 2), (2, 3), (5, 37), (31, 33), (63, 64), (10, 10)]:
        check_slice(E, cfg, ids, cu, table, 64, start, end)
    # one flat row over both sequences: the slice crosses the sequence bound
    for start, end in [(60, 70), (64, 65), (0, 128)]:
        check_slice(E, cfg, ids, cu, table, 0, start, end)


def test_slice_starts_after_eos_and_sequence_bounds(E):
    cfg = small_params(seed=4, eos=7)
    ids, cu = random_stream(12, 3000, 20, 7, 0.08, nseq=5)
    table = torch.randn(cfg["table_rows"], 160).to(torch.bfloat16).cuda()
    eos_pos = np.nonzero(ids == 7)[0]
    starts = sorted(set([int(p) + d for p in eos_pos[:20] for d in (0, 1, 2, 3)] +
                        [int(c) + d for c in cu[1:-1] for d in (0, 1, 2)]))
    for s in starts:
        if 0 <= s < len(ids):
            check_slice(E, cfg, ids, cu, table, 0, s, min(len(ids), s + 45))


@pytest.mark.parametrize("N,K,dtype", [(2, 3, torch.float32), (4, 2, torch.bfloat16)])
def test_slice_generic_shapes(E, N, K, dtype):
    cfg = dict(small_params(seed=N * 10 + K, N=N, K=K, eos=3), dim=64)
    ids, _ = random_stream(N + K, 8 * 500, 30, 3, 0.1)
    cu = np.arange(0, 8 * 500 + 1, 500, dtype=np.int32)
    table = torch.randn(cfg["table_rows"], 64).to(dtype).cuda()
    for start, end in [(0, 500), (1, 499), (250, 251), (3, 100)]:
        check_slice(E, cfg, ids, cu, table, 500, start, end)


def test_slice_of_full_workload_rows(E):
    cfg = head_params("b4x4096")
    ids, cu = token_stream("b4x4096")
    table = torch.empty(cfg["table_rows"], cfg["dim"], dtype=torch.bfloat16, device="cuda")
    fill_device_table(table, WORKLOADS["b4x4096"].seed)
    # eight context-parallel shards of each 4,096-token row
    for r in range(8):
        check_slice(E, cfg, ids, cu, table, 4096, 512 * r, 512 * (r + 1))


def test_slice_rejects_bad_bounds(E):
    cfg = head_params("tiny")
    ids, _ = token_stream("tiny")
    table = dev(host_table("tiny"))
    p = E.make_params(cfg)
    for row_len, start, end in [(64, 10, 5), (64, 0, 65), (60, 0, 10), (-1, 0, 1)]:
        with pytest.raises((E.EngramError, ValueError)):
            E.engram_hash_gather_slice(p, dev(ids), table, start, end, row_len=row_len)
