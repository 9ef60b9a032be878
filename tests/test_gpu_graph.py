"""The library's calls replay inside CUDA graphs (B200).

A training step of the hot path -- engram_hash_gather, engram_backward (sort +
reduce), engram_sparse_adam -- and the PLE tail are captured once into a
torch CUDA graph and replayed; every replay must equal the same calls made
eagerly, bit for bit (all kernels are deterministic). The calls need no host
synchronisation: the optimizer reads num_unique on the device.
"""

import numpy as np
import pytest
import torch

from workloads import head_params, host_dout, token_stream

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def E():
    import hashed_gram_embedding_raw_b200 as E
    torch.cuda.set_device(0)
    E.engram_get_device_error()
    return E


def make_step(E, name):
    cfg = head_params(name)
    params = E.make_params(cfg)
    ids, cu = token_stream(name)
    T, H, D, R = len(ids), params.heads, cfg["dim"], cfg["table_rows"]
    n = T * H
    g = torch.Generator(device="cuda").manual_seed(1)
    st = {
        "ids": torch.from_numpy(ids.copy()).cuda(), "cu": torch.from_numpy(cu.copy()).cuda(),
        "table": (0.02 * torch.randn((R, D), generator=g, device="cuda")).to(torch.bfloat16),
        "m": torch.zeros((R, D), device="cuda"), "v": torch.zeros((R, D), device="cuda"),
        "out": torch.empty((T, H * D), dtype=torch.bfloat16, device="cuda"),
        "idx": torch.empty((T, H), dtype=torch.int32, device="cuda"),
        "dout": host_dout(name, n, D, "bf16").cuda(),
        "uniq": torch.empty(n, dtype=torch.int32, device="cuda"),
        "grads": torch.empty((n, D), device="cuda"),
        "nu": torch.empty(1, dtype=torch.int32, device="cuda"),
        "ws": torch.empty(E.engram_backward_workspace_size(n, R, D), dtype=torch.uint8,
                          device="cuda"),
    }
    counter = {"step": 0}

    def step(step_no):
        E.engram_hash_gather(params, st["ids"], st["table"], cu_seqlens=st["cu"],
                             out=st["out"], out_idx=st["idx"])
        E.engram_backward(st["idx"].view(-1), st["dout"], R, uniq_rows=st["uniq"],
                          row_grads=st["grads"], num_unique=st["nu"], workspace=st["ws"])
        E.engram_sparse_adam(st["table"], st["m"], st["v"], st["uniq"], st["grads"], st["nu"],
                             lr=1e-3, weight_decay=0.01, step=step_no)

    return st, step, counter


@pytest.mark.parametrize("name", ["tiny", "b4x4096"])
def test_training_step_replays_in_a_graph(E, name):
    st_e, step_e, _ = make_step(E, name)
    st_g, step_g, _ = make_step(E, name)
    # warm-up (first calls look up device attributes) on a side stream, as
    # torch requires before capture; both copies then start from equal state
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step_e(1)
        step_g(1)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for k in ("table", "m", "v"):
        assert torch.equal(st_e[k], st_g[k])
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step_g(2)            # the step count is baked into the graph: replay = step 2 again
    for _ in range(3):
        graph.replay()
        step_e(2)
    torch.cuda.synchronize()
    assert E.engram_get_device_error() == 0
    for k in ("out", "idx", "nu", "table", "m", "v"):
        assert torch.equal(st_e[k], st_g[k]), k
    U = int(st_e["nu"].item())
    assert torch.equal(st_e["uniq"][:U], st_g["uniq"][:U])
    assert torch.equal(st_e["grads"][:U], st_g["grads"][:U])


def test_ple_tail_replays_in_a_graph(E):
    T, C, G = 8192, 10240, 2560
    g = torch.Generator(device="cuda").manual_seed(2)
    x = torch.randn((T, C), generator=g, device="cuda").to(torch.bfloat16)
    w = (0.5 * torch.randn((C, 4), generator=g, device="cuda")).to(torch.bfloat16)
    nw = (0.1 * torch.randn(C, generator=g, device="cuda")).to(torch.bfloat16)
    cu = torch.arange(0, T + 1, 4096, dtype=torch.int32, device="cuda")
    out_e, out_g = torch.empty_like(x), torch.empty_like(x)
    norm_e, norm_g = torch.empty_like(x), torch.empty_like(x)

    def run(out, nout):
        E.engram_ple_short_conv(x, w, dilation=3, group_size=G, cu_seqlens=cu, norm_weight=nw,
                                out=out)
        E.engram_grouped_rms_norm(x, G, weight=nw, out=nout)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run(out_e, norm_e)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run(out_g, norm_g)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out_e, out_g) and torch.equal(norm_e, norm_g)
