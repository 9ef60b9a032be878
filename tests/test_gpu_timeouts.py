"""Bounded waits that run out, on a B200.

The library's kernels never spin without a bound: the one-launch radix sort's
grid barrier gives up after a number of polls and raises
ENGRAM_DEVERR_SORT_TIMEOUT, and the PLE tail kernel's waits on other warps give
up after a time and raise ENGRAM_DEVERR_COPY_TIMEOUT; either way the call
returns and the CUDA context stays usable. Two test hooks, read once per
process, shorten those bounds (ENGRAM_TEST_BARRIER_SPIN = polls,
ENGRAM_TEST_CROSS_WAIT_NS = nanoseconds), so each test runs a child process
with the hook set to zero: its waits run out at the first poll that finds them
unfinished. The child checks the error bit, then runs a normal hash call and
checks it against the oracle, so the context is shown to work after the
timeout. (A wait that runs out leaves that call's output unspecified; every
access stays inside the call's own buffers.)
"""

import json
import os
import subprocess
import sys

import pytest

from tests.conftest import ROOT

pytestmark = pytest.mark.gpu

CHILD = r'''
import json, sys
import numpy as np
import torch
sys.path.insert(0, ROOT)
import hashed_gram_embedding_raw_b200 as E
import oracle
from tests.test_oracle_hash import small_params
from workloads import random_stream
torch.cuda.set_device(0)
E.engram_get_device_error()
res = {}
if WHAT == "sort":
    n, R, D = 300_000, 1 << 20, 160
    g = torch.Generator().manual_seed(1)
    idx = torch.randint(0, R, (n,), generator=g, dtype=torch.int32).cuda()
    ws = torch.empty(E.engram_backward_workspace_size(n, R, D), dtype=torch.uint8,
                     device="cuda")
    E.engram_backward_sort(idx, R, D, ws)
else:
    from workloads import ple_inputs
    T, C, G, K, d = 4096, 1024, 256, 4, 3
    x, nw, w, b = ple_inputs(T, C, K, 3, "bf16")
    bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    cu = torch.tensor([0, 1000, 4096], dtype=torch.int32).cuda()
    E.engram_ple_short_conv(bf(x), bf(w), dilation=d, group_size=G, cu_seqlens=cu,
                            norm_weight=bf(nw), conv_bias=bf(b))
torch.cuda.synchronize()
res["flags"] = E.engram_get_device_error()
# the context still works: a hash call, checked against the oracle
cfg = small_params(seed=3, eos=13)
ids, cu = random_stream(5, 5000, 100_000, 13, 0.05, nseq=3)
got = E.engram_hash(E.make_params(cfg), torch.from_numpy(ids.copy()).cuda(),
                    torch.from_numpy(cu.copy()).cuda())
res["hash_ok"] = bool(np.array_equal(got.cpu().numpy(), oracle.hash_ids(ids, cu, cfg)))
res["flags_after"] = E.engram_get_device_error()
print("RESULT " + json.dumps(res))
'''


def run_child(what: str, env_extra: dict) -> dict:
    code = f"ROOT = {ROOT!r}\nWHAT = {what!r}\n" + CHILD
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    return json.loads(line[len("RESULT "):])


def test_sort_grid_barrier_timeout_is_reported():
    import hashed_gram_embedding_raw_b200 as E
    res = run_child("sort", {"ENGRAM_TEST_BARRIER_SPIN": "0"})
    assert res["flags"] & E.ENGRAM_DEVERR_SORT_TIMEOUT
    assert res["hash_ok"] and res["flags_after"] == 0


def test_ple_cross_warp_wait_timeout_is_reported():
    import hashed_gram_embedding_raw_b200 as E
    res = run_child("ple", {"ENGRAM_TEST_CROSS_WAIT_NS": "0"})
    assert res["flags"] & E.ENGRAM_DEVERR_COPY_TIMEOUT
    assert res["hash_ok"] and res["flags_after"] == 0


@pytest.mark.parametrize("what", ["sort", "ple"])
def test_normal_bounds_raise_nothing(what):
    res = run_child(what, {})
    assert res["flags"] == 0 and res["hash_ok"]
