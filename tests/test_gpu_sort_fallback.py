"""The backward sort's two forms on the same inputs, each in a child
process, compared bit for bit: the grid-wide sort in one cooperative launch
(the default) and the separate-launch form -- what a device without
cooperative launch runs: two launches per pass on 2,048-pair tiles -- forced
with ENGRAM_SORT_SEPARATE_LAUNCHES=1. A stable sort has one
result, so the distinct rows and their fp32 sums must be identical bit for
bit. The sizes cover one tile, a ragged single tile, many resident tiles and
more tiles than resident blocks; half the lookups hit a few hot rows. The
sort by head (engram_backward_heads) is compared the same way on the page's
head constants.
"""

import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
import numpy as np
import torch
sys.path.insert(0, sys.argv[1])
import hashed_gram_embedding_raw_b200 as E
rows = 320_001_536
out = {}
for n in (1, 1000, 65_536, 250_007, 2_000_003):
    rng = np.random.Generator(np.random.PCG64(n))
    idx = np.where(rng.random(n) < 0.5, rng.integers(0, 40, n),
                   rng.integers(0, rows, n)).astype(np.int32)
    dout = torch.randn(n, 16, generator=torch.Generator().manual_seed(n % 997))
    u, g, nu = E.engram_backward(torch.from_numpy(idx).cuda(), dout.cuda(), rows)
    U = int(nu.item())
    assert E.engram_get_device_error() == 0
    out["u%d" % n] = u[:U].cpu().numpy()
    out["g%d" % n] = g[:U].cpu().numpy()
from workloads import head_params, random_stream
import oracle
cfg = dict(head_params("full"), dim=16)
p = E.make_params(cfg)
for T, vocab in ((1, 2000), (63, 2000), (15_625, 2000), (65_536, 2000), (65_536, 248_320),
                 (40_000, 248_320), (65_537, 2000), (131_072, 2000)):
    ids, cu = random_stream(T, T, vocab, cfg["eos_id"], 0.01, nseq=1 + T // 4096)
    idx = oracle.hash_ids(ids, cu, cfg).astype(np.int32)
    dout = torch.randn(idx.size, 16, generator=torch.Generator().manual_seed(T % 997))
    u, g, nu = E.engram_backward_heads(p, torch.from_numpy(idx).cuda(), dout.cuda())
    U = int(nu.item())
    assert E.engram_get_device_error() == 0
    out["hu%d_%d" % (T, vocab)] = u[:U].cpu().numpy()
    out["hg%d_%d" % (T, vocab)] = g[:U].cpu().numpy()
np.savez(sys.argv[2], **out)
"""


def run_child(tmp_path, form: str):
    path = tmp_path / (form + ".npz")
    env = dict(os.environ, ENGRAM_SORT_SEPARATE_LAUNCHES="1" if form == "separate" else "0")
    subprocess.run([sys.executable, "-c", CHILD, ROOT, str(path)], env=env, check=True,
                   timeout=600)
    return np.load(path)


def test_sort_forms_agree_bit_for_bit(tmp_path):
    forms = {f: run_child(tmp_path, f) for f in ("default", "separate")}
    base = forms["default"]
    for name, got in forms.items():
        assert sorted(got.files) == sorted(base.files), name
        for k in base.files:
            assert np.array_equal(got[k], base[k]), (name, k)
