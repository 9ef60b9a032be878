"""Host-side multi-rank logic of bench.py on CPU (gloo, world size 2), and the
reference (CPU oracle) arm of the benchmark."""

import json
import os
import subprocess
import sys

import torch.multiprocessing as mp

from tests.conftest import ROOT


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, ws = bench.rank_env()
        bench.barrier()
        m = bench.max_over_ranks(10.0 + 3.5 * rank)
        q.put((r, lr, ws, m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 2000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 0, 2, 13.5), (1, 1, 2, 13.5)]


def test_max_over_ranks_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.25) == 4.25


def _run_reference(env_extra):
    env = dict(os.environ, ENGRAM_REFERENCE_BUDGET_S="2", **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl",
                           "reference", "--workload", "tiny", "--steps", "2", "--warmup",
                           "3"], capture_output=True, text=True, env=env, timeout=300)


def test_reference_arm_prints_one_line():
    r = _run_reference({})
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "tokens/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] == 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["value"] == rec["value"]


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""
