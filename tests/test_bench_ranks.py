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


def _run_reference(env_extra, *extra):
    env = dict(os.environ, ENGRAM_REFERENCE_BUDGET_S="2", **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl",
                           "reference", "--workload", "tiny", "--steps", "2", "--warmup",
                           "3", *extra], capture_output=True, text=True, env=env, timeout=300)


def _one_line(r):
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    return json.loads(lines[0])


def test_reference_arm_prints_one_line():
    rec = _one_line(_run_reference({}))
    assert rec["impl"] == "reference" and rec["unit"] == "tokens/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] == 1
    assert rec["cpu_baseline"]["host_nproc"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["value"] == rec["value"]


def test_reference_arm_counts_the_tokens_it_processed():
    """The calibration asks for more tokens than the 128-token workload holds;
    the oracle caps the sample, and the line must count the capped sample, so
    value x ms_per_step equals one step's tokens and the config is the GPU
    arm's."""
    sys.path.insert(0, ROOT)
    import bench
    rec = _one_line(_run_reference({}))
    tokens = rec["config"]["tokens_per_step"]
    assert tokens == 128
    assert rec["sample_per_step"]["units"] == 128 and rec["sample_per_step"]["of"] == 128
    assert abs(rec["value"] * rec["ms_per_step"] / 1e3 - tokens) < 1e-6 * tokens
    assert abs(rec["sample_per_step"]["ms"] - rec["ms_per_step"]) < 1e-6 * rec["ms_per_step"]
    assert rec["config"] == json.loads(json.dumps(bench.workload_config("tiny", 1,
                                                                       "forward + backward")))


def test_reference_arm_stages_hash_and_gather():
    sys.path.insert(0, ROOT)
    import bench
    for stage, name in (("hash", "hash only (engram_hash)"),
                        ("gather", "gather only (engram_gather)")):
        rec = _one_line(_run_reference({}, "--stage", stage))
        assert rec["metric"] == bench.STAGE_METRICS[stage]
        assert rec["config"]["stage"] == name and rec["value"] > 0
        assert "timed: " + stage in rec["cpu_baseline"]["sample"]


def test_workload_config_records_head_constants():
    sys.path.insert(0, ROOT)
    import bench
    page = bench.workload_config("full", 1)["head_constants"]
    assert page["printed_heads"] == 8 and page["inferred_heads"] == 8
    assert len(page["vocab_sizes"]) == 16 and "inferred" in page["source"]
    seeded = bench.workload_config("b4x4096", 1)["head_constants"]
    assert seeded["prime_seed"] == 1001 and len(seeded["vocab_sizes"]) == 16
    assert "seeded" in seeded["source"]


def test_clock_sampler_summary_counts_timed_samples():
    sys.path.insert(0, ROOT)
    import bench
    import datetime
    clk = bench.ClockSampler("0")
    t = datetime.datetime(2026, 1, 1, 12, 0, 0)

    def row(dt, mhz, cap="Not Active"):
        ts = (t + datetime.timedelta(seconds=dt)).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        return (f"{ts}, 0, {mhz}, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, "
                f"{cap}")

    clk.lines = [row(0.00, 1800), row(0.10, 1965), row(0.20, 1965, "Active"), row(0.30, 1900)]
    base = t.timestamp()
    clk.mark_timed(base + 0.15, base + 0.25)
    s = clk.summary()
    assert s["samples"] == 4 and s["samples_in_timed_region"] == 1
    assert s["sm_mhz_timed_region"] == 1965 and s["sm_mhz_min"] == 1800
    assert s["reasons"] == ["sw_power_cap"] and s["sm_max_mhz"] == 1965


def test_reference_arm_other_ranks_exit_quietly():
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""
