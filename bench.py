"""Benchmark of the Engram N-gram Embedding hot path on B200.

One step = the fused hash+gather forward (engram_hash_gather, writing the
[T, 16*160] rows and the [T, 16] indices) followed by the compact backward
(engram_backward_sort_heads + engram_backward_reduce: distinct rows and fp32
row gradients) over one batch of the named workload, all inputs resident in
HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload full]
    python bench.py --impl reference ...   # the CPU oracle, timed on this host
    python bench.py --stage hash ...       # engram_hash alone (L2 flushed between launches)
    python bench.py --stage gather ...     # engram_gather alone on the hash's indices
    python bench.py --stage fwd ...        # engram_hash_gather alone
    python bench.py --stage bwd ...        # the backward alone (sort + reduce)
    python bench.py --stage ple ...        # the PLE tail kernel on its own workload
    python bench.py --stage ple_bwd ...    # the PLE tail's backward on the same workload
    python bench.py --stage owner ...      # the owner-sharded table (NCCL all-to-alls)
    python bench.py --stage adam ...       # the sparse optimizer step on a table shard

Multi-GPU (torchrun, one rank per GPU): every rank holds its own table
replica and processes its own batch; no data-path collective exists, so the
run is weak scaling and the reported value is all ranks' tokens over the
slowest rank's device time. Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Engram tokens/s (fused hash+gather fwd, scatter bwd); achieved HBM GB/s vs peak"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ ranks

def rank_env():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the process group (identity alone)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------- peaks, clocks

def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples, every `interval_ms`, from
    before the warm-up to the end of the last measured pass. Each sample carries
    nvidia-smi's own timestamp, so the samples inside the timed region can be
    counted apart (mark_timed records its host-clock bounds)."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, interval_ms: int = 10):
        self.gpu_id, self.interval_ms, self.proc = gpu_id, interval_ms, None
        self.lines, self.timed = [], []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", f"-lms={self.interval_ms}"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)        # let the sampler come up before the measured work
        except OSError:
            self.proc = None
        return self

    def mark_timed(self, t0: float, t1: float):
        """Host wall-clock bounds (time.time()) of a timed region."""
        self.timed.append((t0, t1))

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    @staticmethod
    def _stamp(s: str):
        import datetime
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(s, fmt).timestamp()
            except ValueError:
                pass
        return None

    def summary(self):
        sm, mx, reasons, in_timed, sm_timed = [], None, set(), 0, []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 10:
                continue
            try:
                mhz = float(f[2])
                mx = float(f[3])
            except ValueError:
                continue
            sm.append(mhz)
            ts = self._stamp(f[0])
            if ts is not None and any(a - 0.02 <= ts <= b + 0.02 for a, b in self.timed):
                in_timed += 1
                sm_timed.append(mhz)
            for nm, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_mhz_min": min(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "samples_in_timed_region": in_timed,
                "sm_mhz_timed_region": statistics.median(sm_timed) if sm_timed else None,
                "interval_ms": self.interval_ms,
                "window": "from before the warm-up to the end of the last measured pass"}


def gpu_smi_id(torch, device) -> str:
    props = torch.cuda.get_device_properties(device)
    bus = getattr(props, "pci_bus_id", None)
    if bus is not None:
        dom = getattr(props, "pci_domain_id", 0)
        dev = getattr(props, "pci_device_id", 0)
        return f"{dom:08x}:{bus:02x}:{dev:02x}.0"
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    return vis.split(",")[device.index] if vis else str(device.index)


# -------------------------------------------------------- committed traffic

def source_digest(files) -> str:
    """Digest of the named kernel sources (file names under csrc/)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hashed_gram_embedding_raw_b200", "csrc")
    for name in sorted(files):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, units: float):
    """DRAM bytes per launch from profiles/dram_traffic.json, scaled to `units`
    (lookups or tokens): {"total", "read", "write", "read_overfetch"}, where
    read_overfetch = DRAM bytes read / algorithmic bytes read. None if absent or
    taken on other kernel sources (each record carries the digest of the
    sources its kernel is built from)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        k = rec["kernels"][kernel]
        if k["digest"] != source_digest(k["sources"]):
            return None
        out = {"total": k["dram_bytes_per_unit"] * units, "read": None, "write": None,
               "read_overfetch": None}
        if "read_bytes_per_unit" in k:
            out["read"] = k["read_bytes_per_unit"] * units
            out["write"] = k["write_bytes_per_unit"] * units
        if k.get("alg_read_bytes_per_unit"):
            out["read_overfetch"] = k["read_bytes_per_unit"] / k["alg_read_bytes_per_unit"]
        return out
    except (OSError, ValueError, KeyError, TypeError):
        return None


def traffic_fields(kernel: str, units: float) -> dict:
    """The roofline's traffic keys for a kernel (nulls when no current record)."""
    t = committed_traffic(kernel, units)
    return {"traffic": t["total"] if t else None,
            "traffic_read": t["read"] if t else None,
            "traffic_write": t["write"] if t else None,
            "read_overfetch": t["read_overfetch"] if t else None}


# ------------------------------------------------------ host, workload config

def host_info() -> dict:
    """This host's CPU, as the CPU-baseline figures report it."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.lower().startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        usable = len(os.sched_getaffinity(0))
    except AttributeError:
        usable = os.cpu_count()
    return {"host_nproc": usable, "host_logical_cpus": os.cpu_count(), "cpu_model": model}


def head_constants_record(name: str) -> dict:
    """Where the workload's hash constants come from, with their values."""
    from workloads import WORKLOADS, constants, head_params
    w, cfg = WORKLOADS[name], head_params(name)
    rec = {"multipliers": list(cfg["multipliers"]), "vocab_sizes": list(cfg["vocab_sizes"]),
           "eos_id": cfg["eos_id"], "fill_id": cfg["fill_id"]}
    if w.heads == "page":
        rec["source"] = ("page: multipliers, padded rows and the first 8 vocab sizes and "
                         "offsets printed; vocab sizes of heads 8-15 inferred (the next 8 "
                         "consecutive primes), offsets their running sums")
        rec["printed_heads"] = len(constants.PRINTED_VOCAB_SIZES)
        rec["inferred_heads"] = len(constants.INFERRED_VOCAB_SIZES)
    else:
        rec["source"] = (f"seeded stand-in: 16 distinct primes drawn from "
                         f"[{w.prime_range[0]}, {w.prime_range[1]}) by NumPy PCG64 seed "
                         f"{1000 + w.seed}, sorted, offsets their running sums; page multipliers")
        rec["prime_seed"] = 1000 + w.seed
    return rec


def workload_config(name: str, world: int, stage: str = "forward + backward") -> dict:
    """The `config` of a bench line: identical on the GPU arm and the reference
    arm of the same workload and stage."""
    from workloads import WORKLOADS, head_params, token_stream
    w, cfg = WORKLOADS[name], head_params(name)
    T = len(token_stream(name)[0])
    R = cfg["table_rows"]
    return {"workload": name, "stage": stage, "tokens_per_step": T,
            "tokens_per_step_per_gpu": T, "heads": 16, "dim": cfg["dim"], "table_rows": R,
            "table_dtype": w.dtype,
            "parallelism": f"replicas x{world} (own table and batch per GPU)",
            "l2": ("inputs larger than L2 (102.4 GB table; 336 MB out and dout)" if R > 1e8
                   else "per-step working set vs 126 MB L2: see table_rows"),
            "input_seed": w.seed, "inputs": w.description,
            "head_constants": head_constants_record(name)}


# ------------------------------------------------------------ CPU oracle leg

STAGE_NAMES = {"all": "forward + backward", "bwd": "backward only",
               "hash": "hash only (engram_hash)", "gather": "gather only (engram_gather)",
               "fwd": "fused forward only (engram_hash_gather)"}
ORACLE_PARTS = {"all": ("hash", "gather", "backward"), "bwd": ("backward",),
                "hash": ("hash",), "gather": ("gather",), "fwd": ("hash", "gather")}


def oracle_run(name: str, S: int, reps_seconds: float = 0.0, max_reps: int = 1,
               parts=("hash", "gather", "backward")):
    """Time the CPU oracle on the first S tokens of a workload (S is capped at
    the workload's length): the named parts of hash, gather from a host table
    holding the rows those lookups touch (staged untimed), and the row-gradient
    backward. Returns (tokens/s, seconds, reps, description, tokens per rep)."""
    import torch
    import oracle
    from workloads import WORKLOADS, head_params, host_dout, token_stream

    cfg = head_params(name)
    ids, cu = token_stream(name)
    S = min(S, len(ids))
    ids = np.ascontiguousarray(ids[:S])
    cu = np.concatenate([cu[cu < S], [S]]).astype(np.int32)
    H, D = 16, cfg["dim"]
    w = WORKLOADS[name]
    # untimed staging: the rows this sample touches, and its output gradient
    idx0 = oracle.hash_ids(ids, cu, cfg)
    uniq = np.unique(idx0)
    rng = np.random.Generator(np.random.PCG64(7))
    esize = 4 if w.dtype == "f32" else 2
    compact = rng.integers(0, 2 ** 16, size=(len(uniq), D * esize // 2), dtype=np.uint16)
    remap = np.searchsorted(uniq, idx0.reshape(-1))
    dout_raw = None
    if "backward" in parts:
        dout = host_dout(name, S * H, D, w.dtype)
        dout_raw = dout.numpy() if w.dtype == "f32" else \
            dout.view(torch.int16).numpy().view(np.uint16)
    code = oracle.F32 if w.dtype == "f32" else oracle.BF16
    oracle.lib()
    reps, t0 = 0, time.perf_counter()
    while True:
        idx = oracle.hash_ids(ids, cu, cfg) if "hash" in parts else idx0
        if "gather" in parts:
            out = oracle.gather(compact, remap)
            assert out.shape[0] == S * H
        if "backward" in parts:
            u, _ = oracle.backward(idx.reshape(-1), dout_raw, code)
            assert len(u) == len(uniq)
        reps += 1
        el = time.perf_counter() - t0
        if reps >= max_reps or el >= reps_seconds:
            break
    what = " + ".join(parts)
    desc = (f"first {S} of {len(token_stream(name)[0])} tokens of workload '{name}' "
            f"x {reps} rep(s), timed: {what}"
            + ("; gather from a host table of the "
               f"{len(uniq)} rows the sample touches (staged before timing)"
               if "gather" in parts else "")
            + "; single-threaded C oracle")
    return S * reps / el, el, reps, desc, S


def run_reference(args):
    """--impl reference: the oracle, as it stands, on this host's cores, on the
    GPU arm's metric, unit and config. Each step times a bounded sample of the
    step's work (the whole step when it fits the time budget); value = units
    processed / time, and ms_per_step = the time one whole step takes at that
    rate."""
    rank, _, world = rank_env()
    if rank != 0:
        return 0
    name, stage = args.workload, args.stage
    if stage == "adam":
        run, small, unit = adam_oracle_run, 2048, "rows/s"
        full = args.adam_touched
        config, metric, dtype = adam_config(args.adam_rows, args.adam_touched), ADAM_METRIC, "f64"
    elif stage in ("ple", "ple_bwd"):
        bwd = stage == "ple_bwd"
        run = lambda S: ple_oracle_run(S, backward=bwd)  # noqa: E731
        small, unit = 256, UNIT
        config = ple_config(args, world, bwd)
        full = config["tokens_per_step_per_gpu"]
        metric, dtype = (PLE_BWD_METRIC if bwd else PLE_METRIC), "f64"
    elif stage in ORACLE_PARTS:
        parts = ORACLE_PARTS[stage]
        run = lambda S: oracle_run(name, S, parts=parts)  # noqa: E731
        small, unit = 4096, UNIT
        config = workload_config(name, world, STAGE_NAMES[stage])
        full = config["tokens_per_step"]
        metric, dtype = STAGE_METRICS.get(stage, METRIC), "int64/f64"
    else:
        print(json.dumps({"impl": "reference", "unavailable":
                          f"stage {stage} has no oracle arm (its exchanges need several ranks)"}))
        return 0
    # calibrate, then size each step's sample so W + K steps take about the budget
    rate = run(small)[0]
    budget = float(os.environ.get("ENGRAM_REFERENCE_BUDGET_S", "120"))
    S = int(max(small, min(full, rate * budget / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        run(S)
    times, desc, done = [], "", 0
    for _ in range(args.steps):
        _, el, _, desc, got = run(S)
        times.append(el)
        done += got
    total = sum(times)
    value = done / total
    cores = 1
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * full / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": config,
        "sample_per_step": {"units": done // len(times), "of": full,
                            "ms": 1e3 * total / len(times)},
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": desc, **host_info()},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------- GPU leg

STAGE_METRICS = {
    "hash": ("Engram hash tokens/s (engram_hash alone: raw token IDs to 16 head row "
             "indices per token); achieved HBM GB/s vs peak"),
    "gather": ("Engram gather tokens/s (engram_gather alone: 16 row lookups of 160 bf16 "
               "per token from the hash's indices); achieved HBM GB/s vs peak"),
    "fwd": ("Engram forward tokens/s (engram_hash_gather alone: hash and 16 row lookups "
            "per token, rows and indices written); achieved HBM GB/s vs peak"),
}
L2_FLUSH_BYTES = 256 << 20     # twice the B200's 126 MB L2


def run_ours(args):
    """The GPU arm. --stage all (default): the step = engram_hash_gather +
    engram_backward_sort + engram_backward_reduce, captured once as a CUDA
    graph and replayed; bwd: the backward alone; hash / gather: engram_hash or
    engram_gather alone, each launch timed by its own events (the hash's
    working set fits in L2, so L2 is flushed between its launches)."""
    import torch
    import torch.distributed as dist

    import hashed_gram_embedding_raw_b200 as E
    from workloads import WORKLOADS, fill_device_table, head_params, host_dout, token_stream

    rank, local_rank, world = rank_env()
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=device,
                                timeout=datetime.timedelta(seconds=300))

    stage = args.stage
    name = args.workload
    w = WORKLOADS[name]
    cfg = head_params(name)
    params = E.make_params(cfg)
    ids_np, cu_np = token_stream(name)
    T, H, D, R = len(ids_np), params.heads, cfg["dim"], cfg["table_rows"]
    n = T * H
    tdtype = {"bf16": torch.bfloat16, "f32": torch.float32}[w.dtype]
    esize = 2 if w.dtype == "bf16" else 4
    fwd, bwd = stage == "all", stage in ("all", "bwd")
    gathers = stage in ("all", "gather", "fwd")

    table = None
    if gathers:
        table = torch.empty(R, D, dtype=tdtype, device=device)
        fill_device_table(table, w.seed)
    dout_h = host_dout(name, n, D, w.dtype).pin_memory() if bwd else None
    ws = (torch.empty(E.engram_backward_workspace_size(n, R, D), dtype=torch.uint8,
                      device=device) if bwd else None)
    per_launch = stage in ("hash", "gather", "fwd")
    flush = (torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
             if per_launch else None)
    bufs = [{
        "ids": torch.from_numpy(ids_np.copy()).to(device),
        "cu": torch.from_numpy(cu_np.copy()).to(device),
        "dout": dout_h.to(device) if bwd else None,
        "out": torch.empty(T, H * D, dtype=tdtype, device=device) if gathers else None,
        "idx": torch.empty(T, H, dtype=torch.int32, device=device),
        "uniq": torch.empty(n, dtype=torch.int32, device=device) if bwd else None,
        "grads": torch.empty(n, D, dtype=torch.float32, device=device) if bwd else None,
        "nu": torch.empty(1, dtype=torch.int32, device=device),
    } for _ in range(2)]
    stream = torch.cuda.Stream(device)
    if stage in ("bwd", "gather"):   # these take the hash's indices
        for b in bufs:
            E.engram_hash(params, b["ids"], b["cu"], out_idx=b["idx"], stream=stream)

    def step(ev=None, b=None):
        b = bufs[0] if b is None else b
        if stage == "hash":
            E.engram_hash(params, b["ids"], b["cu"], out_idx=b["idx"], stream=stream)
            return
        if stage == "gather":
            E.engram_gather(table, b["idx"].view(-1), out=b["out"].view(n, D), stream=stream)
            return
        if stage == "fwd":
            E.engram_hash_gather(params, b["ids"], table, cu_seqlens=b["cu"], out=b["out"],
                                 out_idx=b["idx"], stream=stream)
            return
        if ev is not None:
            ev[0].record(stream)
        if fwd:
            E.engram_hash_gather(params, b["ids"], table, cu_seqlens=b["cu"], out=b["out"],
                                 out_idx=b["idx"], stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if args.bwd_sort == "heads":
            E.engram_backward_sort_heads(params, b["idx"], ws, stream=stream)
        else:
            E.engram_backward_sort(b["idx"].view(-1), R, D, ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        E.engram_backward_reduce(n, R, b["dout"], b["uniq"], b["grads"], b["nu"], ws,
                                 stream=stream)
        if ev is not None:
            ev[3].record(stream)

    def flush_l2():
        # a read of twice the L2's size: the lines it leaves are clean, so the
        # next launch neither finds its inputs in L2 nor pays for writing back
        # another kernel's dirty lines
        if flush is not None:
            with torch.cuda.stream(stream):
                flush.sum()

    clk = ClockSampler(gpu_smi_id(torch, device))
    clk.__enter__()
    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize(device)
    if E.engram_get_device_error(stream):
        raise RuntimeError("device error flag set during warm-up")
    U = int(bufs[0]["nu"].item()) if bwd else None

    K = args.steps
    graph, launches_per_step = None, None
    if per_launch:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
        launches0 = E.engram_launch_count()
        barrier(device)
        torch.cuda.synchronize(device)
        h0 = time.time()
        for e in evs:
            flush_l2()
            e[0].record(stream)
            step()
            e[1].record(stream)
        torch.cuda.synchronize(device)
        clk.mark_timed(h0, time.time())
        barrier(device)
        launches = E.engram_launch_count() - launches0
        per = [e[0].elapsed_time(e[1]) for e in evs]
        local_ms = sum(per)
        timed_as = ("sum of per-launch CUDA-event times, eager launches; L2 flushed "
                    "between launches by a 256 MB read (not timed), which also writes "
                    "back the previous launch's dirty lines outside the timed region")
    else:
        # one step captured as a CUDA graph and replayed (the library's calls
        # need no host synchronisation), or eager launches
        if args.graph:
            graph = torch.cuda.CUDAGraph()
            c0 = E.engram_launch_count()
            with torch.cuda.graph(graph, stream=stream):
                step()
            launches_per_step = E.engram_launch_count() - c0

            def timed_step():
                with torch.cuda.stream(stream):
                    graph.replay()
        else:
            timed_step = step
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        timed_step()                       # first replay uploads the graph
        torch.cuda.synchronize(device)
        launches0 = E.engram_launch_count()
        barrier(device)
        torch.cuda.synchronize(device)
        h0 = time.time()
        t_start.record(stream)
        for k in range(K):
            timed_step()
        t_end.record(stream)
        torch.cuda.synchronize(device)
        clk.mark_timed(h0, time.time())
        barrier(device)
        launches = (launches_per_step * K if args.graph
                    else E.engram_launch_count() - launches0)
        local_ms = t_start.elapsed_time(t_end)
        per = None
        timed_as = ("CUDA graph of one step, replayed" if args.graph else "eager launches")
    total_ms = max_over_ranks(local_ms, device)

    # per-stage times of the step: a separate eager pass with events between
    # the stages (kept out of the timed steps above)
    if not per_launch:
        KS = max(1, min(K, 50))
        sevs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(KS)]
        for k in range(KS):
            step(sevs[k])
        torch.cuda.synchronize(device)
        fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in sevs)
        sort_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in sevs)
        red_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in sevs)

    # ---- end to end through the public API with host buffers: every step
    # copies its inputs in from pinned host memory and its results back out.
    # Three streams pipeline consecutive steps (copy-in, compute, copy-out,
    # two sets of device buffers), so step k's results travel to the host
    # while step k+1 computes and PCIe carries both directions at once.
    in_names = {"all": ["ids", "cu", "dout"], "bwd": ["idx", "dout"],
                "hash": ["ids", "cu"], "gather": ["idx"], "fwd": ["ids", "cu"]}[stage]
    out_fixed = {"all": ["out", "nu"], "bwd": ["nu"], "hash": ["idx"], "gather": ["out"],
                 "fwd": ["out", "idx"]}[stage]

    def run_e2e(resident_rows: bool):
        """resident_rows (stage all only): read back num_unique alone and leave
        out and the row gradients on the device."""
        e2e_steps = max(1, min(K, args.e2e_steps))
        src = {"ids": torch.from_numpy(ids_np.copy()), "cu": torch.from_numpy(cu_np.copy()),
               "dout": dout_h, "idx": bufs[0]["idx"].cpu()}
        host_in = {k: src[k] if src[k].is_pinned() else src[k].pin_memory() for k in in_names}
        outs = ["nu"] if resident_rows else out_fixed
        host = [{k: torch.empty_like(bufs[0][k], device="cpu").pin_memory() for k in outs}
                for _ in range(2)]
        if bwd and not resident_rows:
            for hb in host:
                hb["uniq"] = torch.empty(n, dtype=torch.int32).pin_memory()
                hb["grads"] = torch.empty(n, D, dtype=torch.float32).pin_memory()
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        in_done = [ev() for _ in range(e2e_steps)]
        comp_done = [ev() for _ in range(e2e_steps)]
        fixed_done = [ev() for _ in range(e2e_steps)]
        out_done = [ev() for _ in range(e2e_steps)]
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h_bytes = [0] * e2e_steps

        def drain(k):
            # step k's rows: the host needs num_unique before copying them out
            hb, b = host[k % 2], bufs[k % 2]
            d2h = sum(hb[x].numel() * hb[x].element_size() for x in outs)
            if bwd and not resident_rows:
                fixed_done[k].synchronize()
                u = int(hb["nu"].item())
                with torch.cuda.stream(s_out):
                    hb["uniq"][:u].copy_(b["uniq"][:u], non_blocking=True)
                    hb["grads"][:u].copy_(b["grads"][:u], non_blocking=True)
                d2h += u * 4 + u * D * 4
            with torch.cuda.stream(s_out):
                out_done[k].record(s_out)
            d2h_bytes[k] = d2h

        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(device)
        torch.cuda.synchronize(device)
        h0 = time.time()
        e0.record(s_in)
        for k in range(e2e_steps):
            b, hb = bufs[k % 2], host[k % 2]
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(comp_done[k - 2])  # inputs of buffer set k%2 free
                for x in in_names:
                    b[x].copy_(host_in[x], non_blocking=True)
                in_done[k].record(s_in)
            stream.wait_event(in_done[k])
            if k >= 2:
                stream.wait_event(out_done[k - 2])     # outputs of buffer set k%2 copied out
            step(b=b)
            comp_done[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[k])
                for x in outs:
                    hb[x].copy_(b[x], non_blocking=True)
                fixed_done[k].record(s_out)
            if k >= 1:
                drain(k - 1)
        drain(e2e_steps - 1)
        e1.record(s_out)
        torch.cuda.synchronize(device)
        clk.mark_timed(h0, time.time())
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), device)
        barrier(device)
        rb = outs + (["uniq_rows[:U]", "row_grads[:U]"] if bwd and not resident_rows else [])
        return {"value": world * T * e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": int(statistics.mean(d2h_bytes)),
                "steps": e2e_steps, "inputs": in_names, "readback": rb,
                "pipeline": "copy-in / compute / copy-out streams, two buffer sets"}

    e2e = run_e2e(False)
    e2e_resident = run_e2e(True) if fwd else None
    clk.__exit__(None, None, None)

    if E.engram_get_device_error(stream):
        raise RuntimeError("device error flag set during timing")

    # ---- numbers
    value = world * T * K / (total_ms / 1e3)
    peak, peak_kind = hbm_peak()
    fwd_bytes = T * (4 + 2 * H * D * esize + H * 4)
    hash_bytes = T * (4 + H * 4) + cu_np.size * 4
    gather_bytes = n * (4 + 2 * D * esize)
    stages = {}
    if per_launch:
        kname = {"hash": "hash_kernel<3, 8>", "gather": "gather_kernel<20>",
                 "fwd": "hash_gather_kernel<3, 8, 20>"}[stage]
        dom_bytes = {"hash": hash_bytes, "gather": gather_bytes, "fwd": fwd_bytes}[stage]
        dom_ms = statistics.mean(per)
        stages[stage] = {"ms": dom_ms, "ms_min": min(per), "ms_max": max(per),
                         "alg_bytes": dom_bytes, "gbs": dom_bytes / dom_ms / 1e6,
                         "frac": dom_bytes / dom_ms / 1e6 / peak}
        dom, tkey, tunits = kname, kname.split("<")[0], (n if stage == "gather" else T)
    else:
        red_bytes = n * D * esize + U * (4 + D * 4)
        bwd_bytes = n * 4 + red_bytes
        if fwd:
            stages["fwd_hash_gather"] = {"ms": fwd_ms, "alg_bytes": fwd_bytes,
                                         "gbs": fwd_bytes / max(fwd_ms, 1e-9) / 1e6,
                                         "frac": fwd_bytes / max(fwd_ms, 1e-9) / 1e6 / peak}
        stages["bwd_sort"] = {"ms": sort_ms}
        stages["bwd_reduce"] = {"ms": red_ms, "alg_bytes": red_bytes,
                                "gbs": red_bytes / red_ms / 1e6,
                                "frac": red_bytes / red_ms / 1e6 / peak}
        stages["bwd_total"] = {"ms": sort_ms + red_ms, "alg_bytes": bwd_bytes,
                               "gbs": bwd_bytes / (sort_ms + red_ms) / 1e6,
                               "frac": bwd_bytes / (sort_ms + red_ms) / 1e6 / peak}
        stages["num_unique"] = U
        # dominant kernel: the fused forward unless the reduce stage takes longer
        if fwd and fwd_ms >= red_ms:
            dom, dom_ms, dom_bytes, tkey, tunits = ("hash_gather_kernel<3, 8, 20>", fwd_ms,
                                                   fwd_bytes, "hash_gather_kernel", T)
        else:
            dom, dom_ms, dom_bytes, tkey, tunits = (
                "segment reduce stage (seg_count + seg_reduce + seg_fixup; seg_reduce "
                "dominates)", red_ms, red_bytes, "seg_reduce", n)
    achieved = dom_bytes / dom_ms / 1e6
    config = workload_config(name, world, STAGE_NAMES[stage])
    line = {
        "metric": STAGE_METRICS.get(stage, METRIC), "value": value, "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": config, "timed_as": timed_as,
        "backward_sort": (None if not bwd else
                          "by head (engram_backward_sort_heads)" if args.bwd_sort == "heads"
                          else "whole row range (engram_backward_sort)"),
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
                     "alg_bytes_per_launch": dom_bytes, **traffic_fields(tkey, tunits)},
        "stages": stages,
        "e2e": e2e,
        "e2e_resident_outputs": e2e_resident,
        "gpu_launches": launches,
    }
    if world == 1 and not args.no_cpu_baseline:
        v, el, reps, desc, _ = oracle_run(name, T, reps_seconds=args.cpu_seconds, max_reps=8,
                                          parts=ORACLE_PARTS[stage])
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                                "sample": desc, "seconds": el, **host_info()}
    else:
        line["cpu_baseline"] = None
    line["clocks"] = clk.summary()
    if rank == 0:
        print(json.dumps(line), flush=True)
    graph = None  # no graph outlives the process group
    if world > 1:
        dist.destroy_process_group()
    return 0


# --------------------------------------------------------- PLE tail stage

PLE_METRIC = ("PLE tail tokens/s (grouped RMS norm + causal depthwise conv + SiLU + residual "
              "over hc_count x hidden channels); achieved HBM GB/s vs peak")


PLE_BWD_METRIC = ("PLE tail backward tokens/s (dx and the norm-scale, conv-weight and bias "
                  "gradients of norm + causal depthwise conv + SiLU + residual over hc_count x "
                  "hidden channels); achieved HBM GB/s vs peak")


def ple_oracle_run(S: int, reps_seconds: float = 0.0, max_reps: int = 1,
                   backward: bool = False):
    """Time the CPU oracle of the PLE tail (or of its backward) on S tokens (one
    sequence) of the page's channel shape. Returns (tokens/s, seconds, reps,
    description)."""
    import oracle
    from workloads import PLE_SHAPES, ple_inputs

    s = PLE_SHAPES["ple_full"]
    x, nw, w, b = ple_inputs(S, s.channels, s.kernel, s.seed, s.dtype)
    dout = np.random.default_rng(s.seed).standard_normal((S, s.channels)) if backward else None
    oracle.lib()
    reps, t0 = 0, time.perf_counter()
    while True:
        if backward:
            out = oracle.short_conv_backward(x, oracle.BF16, None, w, dout, dilation=s.dilation,
                                             group=s.group, norm_w=nw, bias=b,
                                             wdtype=oracle.BF16)[0]
        else:
            out = oracle.short_conv(x, oracle.BF16, None, w, dilation=s.dilation,
                                    group=s.group, norm_w=nw, bias=b, wdtype=oracle.BF16)
        reps += 1
        el = time.perf_counter() - t0
        if reps >= max_reps or el >= reps_seconds:
            break
    assert out.shape == (S, s.channels)
    desc = (f"{S} tokens x {s.channels} channels (one sequence, the page's 4 x 2,560 "
            f"branches, kernel {s.kernel}, dilation {s.dilation}) x {reps} rep(s); "
            f"single-threaded C oracle in fp64{' (backward)' if backward else ''}")
    return S * reps / el, el, reps, desc, S


def ple_shape(args):
    """(shape, tokens, rows) of the PLE stages: the full workload's batch, or
    --ple-tokens worth of whole 4,096-token rows."""
    from workloads import PLE_SHAPES
    s = PLE_SHAPES["ple_full"]
    batch = max(1, args.ple_tokens // s.seq_len) if args.ple_tokens else s.batch
    return s, batch * s.seq_len, batch


def ple_config(args, world: int, backward: bool) -> dict:
    """`config` of the PLE stages, identical on both arms."""
    s, T, batch = ple_shape(args)
    C = s.channels
    return {"workload": "ple_full_bwd" if backward else "ple_full",
            "tokens_per_step": T, "tokens_per_step_per_gpu": T, "channels": C,
            "branches": s.branches, "group": s.group, "kernel": s.kernel,
            "dilation": s.dilation, "flags": "norm + silu + residual",
            "cu_seqlens": f"{batch} rows", "input_seed": 5000 + s.seed,
            "parallelism": f"replicas x{world} (own batch per GPU)",
            "l2": (f"inputs larger than L2 ({T * C * 2 * (2 if backward else 1) / 1e9:.2f} "
                   f"GB in, {T * C * 2 / 1e9:.2f} GB out)"),
            **({"inverse_rms": ("the forward's, saved (made before timing)"
                                if getattr(args, "ple_inv", "computed") == "saved"
                                else "computed by the backward")} if backward else {})}


def adam_config(R: int, U: int) -> dict:
    """`config` of the optimizer stage, identical on both arms."""
    return {"workload": "adam_shard" if (R, U) == (ADAM_ROWS, ADAM_TOUCHED)
            else f"adam_{R}x{ADAM_DIM}_touch{U}", "table_rows": R, "dim": ADAM_DIM,
            "touched_rows": U, "table_dtype": "bf16", "moments": "f32", "lr": 1e-3,
            "weight_decay": 0.01,
            "l2": "inputs larger than L2 (12.8 GB table, 51.2 GB moments, random rows)"}


def run_ple(args, backward: bool = False):
    """--stage ple: engram_ple_short_conv on the page's PLE shape at the full
    workload's batch (16 x 4,096 tokens, C = 4 x 2,560 bf16); --stage ple_bwd:
    engram_ple_short_conv_backward (dx and the weight gradients, two launches)
    on the same shape with a bf16 dout."""
    import torch

    import hashed_gram_embedding_raw_b200 as E
    from workloads import ple_inputs, row_bounds

    rank, local_rank, world = rank_env()
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device,
                                timeout=datetime.timedelta(seconds=300))
    s, T, batch = ple_shape(args)
    C, G, K, d = s.channels, s.group, s.kernel, s.dilation
    g = torch.Generator(device=device).manual_seed(5000 + s.seed)
    x = torch.randn((T, C), generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)
    _, nw_h, w_h, b_h = ple_inputs(1, C, K, s.seed, s.dtype)

    def bf(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)

    nw, w, b = bf(nw_h), bf(w_h), bf(b_h)
    cu = torch.from_numpy(row_bounds(batch, s.seq_len)).to(device)
    out = torch.empty_like(x)
    stream = torch.cuda.Stream(device)
    inv = None
    if backward:
        dout = torch.randn((T, C), generator=g, device=device).to(torch.bfloat16)
        dnw, db = torch.empty(C, device=device), torch.empty(C, device=device)
        dw = torch.empty((C, K), device=device)
        ws = torch.empty(E.engram_ple_short_conv_backward_workspace_size(C, G, K, d, T),
                         dtype=torch.uint8, device=device)
        if args.ple_inv == "saved":
            # the forward's saved inverse RMS, as training has it (untimed)
            inv = torch.empty((T, C // G), device=device)
            E.engram_ple_short_conv(x, w, dilation=d, group_size=G, cu_seqlens=cu,
                                    norm_weight=nw, conv_bias=b, out=out, inv_rms=inv)
            torch.cuda.synchronize(device)

    def step(xx=x, oo=out, gg=None):
        if backward:
            E.engram_ple_short_conv_backward(
                xx, w, dout if gg is None else gg, dilation=d, group_size=G, cu_seqlens=cu,
                norm_weight=nw, conv_bias=b, dx=oo, dnorm_weight=dnw, dconv_weight=dw,
                dconv_bias=db, workspace=ws, inv_rms=inv, stream=stream)
        else:
            E.engram_ple_short_conv(xx, w, dilation=d, group_size=G, cu_seqlens=cu,
                                    norm_weight=nw, conv_bias=b, out=oo, stream=stream)

    clk = ClockSampler(gpu_smi_id(torch, device))
    clk.__enter__()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if E.engram_get_device_error(stream):
        raise RuntimeError("device error flag set during warm-up")
    Ksteps = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(Ksteps)]
    launches0 = E.engram_launch_count()
    barrier(device)
    torch.cuda.synchronize(device)
    h0 = time.time()
    for e in evs:
        e[0].record(stream)
        step()
        e[1].record(stream)
    torch.cuda.synchronize(device)
    clk.mark_timed(h0, time.time())
    barrier(device)
    launches = E.engram_launch_count() - launches0
    per = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = max_over_ranks(evs[0][0].elapsed_time(evs[-1][1]), device)
    kern_ms = statistics.mean(per)

    # end to end through the public call with host buffers: x (and dout) in
    # from pinned memory, out (dx and the weight gradients) back, copy-in /
    # compute / copy-out overlapped on three streams
    e2e_steps = max(1, min(Ksteps, args.e2e_steps))
    x_h = x.cpu().pin_memory()
    g_h = dout.cpu().pin_memory() if backward else None
    out_h = [torch.empty_like(x_h).pin_memory() for _ in range(2)]
    wg_d = [dnw, dw, db] if backward else []
    wg_h = [[torch.empty_like(t, device="cpu").pin_memory() for t in wg_d] for _ in range(2)]
    xd = [x, torch.empty_like(x)]
    gd = [dout, torch.empty_like(dout)] if backward else [None, None]
    od = [out, torch.empty_like(out)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    in_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    comp_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    out_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    h0 = time.time()
    e0.record(s_in)
    for k in range(e2e_steps):
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(comp_done[k - 2])
            xd[k % 2].copy_(x_h, non_blocking=True)
            if backward:
                gd[k % 2].copy_(g_h, non_blocking=True)
            in_done[k].record(s_in)
        stream.wait_event(in_done[k])
        if k >= 2:
            stream.wait_event(out_done[k - 2])
        step(xd[k % 2], od[k % 2], gd[k % 2])
        comp_done[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            out_h[k % 2].copy_(od[k % 2], non_blocking=True)
            for hh, dd in zip(wg_h[k % 2], wg_d):
                hh.copy_(dd, non_blocking=True)
            out_done[k].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize(device)
    clk.mark_timed(h0, time.time())
    clk.__exit__(None, None, None)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device)
    if E.engram_get_device_error(stream):
        raise RuntimeError("device error flag set during timing")

    peak, peak_kind = hbm_peak()
    if backward:   # x, dout in; dx out; weights in; fp32 weight gradients out
        alg = T * C * 2 * 3 + C * (K + 2) * 2 + C * (K + 2) * 4 + cu.numel() * 4
        if inv is not None:
            alg += inv.numel() * 4
        kname = "short_conv_bwd_kernel<bf16,bf16> + conv_bwd_reduce_kernel (one call)"
        tname = "short_conv_bwd_kernel"
    else:
        alg = T * C * 2 * 2 + C * (K + 2) * 2 + cu.numel() * 4
        kname = "short_conv_cls_kernel<bf16,bf16,4>"
        tname = "short_conv_cls_kernel"
    achieved = alg / kern_ms / 1e6
    line = {
        "metric": PLE_BWD_METRIC if backward else PLE_METRIC,
        "value": world * T * Ksteps / (total_ms / 1e3), "unit": UNIT,
        "n_gpus": world, "steps": Ksteps, "warmup": args.warmup,
        "ms_per_step": total_ms / Ksteps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": ple_config(args, world, backward),
        "timed_as": "per-launch CUDA events, eager launches back to back",
        "roofline": {"kernel": kname, "bound": "hbm",
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": achieved / peak,
                     "alg_bytes_per_launch": alg, **traffic_fields(tname, T)},
        "stages": {("ple_short_conv_backward" if backward else "ple_short_conv"): {
            "ms": kern_ms, "alg_bytes": alg, "gbs": achieved, "frac": achieved / peak,
            "ms_min": min(per), "ms_max": max(per)}},
        "e2e": {"value": world * T * e2e_steps / (e2e_ms / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": x_h.numel() * 2 * (2 if backward else 1),
                "d2h_bytes_per_step": x_h.numel() * 2 + sum(t.numel() * 4 for t in wg_d),
                "steps": e2e_steps,
                "pipeline": "copy-in / compute / copy-out streams, two buffer sets"},
        "gpu_launches": launches,
    }
    if world == 1 and not args.no_cpu_baseline:
        rate = ple_oracle_run(256, backward=backward)[0]
        S = int(max(256, min(16384, rate * args.cpu_seconds)))
        v, el, reps, desc, _ = ple_oracle_run(S, backward=backward)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
                                "sample": desc, "seconds": el, **host_info()}
    else:
        line["cpu_baseline"] = None
    line["clocks"] = clk.summary()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------ optimizer stage

ADAM_METRIC = ("Sparse AdamW rows/s (lazy update of the touched rows of a 40,000,192 x 160 bf16 "
               "table shard with fp32 moments); achieved HBM GB/s vs peak")
ADAM_ROWS = 40_000_192        # one eighth of the 320,001,536 padded rows: an 8-way owner shard
ADAM_TOUCHED = 1 << 20        # rows one step updates (about one full-workload backward)
ADAM_DIM = 160
ADAM_BYTES_PER_ROW = 4 + 640 + 2 * 2 * 640 + 2 * 320   # id, grad, m and v r/w, bf16 p r/w


def adam_oracle_run(U: int, reps_seconds: float = 0.0, max_reps: int = 1):
    """Time the CPU oracle's optimizer step on U rows (a U-row table with every
    row touched). Returns (rows/s, seconds, reps, description)."""
    import oracle
    rng = np.random.default_rng(9)
    p = rng.standard_normal((U, ADAM_DIM))
    m = np.zeros_like(p)
    v = np.zeros_like(p)
    rows = np.arange(U, dtype=np.int64)
    g = rng.standard_normal((U, ADAM_DIM)).astype(np.float32)
    oracle.lib()
    reps, t0 = 0, time.perf_counter()
    while True:
        p, m, v = oracle.sparse_adam(p, m, v, rows, g, lr=1e-3, weight_decay=0.01,
                                     step=reps + 1)
        reps += 1
        el = time.perf_counter() - t0
        if reps >= max_reps or el >= reps_seconds:
            break
    desc = (f"{U} rows x {ADAM_DIM} columns, all touched, x {reps} rep(s) (array copies "
            f"included); single-threaded C oracle in fp64")
    return U * reps / el, el, reps, desc, U


def run_adam(args):
    """--stage adam: engram_sparse_adam on an 8-way owner shard of the page's
    table with a full backward's worth of touched rows."""
    import torch

    import hashed_gram_embedding_raw_b200 as E

    rank, local_rank, world = rank_env()
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", device_id=device,
                                timeout=datetime.timedelta(seconds=300))
    R, D, U = args.adam_rows, ADAM_DIM, args.adam_touched
    if not 0 < U <= R:
        raise ValueError("need 0 < --adam-touched <= --adam-rows")
    g = torch.Generator(device=device).manual_seed(8000 + rank)
    table = torch.empty((R, D), dtype=torch.bfloat16, device=device)
    for r0 in range(0, R, 1 << 22):  # chunked fill keeps the fp32 temporary small
        r1 = min(R, r0 + (1 << 22))
        table[r0:r1] = (0.02 * torch.randn((r1 - r0, D), generator=g, device=device)).to(
            torch.bfloat16)
    m = torch.zeros((R, D), dtype=torch.float32, device=device)
    v = torch.zeros((R, D), dtype=torch.float32, device=device)
    rows = torch.randperm(R, generator=g, device=device)[:U].sort().values.to(torch.int32)
    grads = torch.randn((U, D), generator=g, device=device)
    nu = torch.tensor([U], dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device)
    step_no = [0]

    def step(rr=rows, gg=grads, n=nu):
        step_no[0] += 1
        E.engram_sparse_adam(table, m, v, rr, gg, n, lr=1e-3, weight_decay=0.01,
                             step=step_no[0], stream=stream)

    clk = ClockSampler(gpu_smi_id(torch, device))
    clk.__enter__()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if E.engram_get_device_error(stream):
        raise RuntimeError("device error flag set during warm-up")
    K = args.steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(K)]
    launches0 = E.engram_launch_count()
    barrier(device)
    torch.cuda.synchronize(device)
    h0 = time.time()
    for e in evs:
        e[0].record(stream)
        step()
        e[1].record(stream)
    torch.cuda.synchronize(device)
    clk.mark_timed(h0, time.time())
    barrier(device)
    launches = E.engram_launch_count() - launches0
    per = [e[0].elapsed_time(e[1]) for e in evs]
    total_ms = max_over_ranks(evs[0][0].elapsed_time(evs[-1][1]), device)
    kern_ms = statistics.mean(per)

    # end to end: the step's rows and gradients in from pinned memory, the step,
    # and the updated rows (engram_gather) back out, over three streams
    e2e_steps = max(1, min(K, args.e2e_steps))
    rows_h = rows.cpu().pin_memory()
    grads_h = grads.cpu().pin_memory()
    out_h = [torch.empty((U, D), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    rd = [rows, torch.empty_like(rows)]
    gd = [grads, torch.empty_like(grads)]
    od = [torch.empty((U, D), dtype=torch.bfloat16, device=device) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    in_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    comp_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    out_done = [torch.cuda.Event() for _ in range(e2e_steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize(device)
    h0 = time.time()
    e0.record(s_in)
    for k in range(e2e_steps):
        b = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(comp_done[k - 2])
            rd[b].copy_(rows_h, non_blocking=True)
            gd[b].copy_(grads_h, non_blocking=True)
            in_done[k].record(s_in)
        stream.wait_event(in_done[k])
        if k >= 2:
            stream.wait_event(out_done[k - 2])
        step(rd[b], gd[b])
        E.engram_gather(table, rd[b], out=od[b], stream=stream)
        comp_done[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[k])
            out_h[b].copy_(od[b], non_blocking=True)
            out_done[k].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize(device)
    clk.mark_timed(h0, time.time())
    clk.__exit__(None, None, None)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), device)
    if E.engram_get_device_error(stream):
        raise RuntimeError("device error flag set during timing")

    peak, peak_kind = hbm_peak()
    alg = U * ADAM_BYTES_PER_ROW
    achieved = alg / kern_ms / 1e6
    line = {
        "metric": ADAM_METRIC, "value": world * U * K / (total_ms / 1e3), "unit": "rows/s",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/f32",
        "data": "synthetic",
        "config": adam_config(R, U),
        "timed_as": "per-launch CUDA events, eager launches back to back",
        "roofline": {"kernel": "sparse_adam_kernel<bf16,40>", "bound": "hbm",
                     "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": achieved / peak,
                     "alg_bytes_per_launch": alg, **traffic_fields("sparse_adam_kernel", U)},
        "stages": {"sparse_adam": {"ms": kern_ms, "alg_bytes": alg, "gbs": achieved,
                                   "frac": achieved / peak, "ms_min": min(per),
                                   "ms_max": max(per)}},
        "e2e": {"value": world * U * e2e_steps / (e2e_ms / 1e3), "unit": "rows/s",
                "h2d_bytes_per_step": rows_h.numel() * 4 + grads_h.numel() * 4,
                "d2h_bytes_per_step": U * D * 2, "steps": e2e_steps,
                "pipeline": "copy-in / step + gather of the updated rows / copy-out streams"},
        "gpu_launches": launches,
    }
    if world == 1 and not args.no_cpu_baseline:
        rate = adam_oracle_run(2048)[0]
        n = int(max(2048, min(1 << 18, rate * args.cpu_seconds)))
        val, el, reps, desc, _ = adam_oracle_run(n)
        line["cpu_baseline"] = {"value": val, "unit": "rows/s", "cores": 1, "kind": "oracle",
                                "sample": desc, "seconds": el, **host_info()}
    else:
        line["cpu_baseline"] = None
    line["clocks"] = clk.summary()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ------------------------------------------------- owner-sharded stage

OWNER_METRIC = ("Engram tokens/s through the owner-sharded table (hash, owner grouping, "
                "all-to-all of rows and values, owner lookup, request-order restore; backward "
                "routed to the owners and reduced there)")


def run_owner(args):
    """--stage owner: the page's owner-sharded lookup and backward on the full
    workload, every rank holding 1/N of the 320,001,536-row table and
    requesting its own 16 x 4,096-token batch; the exchanges are NCCL
    all-to-alls (a group of one rank when N = 1)."""
    import datetime

    import torch
    import torch.distributed as dist

    import hashed_gram_embedding_raw_b200 as E
    from hashed_gram_embedding_raw_b200 import owner
    from workloads import WORKLOADS, fill_device_table, head_params, host_dout, token_stream

    rank, local_rank, world = rank_env()
    assert torch.cuda.is_available(), "bench.py needs a CUDA device"
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if world > 1:
        dist.init_process_group("nccl", device_id=device,
                                timeout=datetime.timedelta(seconds=300))
    else:
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        store = dist.TCPStore("127.0.0.1", port, 1, True,
                              timeout=datetime.timedelta(seconds=60))
        dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=device,
                                timeout=datetime.timedelta(seconds=300))
    name = args.workload
    w = WORKLOADS[name]
    cfg = head_params(name)
    params = E.make_params(cfg)
    R, D, H = cfg["table_rows"], cfg["dim"], params.heads
    rpo = owner.rows_per_owner(params, world)
    tdtype = {"bf16": torch.bfloat16, "f32": torch.float32}[w.dtype]
    shard = torch.empty((rpo, D), dtype=tdtype, device=device)
    fill_device_table(shard, w.seed + rank)
    ids_np, cu_np = token_stream(name)
    T = len(ids_np)
    ids = torch.from_numpy(ids_np.copy()).to(device)
    cu = torch.from_numpy(cu_np.copy()).to(device)
    dout = host_dout(name, T * H, D, w.dtype, seed_offset=rank).to(device)

    capacity = owner.agree_capacity(params, world, ids, cu)

    def step():
        out, routing = owner.run_collective(
            owner.forward_steps(params, shard, world, ids, cu, capacity=capacity))
        return owner.run_collective(owner.backward_steps(params, world, routing, dout))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if E.engram_get_device_error():
        raise RuntimeError("device error flag set during warm-up")
    K = args.steps
    stream = torch.cuda.current_stream(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = E.engram_launch_count()
    barrier(device)
    torch.cuda.synchronize(device)
    with ClockSampler(gpu_smi_id(torch, device)) as clk:
        h0 = time.time()
        e0.record(stream)
        for _ in range(K):
            step()
        e1.record(stream)
        torch.cuda.synchronize(device)
        clk.mark_timed(h0, time.time())
    barrier(device)
    launches = E.engram_launch_count() - launches0
    total_ms = max_over_ranks(e0.elapsed_time(e1), device)
    if E.engram_get_device_error():
        raise RuntimeError("device error flag set during timing")
    esize = 2 if w.dtype == "bf16" else 4
    line = {
        "metric": OWNER_METRIC, "value": world * T * K / (total_ms / 1e3), "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": total_ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": name + "_owner", "tokens_per_step_per_gpu": T,
                   "owners": world, "rows_per_owner": rpo,
                   "exchange": "NCCL all_to_all_single, equal splits of a fixed capacity",
                   "capacity": capacity,
                   "all_to_all_bytes_per_step_per_gpu": world * capacity * (4 + 2 * D * esize),
                   "l2": "inputs larger than L2"},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "cpu_baseline": None,
        "note": ("eager launches; the capacity (the largest owner segment of this batch "
                 "over all ranks, rounded up to 256) is agreed in a setup pass, so no count "
                 "crosses to the host inside a step"),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="full",
                    choices=["tiny", "b4x4096", "thd64k", "full", "long256k"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--adam-rows", type=int, default=ADAM_ROWS,
                    help="--stage adam: table rows (default: an 8-way shard of the page table)")
    ap.add_argument("--adam-touched", type=int, default=ADAM_TOUCHED,
                    help="--stage adam: rows one step updates")
    ap.add_argument("--ple-tokens", type=int, default=0,
                    help="--stage ple / ple_bwd: whole 4,096-token rows to use instead of "
                         "the workload's 16 (a smaller case for profiling)")
    ap.add_argument("--bwd-sort", choices=["heads", "plain"], default="heads",
                    help="backward sort: by head (engram_backward_sort_heads, the default) "
                         "or over the whole row range (engram_backward_sort)")
    ap.add_argument("--ple-inv", choices=["saved", "computed"], default="saved",
                    help="--stage ple_bwd: take the forward's saved inverse RMS (training's "
                         "path, default) or compute it in the backward")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", dest="graph", action="store_true", default=True,
                    help="time the step as a replayed CUDA graph (default)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time eager launches instead")
    ap.add_argument("--stage",
                    choices=["all", "bwd", "fwd", "hash", "gather", "ple", "ple_bwd", "adam",
                             "owner"],
                    default="all",
                    help="all: forward + backward (the step); bwd: the backward alone "
                         "(indices from engram_hash, no table allocated); fwd: "
                         "engram_hash_gather alone; hash: "
                         "engram_hash alone; gather: engram_gather alone on the hash's "
                         "indices; ple: the PLE "
                         "tail (norm + short conv) on its own workload; ple_bwd: its "
                         "backward on the same workload; owner: the owner-sharded table "
                         "with all-to-all exchanges; adam: the sparse "
                         "optimizer step on an 8-way owner shard of the table")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)      # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    if args.stage == "ple":
        return run_ple(args)
    if args.stage == "ple_bwd":
        return run_ple(args, backward=True)
    if args.stage == "owner":
        return run_owner(args)
    if args.stage == "adam":
        return run_adam(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
