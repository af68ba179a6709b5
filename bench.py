#!/usr/bin/env python
"""Benchmark of the fused DLRMv1 sparse/interaction stage on B200.

One step = one call of ``dlrm_sparse_interact`` over one batch: the
multi-table EmbeddingBag sum of all F tables, the pooled vectors written to
HBM, and the strict-lower-triangle dots over [dense, pooled]. Default
workload: B=2048, F=32 tables of 1e6 x 64 f32, L=16, Zipf(1.05) indices.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Under torchrun each rank is an independent
replica with its own batch (no collective on the data path); the timing is
the max over ranks. ``--impl reference`` times the CPU oracle on the host
cores on bounded samples of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dlrm_embedding_bag_b200 import synthetic as syn  # noqa: E402

PROFILES = os.path.join(ROOT, "profiles")
CSRC = os.path.join(ROOT, "dlrm_embedding_bag_b200", "csrc")
FALLBACK_HBM_GBS = 6650.0
E2E_BATCHES = 4
METRIC = "pooled lookups/s (fused EmbeddingBag-sum + lower-triangle interaction)"


# ----------------------------------------------------------------------------- helpers

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="c3", choices=sorted(syn.CONFIGS))
    ap.add_argument("--rows", type=int, default=None,
                    help="override the rows per table (a smaller case for profiling)")
    ap.add_argument("--batch", type=int, default=None, help="override the batch size")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-depth", type=int, default=4,
                    help="batches in flight on the end-to-end host pipeline (one stream each)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tables", choices=["f32", "bf16"], default="f32",
                    help="table element type (bf16: rows widened exactly, pooled in f32)")
    ap.add_argument("--pool", choices=["sum", "mean", "max"], default="sum")
    ap.add_argument("--weighted", action="store_true", help="per-sample weights (sum mode)")
    ap.add_argument("--ragged", action="store_true",
                    help="bag lengths drawn uniformly from [0, 2L] (same total entries)")
    ap.add_argument("--sweep", action="store_true",
                    help="time the fused stage on the 11 x 5 batch x table-count sweep instead")
    ap.add_argument("--mlp", action="store_true",
                    help="time the DLRMv1 MLP layers (tcgen05) and the full forward instead")
    ap.add_argument("--kernel", choices=["fused", "gather", "interact"], default="fused",
                    help="time the fused stage (default), the gather alone (embbag_sum_multi / "
                         "embbag_pool_multi) or the interaction alone (interact_lower_tri)")
    ap.add_argument("--path", choices=["auto", "ldg"], default="auto",
                    help="gather path of the library (auto = the measured fastest)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU time budget of the oracle baseline sample")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    return args


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device) -> float:
    """The maximum of x over all ranks (x itself on one rank); every rank calls it."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def algorithmic_bytes(w: syn.Workload, write_pooled: bool = True, esz: int = 4,
                      weighted: bool = False) -> int:
    """Bytes the fused step must move once: rows (esz bytes per element),
    indices, per-sample weights, offsets, dense, outputs."""
    B, F, L, D, P = w.B, w.F, w.L, w.D, w.P
    rows = B * F * L * D * esz
    idx = B * F * L * 4 * (2 if weighted else 1)
    offs = B * F * 4
    dense = B * D * 4
    pooled = B * F * D * 4 if write_pooled else 0
    inter = B * ((D + P) if w.concat_dense else P) * 4
    return rows + idx + offs + dense + pooled + inter


def hold_stream(steps: int, per_step_ms: float = 0.1) -> None:
    """Keep the current stream busy (a device-side spin of about steps x
    per_step_ms, at most 50 ms) while the host queues the steps that follow,
    so that each step's CUDA events bracket the GPU's work and not a gap in
    which the GPU waited for the host to launch it. The spin runs before the
    first step, outside every step's events."""
    import torch
    ms = min(50.0, steps * per_step_ms)
    torch.cuda._sleep(int(ms * 2.0e6))  # cycles at about 2 GHz


def pcie_copy_rates(h2d_bytes: int, d2h_bytes: int, dev, reps: int = 20,
                    trials: int = 5) -> dict:
    """Plain copies of one step's sizes between page-locked host memory and
    the device: host-to-device alone, device-to-host alone, and both at once
    on two streams (GB/s over the bytes moved, the device synchronised on both
    sides of `reps` copies). Each rate is the best of `trials` such runs after
    a warm-up of about 100 copies: the first copies of a process ran at well
    under half the rate, so a single run is not a ceiling. The last rate is the
    ceiling of a pipeline that overlaps a step's inputs with another step's
    outputs."""
    import torch
    hin = torch.ones(h2d_bytes, dtype=torch.uint8).pin_memory()
    hout = torch.ones(d2h_bytes, dtype=torch.uint8).pin_memory()
    din = torch.empty(h2d_bytes, dtype=torch.uint8, device=dev)
    dout = torch.empty(d2h_bytes, dtype=torch.uint8, device=dev)
    s1, s2 = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def run(h2d, d2h, n):
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(n):
            if h2d:
                with torch.cuda.stream(s1):
                    din.copy_(hin, non_blocking=True)
            if d2h:
                with torch.cuda.stream(s2):
                    hout.copy_(dout, non_blocking=True)
        torch.cuda.synchronize(dev)
        return n * ((h2d_bytes if h2d else 0) + (d2h_bytes if d2h else 0)) / (
            time.perf_counter() - t0) / 1e9

    run(True, True, 100)
    return {"h2d_gbs": max(run(True, False, reps) for _ in range(trials)),
            "d2h_gbs": max(run(False, True, reps) for _ in range(trials)),
            "duplex_gbs": max(run(True, True, reps) for _ in range(trials)),
            "method": f"best of {trials} runs of {reps} copies, after 100 warm-up copies"}

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return json.load(fh)
    except OSError:
        return None


# The sources the benchmarked fused kernel and its launch are built from: a
# recorded DRAM traffic figure stays valid while none of them changes.
FUSED_SOURCES = [os.path.join(CSRC, n) for n in (
    "device_common.cuh", "interact_common.cuh", "kernels.cuh", "inst_f32x4s.cu", "kernels.cu",
    "launch.h", "api.cu")] + [os.path.join(ROOT, "include", "dlrm_sparse.h")]


def source_digest() -> str:
    h = hashlib.sha256()
    for path in FUSED_SOURCES:
        with open(path, "rb") as fh:
            h.update(os.path.basename(path).encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel is unchanged."""
    path = os.path.join(PROFILES, "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh)
    except OSError:
        return None
    ent = rec.get(workload)
    if not ent or ent.get("source_digest") != source_digest():
        return None
    return ent.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML in a thread."""

    NAMES = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
             0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
             0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
             0x100: "display_clock_setting"}
    BAD = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self.ok = False
        try:
            import pynvml as nv

            import torch

            nv.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            handle = None
            try:
                bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id,
                                            props.pci_device_id)
                handle = nv.nvmlDeviceGetHandleByPciBusId_v2(bus)
            except Exception:  # noqa: BLE001
                handle = nv.nvmlDeviceGetHandleByIndex(device_index)
            self.nv, self.h = nv, handle
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.error = repr(e)
        self._stop = threading.Event()
        self._t = None

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self.h)

    def sample(self):
        if not self.ok:
            return
        nv = self.nv
        try:
            self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                 nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0, self._reasons()))
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(self.period)

    def start(self):
        self.sample()
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()

    def stop(self):
        self._stop.set()
        if self._t:
            self._t.join()
        self.sample()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "error", "nvml unavailable")}
        if not self.samples:
            return {"samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= int(s[2])
        reasons = sorted(n for b, n in self.NAMES.items() if bits & b)
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(mhz), "power_w_max": max(s[1] for s in self.samples),
                "samples": len(self.samples), "reasons": reasons}

    def bad(self):
        return bool(set(self.summary().get("reasons", [])) & self.BAD)


# ----------------------------------------------------------------------------- CPU oracle leg

def host_tables_for(w: syn.Workload, idx_sub: np.ndarray, source=None, seed: int = 0):
    """Full-size host tables in which only the rows the sample references hold data.

    The tables are allocated zeroed (so untouched pages stay unmapped) and
    the referenced rows are filled -- from the device tables when given
    (same values as the GPU run), else from N(0, 0.1). The oracle then reads
    the same row addresses in the same 4*N*D-byte tables as the full workload.
    """
    import torch

    tables = []
    rng = np.random.default_rng(seed)
    for k in range(w.F):
        t = np.zeros((w.N, w.D), dtype=np.float32)
        rows = np.unique(idx_sub[k])
        if source is not None:
            vals = source[k].index_select(0, torch.from_numpy(rows.astype(np.int64)).to(
                source[k].device)).cpu().numpy()
        else:
            vals = rng.normal(0.0, 0.1, (rows.size, w.D)).astype(np.float32)
        t[rows] = vals
        tables.append(t)
    return tables


def oracle_sample(w: syn.Workload, S: int, replica: int = 0, source=None):
    """The first S samples of the workload's batch, ready for the oracle."""
    idx = syn.make_indices(w, replica)[:, : S * w.L]
    idx = np.ascontiguousarray(idx)
    sub = w.scaled(B=S)
    off = syn.make_offsets(sub)
    rng = np.random.default_rng(3000)
    dense = rng.normal(0.0, 1.0, (S, w.D)).astype(np.float32)
    tables = host_tables_for(w, idx, source=source)
    return tables, idx, off, dense


def time_oracle(orc, tables, idx, off, dense, S, L, concat, budget_s, min_calls=1):
    times = []
    t_end = time.perf_counter() + budget_s
    while len(times) < min_calls or time.perf_counter() < t_end:
        t0 = time.perf_counter()
        orc.sparse_interact(tables, idx, off, dense, S, L, concat_dense=concat)
        times.append(time.perf_counter() - t0)
    return times


def host_cpu():
    """Host core count and CPU model (``nproc`` / ``lscpu``)."""
    import subprocess

    cores = os.cpu_count() or 1
    model = ""
    try:
        cores = int(subprocess.run(["nproc"], capture_output=True, text=True,
                                   check=True).stdout.strip())
        for line in subprocess.run(["lscpu"], capture_output=True, text=True,
                                   check=True).stdout.splitlines():
            if line.startswith("Model name:"):
                model = line.split(":", 1)[1].strip()
    except (OSError, subprocess.SubprocessError, ValueError):
        pass
    return cores, model


def cpu_baseline(w: syn.Workload, source, budget_s: float):
    """The oracle timed on one core and on all host cores.

    All cores: the whole batch is cut into one contiguous chunk of samples per
    core, and one thread per core calls the oracle's C code on its chunk
    (ctypes releases the interpreter lock for the call), so every core runs
    the same per-sample loops in parallel over samples."""
    import concurrent.futures as cf

    import oracle  # test infrastructure: this leg times the oracle as it stands

    orc = oracle.default()
    S = min(w.B, 512)
    tables, idx, off, dense = oracle_sample(w, S, source=source)
    orc.sparse_interact(tables, idx, off, dense, S, w.L, concat_dense=w.concat_dense)  # warm
    times = time_oracle(orc, tables, idx, off, dense, S, w.L, w.concat_dense, budget_s / 2)
    single = S * w.F * w.L / statistics.median(times)

    cores, model = host_cpu()
    SB = w.B
    tables_b, idx_b, _, dense_b = oracle_sample(w, SB, source=source)
    n = max(1, min(cores, SB))
    bounds = [(SB * c // n, SB * (c + 1) // n) for c in range(n)]
    chunks = []
    for s0, s1 in bounds:
        sub = w.scaled(B=s1 - s0)
        chunks.append((np.ascontiguousarray(idx_b[:, s0 * w.L:s1 * w.L]), syn.make_offsets(sub),
                       np.ascontiguousarray(dense_b[s0:s1]), s1 - s0))

    def one(ch):
        ci, co, cd, cb = ch
        orc.sparse_interact(tables_b, ci, co, cd, cb, w.L, concat_dense=w.concat_dense)

    with cf.ThreadPoolExecutor(max_workers=n) as ex:
        list(ex.map(one, chunks))  # warm
        par = []
        t_end = time.perf_counter() + budget_s / 2
        while len(par) < 3 or time.perf_counter() < t_end:
            t0 = time.perf_counter()
            list(ex.map(one, chunks))
            par.append(time.perf_counter() - t0)
    allc = SB * w.F * w.L / statistics.median(par)
    return {"value": allc, "unit": "lookups/s", "cores": n, "kind": "oracle",
            "cpu": model, "nproc": cores,
            "sample": f"all {SB} samples of {w.name} (all {w.F} tables, L={w.L}) cut into {n} "
                      f"chunks, one thread per core calling the oracle on its chunk; full-size "
                      f"host tables holding the referenced rows; median of {len(par)} passes",
            "single_core": {"value": single, "unit": "lookups/s", "cores": 1,
                            "sample": f"first {S} samples, median of {len(times)} "
                                      f"single-thread oracle calls"}}


def run_reference(args, w: syn.Workload):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle  # the reference arm of this benchmark is the oracle

    S = min(w.B, 128)
    tables, idx, off, dense = oracle_sample(w, S)
    orc = oracle.default()
    for _ in range(args.warmup):
        orc.sparse_interact(tables, idx, off, dense, S, w.L, concat_dense=w.concat_dense)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.sparse_interact(tables, idx, off, dense, S, w.L, concat_dense=w.concat_dense)
    dt = time.perf_counter() - t0
    value = args.steps * S * w.F * w.L / dt
    sample = (f"each step: first {S} of {w.B} samples of {w.name}, full-size host tables "
              f"holding the referenced rows, one single-thread oracle call")
    line = {"metric": METRIC, "value": value, "unit": "lookups/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(w, args.gpus), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": "lookups/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "lookups/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w: syn.Workload, n: int, args=None):
    tables = getattr(args, "tables", "f32")
    pool = getattr(args, "pool", "sum")
    weighted = getattr(args, "weighted", False)
    ragged = getattr(args, "ragged", False)
    name = w.name
    extra = [x for x in (tables if tables != "f32" else "", pool if pool != "sum" else "",
                         "weighted" if weighted else "", "ragged" if ragged else "") if x]
    if extra:
        name = name + "_" + "_".join(extra)
    return {"workload": name, "B": w.B, "F": w.F, "N": w.N, "D": w.D, "L": w.L,
            "tables": f"{tables} (rows widened to f32)" if tables != "f32" else "f32",
            "pooling": pool + (" with per-sample weights" if weighted else ""),
            "index_dist": (f"zipf(alpha={w.alpha}) over rows, rank->row permuted"
                           if w.dist == "zipf" else "uniform"),
            "offsets": ("ragged: sorted uniform cut points, mean length L" if ragged
                        else "fixed stride b*L"),
            "outputs": "pooled (B,F,D) f32 + interaction (B,%s) f32" %
                       ("D+P" if w.concat_dense else "P"),
            "l2": "flushed before every step (256 MiB write outside the per-step events)",
            "parallelism": "replicas" if n > 1 else "single GPU"}


# ----------------------------------------------------------------------------- our arm

def run_ours(args, w: syn.Workload):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    from dlrm_embedding_bag_b200 import ops

    ops.set_gather_path(args.path)
    general = args.tables != "f32" or args.pool != "sum" or args.weighted or args.ragged
    # the link's copy ceiling for the e2e figure, taken first, while the process
    # holds nothing else (measured after the e2e pipeline in the same process,
    # the both-directions figure came out at 44 instead of 76-79 GB/s)
    link = None
    if not args.no_e2e and not general and args.kernel == "fused":
        link = pcie_copy_rates(4 * (w.F * w.B * w.L + w.F * w.B + w.B * w.D),
                               4 * w.B * ((w.D + w.P) if w.concat_dense else w.P), dev)
    # inputs resident in HBM before timing: tables, this replica's batch, outputs
    weights = syn.make_weights(w, dev)
    if args.tables == "bf16":
        weights = [t.to(torch.bfloat16) for t in weights]
        torch.cuda.empty_cache()
    idx_np = syn.make_indices(w, replica=rank)
    off_np = syn.make_ragged_offsets(w) if args.ragged else syn.make_offsets(w)
    idx = torch.from_numpy(idx_np).to(dev)
    off = torch.from_numpy(off_np).to(dev)
    dense = syn.make_dense(w, dev)
    psw = torch.from_numpy(syn.make_sample_weights(w)).to(dev) if args.weighted else None
    pooled = torch.empty((w.B, w.F, w.D), dtype=torch.float32, device=dev)
    inter = torch.empty((w.B, (w.D + w.P) if w.concat_dense else w.P), dtype=torch.float32,
                        device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)

    if args.kernel == "gather":
        def call(_stream):
            if general:
                ops.embbag_pool_multi(weights, idx, off, mode=args.pool, per_sample_weights=psw,
                                      out=pooled)
            else:
                ops.embbag_sum_multi(weights, idx, off, w.L, out=pooled)
    elif args.kernel == "interact":
        # the pooled vectors the interaction reads, made once outside the timing
        ops.embbag_sum_multi(weights, idx, off, w.L, out=pooled)
        inter = torch.empty((w.B, w.P), dtype=torch.float32, device=dev)

        def call(_stream):
            ops.interact_lower_tri(dense, pooled, out=inter)
    elif general:
        call = ops.PoolInteractCall(weights, idx, off, dense, mode=args.pool,
                                    per_sample_weights=psw, concat_dense=w.concat_dense,
                                    pooled_out=pooled, inter_out=inter)
    else:
        call = ops.SparseInteractCall(weights, idx, off, dense, w.L,
                                      concat_dense=w.concat_dense, pooled_out=pooled,
                                      inter_out=inter)
    stream = torch.cuda.current_stream().cuda_stream

    def step():
        call(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed_region():
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        sampler = ClockSampler(local)
        barrier()
        sampler.start()
        n0 = ops.launch_count()
        w0 = time.perf_counter()
        hold_stream(args.steps)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - w0
        launches = ops.launch_count() - n0
        barrier()
        sampler.stop()
        per = [s.elapsed_time(e) for s, e in zip(starts, ends)]
        return per, wall, launches, sampler

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    per, wall, launches, sampler = timed_region()
    remeasured = False
    if sampler.bad():
        per, wall, launches, sampler = timed_region()
        remeasured = True

    total_ms = max_over_ranks(float(sum(per)), world, dev)
    lookups = world * args.steps * w.B * w.F * w.L
    value = lookups / (total_ms / 1e3)
    ms_step = total_ms / args.steps

    # Cold steps with a clean L2: the flush above writes 256 MiB, so L2 starts
    # each step full of the flush's dirty lines, and the step's misses pay for
    # writing them back. Here each write-flush is followed by a read of another
    # buffer larger than L2 (outside the step's events), so the step starts with
    # its inputs out of L2 and nothing dirty in it.
    sweep = torch.ones(flush.numel() // 4, dtype=torch.float32, device=dev)
    sweep_sum = torch.empty((), dtype=torch.float32, device=dev)

    def cold_clean(run_step):
        ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        torch.cuda.synchronize()
        hold_stream(args.steps, 0.2)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            sweep_sum.copy_(sweep.sum())
            ev_s[i].record()
            run_step()
            ev_e[i].record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in zip(ev_s, ev_e)) / args.steps

    extras = {}
    if world == 1 and args.kernel != "interact":
        # the device's random-row read rate for the stage's row size, without
        # index loads: dlrm_probe_row_gather over a 4 GiB buffer (32 x L2), 8 M
        # rows per call, cold and clean L2 before each call, best of 3
        probe = torch.empty(4 << 30, dtype=torch.uint8, device=dev)
        sink = torch.zeros(1, dtype=torch.int32, device=dev)
        row_bytes = w.D * (2 if args.tables == "bf16" else 4)
        ceiling = {}
        for rb in sorted({128, 256, row_bytes} & {16, 32, 64, 128, 256, 512}):
            best = None
            for t in range(3):
                flush.fill_(t)
                sweep_sum.copy_(sweep.sum())
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                ops.probe_row_gather(probe, rb, 8 << 20, sink, seed=t)
                e1.record()
                torch.cuda.synchronize()
                ms = e0.elapsed_time(e1)
                best = ms if best is None else min(best, ms)
            ceiling[str(rb)] = {"rows_per_s": (8 << 20) / (best / 1e3),
                                "gbs": (8 << 20) * rb / (best / 1e3) / 1e9}
        del probe
        extras["row_read_ceiling"] = {
            "row_bytes": ceiling, "stage_row_bytes": row_bytes,
            "method": "dlrm_probe_row_gather: 8 M random rows of a 4 GiB buffer per call, row ids "
                      "hashed in registers (no index loads), 128-bit loads without L1 allocation, "
                      "cold clean L2, best of 3"}
    if world == 1:
        cc_ms = cold_clean(step)
        extras["cold_clean_l2"] = {
            "ms_per_step": cc_ms, "value": w.B * w.F * w.L / (cc_ms / 1e3), "unit": "lookups/s",
            "protocol": "each step after the 256 MiB write-flush and a read of another "
                        "256 MiB buffer (L2 without the flush's dirty lines)"}
    if world == 1 and args.kernel == "fused" and not general:
        # warm-L2 timing, the pages' harness protocol: 5 rounds of 20 back-to-back
        # steps (no flush between them), median of the round medians
        rounds = []
        for _ in range(5):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(21)]
            torch.cuda.synchronize()
            hold_stream(20)
            ev[0].record()
            for i in range(20):
                step()
                ev[i + 1].record()
            torch.cuda.synchronize()
            rounds.append(statistics.median(ev[i].elapsed_time(ev[i + 1]) for i in range(20)))
        warm_ms = statistics.median(rounds)
        extras["warm_l2"] = {"ms_per_step": warm_ms, "value": w.B * w.F * w.L / (warm_ms / 1e3),
                             "unit": "lookups/s",
                             "protocol": "5 rounds x 20 steps without L2 flush, median of round "
                                         "medians"}
        if w.dist == "zipf":
            # the same shapes with uniform indices: every row from HBM, the pure
            # bandwidth check of the gather (tables shared with the run above)
            wu = w.scaled(name=w.name.replace("zipf" + str(w.alpha), "uniform"),
                          dist="uniform", alpha=0.0)
            idx_u = torch.from_numpy(syn.make_indices(wu, replica=rank)).to(dev)
            call_u = ops.SparseInteractCall(weights, idx_u, off, dense, w.L,
                                            concat_dense=w.concat_dense, pooled_out=pooled,
                                            inter_out=inter)
            for _ in range(args.warmup):
                flush.fill_(1)
                call_u(stream)
            ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
            ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
            hold_stream(args.steps)
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                ev_s[i].record()
                call_u(stream)
                ev_e[i].record()
            torch.cuda.synchronize()
            u_ms = sum(a.elapsed_time(b) for a, b in zip(ev_s, ev_e)) / args.steps
            uc_ms = cold_clean(lambda: call_u(stream))
            extras["hbm_check"] = {"workload": wu.name, "ms_per_step": u_ms,
                                   "cold_clean_l2": {
                                       "ms_per_step": uc_ms,
                                       "achieved_gbs": algorithmic_bytes(wu) / (uc_ms / 1e3) / 1e9},
                                   "value": w.B * w.F * w.L / (u_ms / 1e3),
                                   "unit": "lookups/s",
                                   "achieved_gbs": algorithmic_bytes(wu) / (u_ms / 1e3) / 1e9,
                                   "algorithmic_bytes_per_launch": algorithmic_bytes(wu),
                                   "traffic": recorded_traffic(wu.name)}
            del idx_u, call_u

    # e2e through the host-buffer entry point: every step copies its batch's
    # indices, offsets and dense rows in from pinned host memory and its
    # interaction rows back out. Steps cycle over E2E_BATCHES distinct batches
    # (tables 8 GB > L2) on a pipeline of --e2e-depth streams, so one batch's
    # copies overlap other batches' kernels and copies; the region is timed
    # with events.
    e2e = None
    if not args.no_e2e and not general and args.kernel == "fused":
        pipe = ops.HostPipeline(weights, w.B, w.L, concat_dense=w.concat_dense, want_pooled=True,
                                depth=args.e2e_depth)
        batches = []
        stage0 = pipe.slots[0][0]
        for j in range(E2E_BATCHES):
            ij = syn.make_indices(w, replica=rank * E2E_BATCHES + j) if j else idx_np
            # one page-locked block per batch: a single host-to-device copy
            batches.append(stage0.pack(torch.from_numpy(ij.reshape(-1)), torch.from_numpy(off_np),
                                       dense.cpu()))
        outs = [torch.empty(tuple(inter.shape), dtype=torch.float32).pin_memory()
                for _ in range(args.e2e_depth)]
        for i in range(args.warmup):
            pipe.submit(*batches[i % E2E_BATCHES], outs[i % args.e2e_depth])
        pipe.drain()
        barrier()
        cur = torch.cuda.current_stream()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(cur)
        for _, st, _ in pipe.slots:
            st.wait_event(t0)
        for i in range(args.steps):
            pipe.submit(*batches[i % E2E_BATCHES], outs[i % args.e2e_depth])
        for _, st, _ in pipe.slots:
            ev = torch.cuda.Event()
            ev.record(st)
            cur.wait_event(ev)
        t1.record(cur)
        barrier()
        e2e_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)

        # the same with the batch in three separate page-locked buffers (a
        # caller that does not pack): three host-to-device copies per step
        loose = []
        for j in range(E2E_BATCHES):
            ij, oj, dj = batches[j]
            loose.append((ij.clone().pin_memory(), oj.clone().pin_memory(),
                          dj.clone().pin_memory()))
        for i in range(args.warmup):
            pipe.submit(*loose[i % E2E_BATCHES], outs[i % args.e2e_depth])
        pipe.drain()
        barrier()
        u0 = torch.cuda.Event(enable_timing=True)
        u1 = torch.cuda.Event(enable_timing=True)
        u0.record(cur)
        for _, st, _ in pipe.slots:
            st.wait_event(u0)
        for i in range(args.steps):
            pipe.submit(*loose[i % E2E_BATCHES], outs[i % args.e2e_depth])
        for _, st, _ in pipe.slots:
            ev = torch.cuda.Event()
            ev.record(st)
            cur.wait_event(ev)
        u1.record(cur)
        barrier()
        loose_ms = max_over_ranks(u0.elapsed_time(u1), world, dev)
        # what packing one batch into a reused page-locked block costs on the
        # host (outside the timed region above; batch 0 is rewritten with its
        # own values)
        pipe.drain()
        idx_t, off_t, dense_t = (torch.from_numpy(idx_np.reshape(-1)), torch.from_numpy(off_np),
                                 dense.cpu())
        bi, bo, bd = batches[0]
        p0 = time.perf_counter()
        for _ in range(5):
            bi.copy_(idx_t)
            bo.copy_(off_t)
            bd.copy_(dense_t)
        pack_ms = (time.perf_counter() - p0) / 5 * 1e3
        # host cost of one submit when none waits (the ring drained first)
        sub_s, nsub = 0.0, 0
        for r in range(10):
            pipe.drain()
            h0 = time.perf_counter()
            for i in range(args.e2e_depth):
                pipe.submit(*batches[(r + i) % E2E_BATCHES], outs[i])
            sub_s += time.perf_counter() - h0
            nsub += args.e2e_depth
        pipe.drain()
        submit_ms = sub_s / nsub * 1e3
        assert link is not None
        # again now that the process has moved a few GB through the link: its
        # first copies can run at under half the rate (seen on one B200 machine at
        # 22 GB/s host-to-device at the start); the best of both is the ceiling
        later = pcie_copy_rates(pipe.h2d_bytes(), pipe.d2h_bytes(), dev)
        link = {k: (max(link[k], later[k]) if k.endswith("_gbs") else link[k]) for k in link}
        link["method"] += "; taken at the start of the run and after the e2e loops, best of both"
        step_bytes = pipe.h2d_bytes() + pipe.d2h_bytes()
        link["e2e_gbs"] = step_bytes / (e2e_ms / args.steps / 1e3) / 1e9
        link["frac_of_duplex"] = link["e2e_gbs"] / link["duplex_gbs"]
        e2e = {"value": lookups / (e2e_ms / 1e3), "unit": "lookups/s",
               "h2d_bytes_per_step": pipe.h2d_bytes(), "d2h_bytes_per_step": pipe.d2h_bytes(),
               "ms_per_step": e2e_ms / args.steps,
               "host_submit_ms_per_batch": submit_ms,
               "unpacked": {"value": lookups / (loose_ms / 1e3), "ms_per_step": loose_ms / args.steps,
                            "note": "indices, offsets and dense in three separate pinned "
                                    "buffers: three host-to-device copies per step"},
               "host_pack_ms_per_batch": pack_ms,
               "link": link,
               "path": f"dlrm_sparse_interact_host via ops.HostPipeline ({args.e2e_depth} streams): one "
                       f"pinned [indices|offsets|dense] block in, interaction rows out, {E2E_BATCHES} distinct "
                       f"batches in rotation; pooled written to device staging"}

    if rank == 0:
        peaks = measured_peaks()
        if peaks and peaks.get("hbm_gbs"):
            peak, peak_src = float(peaks["hbm_gbs"]), "measured"
        else:
            peak, peak_src = FALLBACK_HBM_GBS, "fallback"
        per_launch = algorithmic_bytes(w, esz=2 if args.tables == "bf16" else 4,
                                       weighted=args.weighted)
        kernel_name = "fused_kernel (dlrm_sparse_interact)"
        if args.kernel == "gather":
            per_launch = algorithmic_bytes(w, esz=2 if args.tables == "bf16" else 4,
                                           weighted=args.weighted) - 4 * w.B * w.D \
                - 4 * w.B * ((w.D + w.P) if w.concat_dense else w.P)
            kernel_name = "gather (embbag_sum_multi)"
        elif args.kernel == "interact":
            per_launch = 4 * w.B * w.D + 4 * w.B * w.F * w.D + 4 * w.B * w.P
            kernel_name = "interact_kernel (interact_lower_tri)"
        achieved = per_launch / (ms_step / 1e3) / 1e9
        rows_gbs = (w.B * w.F * w.L * w.D * (2 if args.tables == "bf16" else 4)
                    / (ms_step / 1e3) / 1e9)
        clocks = sampler.summary()
        line = {
            "metric": METRIC, "value": value, "unit": "lookups/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": workload_config(w, world, args),
            "samples_per_s": world * args.steps * w.B / (total_ms / 1e3),
            "gather_row_gbs": rows_gbs,
            "roofline": {"bound": "hbm", "kernel": kernel_name,
                         "achieved": achieved, "peak": peak, "peak_source": peak_src,
                         "unit": "GB/s", "frac": achieved / peak,
                         "algorithmic_bytes_per_launch": per_launch,
                         "traffic": recorded_traffic(w.name)},
            "gather_path": ops.last_gather_path(),
            "clocks": clocks, "remeasured": remeasured,
            "gpu_launches": launches,
            "region_wall_ms": 1e3 * wall,
            "region_hold_ms": min(50.0, args.steps * 0.1),
            "step_ms_p50": statistics.median(per), "step_ms_min": min(per),
            "e2e": e2e,
        }
        line.update(extras)
        if "hbm_check" in line:
            line["hbm_check"]["peak"] = peak
            line["hbm_check"]["frac"] = line["hbm_check"]["achieved_gbs"] / peak
            cc = line["hbm_check"]["cold_clean_l2"]
            cc["frac"] = cc["achieved_gbs"] / peak
        if "row_read_ceiling" in line:
            rc_ = line["row_read_ceiling"]
            lim = rc_["row_bytes"].get(str(rc_["stage_row_bytes"]))
            if lim is not None:
                # lookups/s of the stage against rows/s of the probe at the same row size
                rc_["stage_frac"] = line["value"] / lim["rows_per_s"]
                if "hbm_check" in line:
                    hc = line["hbm_check"]
                    hc["row_ceiling_frac"] = hc["value"] / lim["rows_per_s"]
                    hc["cold_clean_l2"]["row_ceiling_frac"] = (
                        w.B * w.F * w.L / (hc["cold_clean_l2"]["ms_per_step"] / 1e3) /
                        lim["rows_per_s"])
        if "cold_clean_l2" in line:
            cc = line["cold_clean_l2"]
            cc["achieved_gbs"] = per_launch / (cc["ms_per_step"] / 1e3) / 1e9
            cc["frac"] = cc["achieved_gbs"] / peak
            if args.kernel == "interact":
                cc["value"], cc["unit"] = w.B / (cc["ms_per_step"] / 1e3), "samples/s"
        if general:
            line["e2e"] = None
            line["e2e_note"] = "end-to-end host path covers the fixed-stride f32 sum stage only"
        if args.kernel != "fused":
            line["metric"] = (METRIC.replace("fused EmbeddingBag-sum + lower-triangle "
                                             "interaction", "EmbeddingBag gather alone")
                              if args.kernel == "gather"
                              else "interaction samples/s (lower-triangle dots alone)")
            if args.kernel == "interact":
                line["value"] = line["samples_per_s"]
                line["unit"] = "samples/s"
            line["roofline"]["traffic"] = None
            line["e2e"] = None
            line["e2e_note"] = "end-to-end host path covers the fused stage only"
        if world == 1 and not args.no_cpu_baseline and not general and args.kernel == "fused":
            line["cpu_baseline"] = cpu_baseline(w, weights, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- sweep

def run_sweep(args):
    """The fused stage on every cell of the batch x table-count sweep (100000 x 64
    tables, L=8, uniform indices). One JSON line with one entry per cell."""
    import torch
    from dlrm_embedding_bag_b200 import ops

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    cells = list(syn.sweep())
    Fmax = max(c.F for c in cells)
    tables = syn.make_weights(cells[0].scaled(F=Fmax), dev)  # table k is the same in every cell
    out = []
    for w in cells:
        idx = torch.from_numpy(syn.make_indices(w)).to(dev)
        off = torch.from_numpy(syn.make_offsets(w)).to(dev)
        dense = syn.make_dense(w, dev)
        inter = torch.empty((w.B, w.P), device=dev)
        call = ops.SparseInteractCall(tables[:w.F], idx, off, dense, w.L, inter_out=inter)
        s = torch.cuda.current_stream().cuda_stream
        for _ in range(args.warmup):
            flush.fill_(1)
            call(s)
        torch.cuda.synchronize()
        st = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        hold_stream(args.steps)
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            st[i].record()
            call(s)
            en[i].record()
        torch.cuda.synchronize()
        ms = statistics.median([a.elapsed_time(b) for a, b in zip(st, en)])
        out.append({"B": w.B, "F": w.F, "us": 1e3 * ms,
                    "lookups_per_s": w.B * w.F * w.L / (ms / 1e3),
                    "samples_per_s": w.B / (ms / 1e3)})
    big = max(out, key=lambda c: (c["B"], c["F"]))
    line = {"metric": METRIC + " over the batch x num_cat sweep", "value": big["lookups_per_s"],
            "unit": "lookups/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "dtype": "f32", "data": "synthetic",
            "config": {"workload": "sweep: B in 1..1024 (11 values) x F in {1,4,8,16,32}, "
                                   "100000 x 64 f32 tables, L=8 uniform, fixed-stride offsets",
                       "l2": "flushed before every step", "value_cell": "B=1024, F=32",
                       "timing": "median of steps per cell"},
            "cells": out}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- MLP layers

def run_mlp(args, w: syn.Workload):
    """Time each DLRMv1 MLP layer (bf16 tcgen05 GEMM + bias + activation) at the
    workload's batch and at 32x that batch, and the full DLRMv1 forward
    (bottom MLP, sparse stage, top MLP) at the workload's batch. One JSON line."""
    import torch
    from dlrm_embedding_bag_b200 import mlp, ops

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)

    def timeit(fn, steps, warmup):
        for _ in range(warmup):
            flush.fill_(1)
            fn()
        torch.cuda.synchronize()
        st = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        en = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        hold_stream(steps, 0.2)
        for i in range(steps):
            flush.fill_(i & 0xFF)
            st[i].record()
            fn()
            en[i].record()
        torch.cuda.synchronize()
        return statistics.median([a.elapsed_time(b) for a, b in zip(st, en)])

    P = w.P
    bottom_w = [syn.DENSE_FEATURES, *syn.BOTTOM_HIDDEN, w.D]
    top_w = [w.D + P, *syn.TOP_HIDDEN, 1]
    layers = []
    for B in (w.B, 32 * w.B):
        g = torch.Generator(device=dev)
        g.manual_seed(B)
        for name, widths, last, split in (("bottom", bottom_w, "relu", False),
                                          ("top", top_w, "sigmoid", True)):
            ls = syn.make_mlp_layers(widths[0], widths[1:], 7 if name == "bottom" else 8, dev,
                                     last=last)
            for i, (wt, b, act) in enumerate(ls):
                K, N = wt.shape[1], wt.shape[0]
                if split and i == 0:
                    a_lo = mlp.bf16_empty(B, w.D, dev)
                    a_lo.copy_(torch.randn(B, w.D, device=dev, generator=g).to(torch.bfloat16))
                    a_hi = mlp.bf16_empty(B, P, dev)
                    a_hi.copy_(torch.randn(B, P, device=dev, generator=g).to(torch.bfloat16))
                else:
                    a_lo = mlp.bf16_empty(B, K, dev)
                    a_lo.copy_(torch.randn(B, K, device=dev, generator=g).to(torch.bfloat16))
                    a_hi = None
                last_layer = i == len(ls) - 1
                y32 = torch.empty((B, N), device=dev) if last_layer else None
                y16 = None if last_layer else mlp.bf16_empty(B, N, dev)

                def fn(a_lo=a_lo, a_hi=a_hi, wt=wt, b=b, act=act, y32=y32, y16=y16):
                    mlp.linear_bf16(a_lo, wt, b, act, a_hi=a_hi, out_f32=y32, out_bf16=y16,
                                    f32=y32 is not None, bf16=y16 is not None)

                ms = timeit(fn, args.steps, args.warmup)
                flops = 2.0 * B * N * K
                layers.append({"mlp": name, "layer": i, "B": B, "K": K, "N": N,
                               "split_a": bool(split and i == 0), "act": act, "mode": "bf16",
                               "us": 1e3 * ms, "tflops": flops / (ms / 1e3) / 1e12})
                # the same layer with f32 activations (three exact bf16 planes per
                # value: three times the tensor work of the bf16 layer)
                p_lo = mlp.split_bf16x3(a_lo.float())
                p_hi = mlp.split_bf16x3(a_hi.float()) if a_hi is not None else None
                yp = None if last_layer else mlp.planes_empty(B, N, dev)

                def fn32(p_lo=p_lo, p_hi=p_hi, wt=wt, b=b, act=act, y32=y32, yp=yp):
                    mlp.linear_f32a(p_lo, wt, b, act, a_hi=p_hi, out_f32=y32, out_planes=yp,
                                    f32=y32 is not None, planes=yp is not None)

                ms32 = timeit(fn32, args.steps, args.warmup)
                layers.append({"mlp": name, "layer": i, "B": B, "K": K, "N": N,
                               "split_a": bool(split and i == 0), "act": act, "mode": "f32",
                               "us": 1e3 * ms32, "tflops": flops / (ms32 / 1e3) / 1e12,
                               "tensor_tflops": 3 * flops / (ms32 / 1e3) / 1e12})
    # the full forward at the workload's batch
    bottom = mlp.MLP(syn.make_mlp_layers(bottom_w[0], bottom_w[1:], 7, dev), mode="bf16")
    top = mlp.MLP(syn.make_mlp_layers(top_w[0], top_w[1:], 8, dev, last="sigmoid"),
                  mode="bf16")
    weights = syn.make_weights(w, dev)
    idx = torch.from_numpy(syn.make_indices(w)).to(dev)
    off = torch.from_numpy(syn.make_offsets(w)).to(dev)
    x = syn.make_dense_features(w.B, dev)
    n0 = ops.launch_count()
    mlp.dlrm_forward(bottom, top, x, weights, idx, off, w.L)
    fwd_launches = ops.launch_count() - n0
    fwd_ms = timeit(lambda: mlp.dlrm_forward(bottom, top, x, weights, idx, off, w.L),
                    args.steps, args.warmup)
    # the same forward captured once into a CUDA graph and replayed (no launch gaps)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        mlp.dlrm_forward(bottom, top, x, weights, idx, off, w.L)  # allocations outside capture
        with torch.cuda.graph(graph, stream=side):
            graph_out = mlp.dlrm_forward(bottom, top, x, weights, idx, off, w.L)  # noqa: F841
    torch.cuda.current_stream().wait_stream(side)
    graph_ms = timeit(graph.replay, args.steps, args.warmup)
    # the same forward with f32 activations throughout (the pages' arithmetic)
    bottom32 = mlp.MLP(bottom.layers, mode="f32")
    top32 = mlp.MLP(top.layers, mode="f32")
    x32 = x.float().contiguous()
    n0 = ops.launch_count()
    mlp.dlrm_forward(bottom32, top32, x32, weights, idx, off, w.L)
    fwd32_launches = ops.launch_count() - n0
    fwd32_ms = timeit(lambda: mlp.dlrm_forward(bottom32, top32, x32, weights, idx, off, w.L),
                      args.steps, args.warmup)
    side32 = torch.cuda.Stream()
    side32.wait_stream(torch.cuda.current_stream())
    graph32 = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side32):
        mlp.dlrm_forward(bottom32, top32, x32, weights, idx, off, w.L)
        with torch.cuda.graph(graph32, stream=side32):
            graph32_out = mlp.dlrm_forward(bottom32, top32, x32, weights, idx, off, w.L)  # noqa: F841
    torch.cuda.current_stream().wait_stream(side32)
    graph32_ms = timeit(graph32.replay, args.steps, args.warmup)
    big = max((r for r in layers if r["mode"] == "bf16"), key=lambda r: r["B"] * r["N"] * r["K"])
    big32 = max((r for r in layers if r["mode"] == "f32"), key=lambda r: r["B"] * r["N"] * r["K"])
    peaks = measured_peaks() or {}
    peak = float(peaks.get("bf16_tflops") or 1590.0)
    line = {
        "metric": "DLRMv1 MLP layer TFLOP/s (tcgen05, f32 accumulate, fused bias+act; bf16 "
                  "activations, and f32 activations as three exact bf16 planes)",
        "value": big["tflops"], "unit": "TFLOP/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"DLRMv1 MLPs bottom {'-'.join(map(str, bottom_w))}, top "
                               f"{'-'.join(map(str, top_w))} (top layer 0 split-A "
                               f"[D={w.D} | P={P}]) at B={w.B} and {32 * w.B}",
                   "l2": "flushed between steps"},
        "roofline": {"bound": "tensor", "kernel": f"linear_bf16_kernel B={big['B']} "
                     f"K={big['K']} N={big['N']}", "achieved": big["tflops"], "peak": peak,
                     "peak_source": "measured (burst)" if peaks.get("bf16_tflops") else "fallback",
                     "unit": "TFLOP/s", "frac": big["tflops"] / peak},
        "layers": layers,
        "forward": {"workload": w.name, "B": w.B, "us": 1e3 * fwd_ms,
                    "samples_per_s": w.B / (fwd_ms / 1e3), "gpu_launches": fwd_launches,
                    "graph_us": 1e3 * graph_ms, "graph_samples_per_s": w.B / (graph_ms / 1e3),
                    "steps": "bottom MLP (3 layers), fused sparse stage, z to bf16, top MLP "
                             "(3 layers, first split-A)"},
        "forward_f32": {"workload": w.name, "B": w.B, "us": 1e3 * fwd32_ms,
                        "samples_per_s": w.B / (fwd32_ms / 1e3), "gpu_launches": fwd32_launches,
                        "graph_us": 1e3 * graph32_ms,
                        "graph_samples_per_s": w.B / (graph32_ms / 1e3),
                        "steps": "features split into planes, bottom MLP (3 f32-activation "
                                 "layers), fused sparse stage, z split into planes, top MLP"},
        "f32_layer": {"kernel": f"linear_f32a B={big32['B']} K={big32['K']} N={big32['N']}",
                      "us": big32["us"], "tflops": big32["tflops"],
                      "tensor_tflops": big32["tensor_tflops"],
                      "tensor_frac": big32["tensor_tflops"] / peak},
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    args = parse_args(argv)
    w = syn.CONFIGS[args.config]
    if args.rows or args.batch:
        B = args.batch or w.B
        N = args.rows or w.N
        w = w.scaled(B=B, N=N, name=f"{w.name}_B{B}_N{N}")
    if args.impl == "reference":
        return run_reference(args, w)
    if args.mlp:
        return run_mlp(args, w)
    if args.sweep:
        return run_sweep(args)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
