"""Benchmark: batched row-wise TopK on B200, effective HBM GB/s (and rows/s).

One step = one ``dsel_topk`` call over one batch of the selected workload (default:
the bfloat16 Lightning-Indexer batch, 64 rows x 131,072 positions, k = 512,
unsorted, indices only, int32).  Steps rotate over input copies whose total size is
more than four times the L2 cache, so every step reads its input from HBM.  The
timed region is CUDA-graph replays of those steps, bracketed by a barrier and a
device synchronise, timed with CUDA events on the launching stream; the max over
ranks is reported.  Under torchrun every rank processes its own batch (weak
scaling, no collective on the data path).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                       [--impl ours|reference] [--torch-topk]

``--torch-topk`` adds ``context_torch_topk`` to the line: torch.topk timed on the same
inputs, as context for the pages' comparison with it (never part of ``value``).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "effective HBM GB/s and rows/s for TopK (bf16 k=512; fp32 V=129,280) on 1 B200"
KERNEL_SOURCES = ["row_wise_topk_b200/csrc/dsel_device.cuh", "row_wise_topk_b200/csrc/dsel_kernels.cuh",
                  "row_wise_topk_b200/csrc/dsel_api.cu", "row_wise_topk_b200/csrc/dsel_plan.cpp",
                  "row_wise_topk_b200/csrc/dsel_shard.cu",
                  "row_wise_topk_b200/csrc/dsel_plan.h", "row_wise_topk_b200/csrc/dsel_resident.cuh",
                  "row_wise_topk_b200/csrc/dsel_slice.cuh"]
FALLBACK_HBM_GBS = 6650.0
SAMPLE_T, SAMPLE_P = 1.0, 0.9      # temperature and top-p of the sample_B_k workloads
LONG_SPLIT_N = 1 << 28             # the long_split_k row: 2^28 float32 positions (1 GiB)


def make_workload(name: str) -> W.Workload:
    if name == "indexer":
        return W.indexer_drift()
    if name == "indexer_varlen":
        return W.indexer_varlen()
    if name == "indexer_varlen_values":     # the same batch with the values returned too
        w = W.indexer_varlen(return_value=1)
        w.name += "_values"
        return w
    if name.startswith("sampler"):        # sampler_B_k, e.g. sampler_256_4096
        _, b, k = name.split("_")
        return W.sampler_logits(int(b), int(k))
    if name.startswith("sample_"):        # sample_B_k: TopK + the sampling draw, tokens only
        _, b, k = name.split("_")
        w = W.sampler_logits(int(b), int(k))
        w.name = "topk_sample_" + w.name + f"_t{SAMPLE_T}_p{SAMPLE_P}"
        return w
    if name.startswith("long_split"):     # long_split_k: one 2^28 row (the reference arm's view)
        return W.long_rows(1, LONG_SPLIT_N, int(name.split("_")[2]), "uniform")
    if name.startswith("long"):           # long_1_1000 (1 x 2^28), long_16_4096 (16 x 2^24),
        parts = name.split("_")           # long_16_4096_22 (16 x 2^22: a reduced case for profiling)
        r, k = int(parts[1]), int(parts[2])
        n = (1 << int(parts[3])) if len(parts) > 3 else ((1 << 28) if r == 1 else (1 << 24))
        return W.long_rows(r, n, k, "uniform")
    if name == "pr1":
        return W.pr1_duplicates()
    raise SystemExit(f"unknown workload {name}")


def roofline_launch_ms(region_ms_per_step: float, launches_per_step: int, isolated_ms) -> float:
    """Average duration of one launch of the dominant kernel over the timed region.

    When a step is that one launch, it is the region's time per step (CUDA events
    around the whole timed region, launches back to back as the workload runs them).
    With a second (merge) launch per step the region cannot separate them, and the
    mean of the isolated event-pair times of the step is used instead."""
    if launches_per_step == 1:
        return region_ms_per_step
    return statistics.mean(isolated_ms)


def kernel_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(workload: str):
    """Per-launch DRAM bytes of the streaming kernel from a committed ncu summary, if
    it was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(workload)
    if not e or e.get("kernel_hash") != kernel_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sel = [l for t, l in self.lines if self.t0 is None or (self.t0 - 0.06 <= t <= self.t1 + 0.06)]
        if not sel:
            sel = [l for _, l in self.lines[-3:]]
        mhz, max_mhz, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in sel:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                max_mhz = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max_mhz, "reasons": sorted(reasons),
                "samples": len(mhz)}


def physical_gpu_index(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    if local < len(vis) and vis[local].strip().isdigit():
        return int(vis[local])
    return local


# --------------------------------------------------------------------------- #
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(value: float, pg, device=None) -> float:
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step: int, steps: int, elapsed_ms: float, world: int) -> float:
    """Whole-job effective GB/s: every rank processes its own batch of the workload
    (weak scaling), and the slowest rank's time counts."""
    return world * bytes_per_step * steps / (elapsed_ms / 1e3) / 1e9


def cpu_oracle_throughput(w: W.Workload, budget_s: float):
    """Times the CPU oracle (as it stands) on whole rows of the workload until the
    budget is spent; returns (GB/s effective, rows/s, rows timed)."""
    import oracle.sample_oracle as S
    import oracle.topk_oracle as O
    sampling = w.name.startswith("topk_sample_")
    u = W.uniforms(w.rows)
    lens = w.valid_lengths()
    idx_b = 4 if w.index_dtype == "i32" else 8
    val_b = w.elem_bytes if w.return_value else 0
    out_b = (4 + 8 + 4) if sampling else w.k * (idx_b + val_b)
    done_rows, done_bytes, t_used = 0, 0, 0.0
    r = 0
    while t_used < budget_s and done_rows < 100000:
        sub = slice(r % w.rows, r % w.rows + 1)
        end = None if w.end is None else w.end[sub]
        t0 = time.perf_counter()
        if sampling:
            S.oracle_sample(w.x[sub], w.k, SAMPLE_T, SAMPLE_P, u[sub], end=end, nan_mode=w.nan_mode)
        else:
            O.oracle_topk(w.x[sub], w.dtype, w.k, end=end, sorted_index=w.sorted_index,
                          return_value=w.return_value, index_dtype=w.index_dtype, nan_mode=w.nan_mode)
        t_used += time.perf_counter() - t0
        done_rows += 1
        done_bytes += int(lens[r % w.rows]) * w.elem_bytes + out_b + (4 if w.end is not None else 0)
        r += 1
    return done_bytes / t_used / 1e9, done_rows / t_used, done_rows, t_used


# --------------------------------------------------------------------------- #
# The CPU oracle on all host cores: a pool of spawned worker processes (spawned,
# never forked, so that no worker inherits a CUDA context), each timing whole
# rows of the workload held once in shared memory.
# --------------------------------------------------------------------------- #
_POOL_X = None
_POOL_META = None
_POOL_SHM = None


def _pool_init(shm_name, shape, np_dtype, meta):
    global _POOL_X, _POOL_META, _POOL_SHM
    from multiprocessing import shared_memory
    sys.path.insert(0, ROOT)
    _POOL_SHM = shared_memory.SharedMemory(name=shm_name)
    _POOL_X = np.ndarray(shape, dtype=np_dtype, buffer=_POOL_SHM.buf)
    _POOL_META = meta


def _pool_rows(task):
    """Times the oracle on rows r0, r0 + step, ... until `budget` seconds of wall
    time have passed; returns (rows, effective bytes, seconds)."""
    import oracle.sample_oracle as S
    import oracle.topk_oracle as O
    r0, step, budget = task
    m = _POOL_META
    end_all, lens, u = m["end"], m["lens"], m["u"]
    t0 = time.perf_counter()
    rows = nbytes = 0
    r = r0
    while time.perf_counter() - t0 < budget and rows < 100000:
        rr = r % m["rows"]
        sub = slice(rr, rr + 1)
        end = None if end_all is None else end_all[sub]
        if m["sampling"]:
            S.oracle_sample(_POOL_X[sub], m["k"], SAMPLE_T, SAMPLE_P, u[sub], end=end, nan_mode=m["nan_mode"])
        else:
            O.oracle_topk(_POOL_X[sub], m["dtype"], m["k"], end=end, sorted_index=m["sorted_index"],
                          return_value=m["return_value"], index_dtype=m["index_dtype"], nan_mode=m["nan_mode"])
        rows += 1
        nbytes += int(lens[rr]) * m["elem_bytes"] + m["out_b"]
        r += step
    return rows, nbytes, time.perf_counter() - t0


class OraclePool:
    """All host cores running the oracle over whole rows of one workload."""

    def __init__(self, w: W.Workload, sampling: bool, cores: int = 0):
        import multiprocessing as mp
        from multiprocessing import shared_memory
        self.cores = cores or (os.cpu_count() or 1)
        self.shm = shared_memory.SharedMemory(create=True, size=max(1, w.x.nbytes))
        np.ndarray(w.x.shape, dtype=w.x.dtype, buffer=self.shm.buf)[...] = w.x
        idx_b = 4 if w.index_dtype == "i32" else 8
        val_b = w.elem_bytes if w.return_value else 0
        meta = {"rows": w.rows, "k": w.k, "dtype": w.dtype, "sorted_index": w.sorted_index,
                "return_value": w.return_value, "index_dtype": w.index_dtype, "nan_mode": w.nan_mode,
                "sampling": sampling, "end": w.end, "lens": w.valid_lengths(), "u": W.uniforms(w.rows),
                "elem_bytes": w.elem_bytes,
                "out_b": ((4 + 8 + 4) if sampling else w.k * (idx_b + val_b)) + (4 if w.end is not None else 0)}
        self.pool = mp.get_context("spawn").Pool(self.cores, initializer=_pool_init,
                                                  initargs=(self.shm.name, w.x.shape, w.x.dtype, meta))

    def throughput(self, budget_s: float, start_row: int = 0):
        """(GB/s, rows/s, rows, wall seconds) of all workers over `budget_s` seconds."""
        t0 = time.perf_counter()
        res = self.pool.map(_pool_rows, [(start_row + i, self.cores, budget_s) for i in range(self.cores)])
        wall = time.perf_counter() - t0
        rows = sum(r[0] for r in res)
        nbytes = sum(r[1] for r in res)
        span = max(r[2] for r in res)
        return nbytes / span / 1e9, rows / span, rows, wall

    def close(self):
        self.pool.close()
        self.pool.join()
        self.shm.close()
        self.shm.unlink()


def run_reference(args, w, world, rank):
    """Reference arm: the CPU oracle timed on the host cores, one bounded sample of
    the workload per step (rank 0 only)."""
    if rank != 0:
        return
    # about a minute for the whole run, and no more than --cpu-seconds per step
    per_step_budget = max(0.2, min(args.cpu_seconds, 60.0 / max(args.steps + args.warmup, 1)))
    pool = OraclePool(w, args.workload.startswith("sample_"))
    try:
        for i in range(args.warmup):
            pool.throughput(per_step_budget / 4, start_row=i)
        vals, rows_s, nrows, secs = [], [], 0, 0.0
        for i in range(args.steps):
            gbs, rps, n, t = pool.throughput(per_step_budget, start_row=i * pool.cores)
            vals.append(gbs)
            rows_s.append(rps)
            nrows += n
            secs += t
    finally:
        pool.close()
    value = statistics.median(vals)
    sample = (f"{nrows} whole rows of {w.name} over {args.steps} steps, {pool.cores} worker processes "
              f"({secs:.1f} s wall)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "rows_per_s": round(statistics.median(rows_s), 2), "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1000.0 * secs / max(args.steps, 1), 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": workload_config(args, w, world),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": pool.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(args, w, world):
    return {"workload": w.name, "rows": w.rows, "row_stride": w.row_stride, "k": w.k,
            "dtype": w.dtype, "sorted_index": w.sorted_index, "return_value": w.return_value,
            "index_dtype": w.index_dtype, "end": w.end is not None,
            "global_batch": w.rows * world, "parallelism": f"dp{world} (rows per rank, no collective)",
            "l2": "inputs rotate over copies totalling > 4x L2, so every step reads HBM"}


def run_ours(args, w, world, rank, local, pg):
    import torch
    import row_wise_topk_b200 as T

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(device=dev)
    eb = w.elem_bytes
    in_bytes = w.rows * w.row_stride * eb
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    n_copies = int(max(2, min(64, -(-4 * l2 // in_bytes) + 1)))
    signed = w.x.view(np.int16) if eb == 2 else w.x.view(np.int32)
    host = torch.from_numpy(np.ascontiguousarray(signed)).pin_memory()
    copies = [torch.empty_like(host, device=dev) for _ in range(n_copies)]
    for c in copies:
        c.copy_(host, non_blocking=True)
    end_dev = None if w.end is None else torch.from_numpy(w.end).to(dev)
    itorch = torch.int32 if w.index_dtype == "i32" else torch.int64
    idx_out = torch.empty((w.rows, w.k), dtype=itorch, device=dev)
    val_out = torch.empty((w.rows, w.k), dtype=copies[0].dtype, device=dev) if w.return_value else None
    dt = T.DSEL_BF16 if w.dtype == "bf16" else T.DSEL_F32
    idt = T.DSEL_I32 if w.index_dtype == "i32" else T.DSEL_I64
    nm = T.DSEL_NAN_FLAG if w.nan_mode == "flag" else T.DSEL_NAN_TRAP
    sptr = stream.cuda_stream

    sampling = args.workload.startswith("sample_")
    u_dev = torch.from_numpy(W.uniforms(w.rows)).to(dev)
    tok_out = torch.empty(w.rows, dtype=torch.int64, device=dev)
    prob_out = torch.empty(w.rows, dtype=torch.float32, device=dev)

    def step(i):
        if sampling:
            st = T.dsel_topk_sample(copies[i % n_copies].data_ptr(), w.rows, w.row_stride,
                                    None if end_dev is None else end_dev.data_ptr(), w.k, SAMPLE_T, SAMPLE_P,
                                    u_dev.data_ptr(), nm, None, None, tok_out.data_ptr(), prob_out.data_ptr(),
                                    sptr)
        else:
            st = T.dsel_topk(copies[i % n_copies].data_ptr(), dt, w.rows, w.row_stride,
                             None if end_dev is None else end_dev.data_ptr(), w.k, w.sorted_index,
                             w.return_value, idt, nm, None if val_out is None else val_out.data_ptr(),
                             idx_out.data_ptr(), sptr)
        if st != 0:
            raise T.DselError(st)

    torch.cuda.synchronize(dev)
    # one eager call first (sets kernel attributes, allocates any workspace)
    with torch.cuda.stream(stream):
        step(0)
    torch.cuda.synchronize(dev)

    # graph of S steps (S = number of input copies, so each replay touches every copy once).
    # The timed region replays `graph`, which has nothing between the launches; a
    # second graph with an event pair around every launch gives, in a separate timed
    # pass, the kernels' own durations for the roofline (event nodes between launches
    # add several microseconds per step, so they stay out of the throughput figure).
    S = n_copies
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(S):
            step(i)
    graph_ev = torch.cuda.CUDAGraph()
    ev_a = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(S)]
    ev_b = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(S)]
    with torch.cuda.graph(graph_ev, stream=stream):
        for i in range(S):
            ev_a[i].record()
            step(i)
            ev_b[i].record()
    st_plan, plan = T.dsel_plan_device(dt, w.rows, w.row_stride, w.k,
                                       T.DSEL_ORDER_VALUE if sampling else w.sorted_index)
    if st_plan != 0:
        raise T.DselError(st_plan)
    launches_per_step = 1 + (1 if plan["groups"] > 1 else 0)

    # warm-up
    with torch.cuda.stream(stream):
        for _ in range(max(1, -(-args.warmup // S))):
            graph.replay()
    torch.cuda.synchronize(dev)

    # the timed region runs at least the requested steps and at least min_seconds,
    # so that the clock samples (every 50 ms) fall inside it; `steps` reports the
    # steps actually timed
    probe0 = torch.cuda.Event(enable_timing=True)
    probe1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        probe0.record()
        graph.replay()
        probe1.record()
    torch.cuda.synchronize(dev)
    est_ms = max(probe0.elapsed_time(probe1) / S, 1e-4)
    steps = int(max(args.steps, -(-args.min_seconds * 1000.0 // est_ms)))
    steps = int(max_over_ranks(float(steps), pg, dev))   # every rank times the same steps
    rem = steps % S
    graph_rem = None
    if rem:
        graph_rem = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph_rem, stream=stream):
            for i in range(rem):
                step(i)
    full = steps // S

    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    time.sleep(0.3)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler.mark("t0")
    with torch.cuda.stream(stream):
        t_start.record()
        for _ in range(full):
            graph.replay()
        if graph_rem is not None:
            graph_rem.replay()
        t_end.record()
    torch.cuda.synchronize(dev)
    sampler.mark("t1")
    if pg is not None:
        pg.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    # isolated launch durations: a second timed pass through the graph with events
    # around every launch, on the same stream (at most ~2 s of replays); the events
    # between launches add their own overhead and stop consecutive launches from
    # overlapping, so these read above the timed region's average
    per_step_ms = [elapsed_ms / steps]
    try:
        reps = max(1, min(full, int(2000.0 / max(elapsed_ms / max(full, 1), 1e-3))))
        with torch.cuda.stream(stream):
            for _ in range(reps):
                graph_ev.replay()
        torch.cuda.synchronize(dev)
        per_step_ms = [ev_a[i].elapsed_time(ev_b[i]) for i in range(S)]
    except Exception:      # event nodes unavailable: fall back to the region average
        pass
    time.sleep(0.2)
    clocks = sampler.stop()

    elapsed_ms = max_over_ranks(elapsed_ms, pg, dev)
    ms_per_step = elapsed_ms / steps
    if sampling:   # valid logits read once, u read, token + probability written (+ end)
        eff = int(w.valid_lengths().sum()) * eb + w.rows * (4 + 8 + 4) + (0 if w.end is None else 4 * w.rows)
    else:
        eff = w.effective_bytes()
    value = whole_job_gbs(eff, steps, elapsed_ms, world)
    rows_per_s = world * w.rows * steps / (elapsed_ms / 1e3)

    # roofline of the dominant kernel: algorithmic bytes per launch / average launch time
    kern_ms = roofline_launch_ms(ms_per_step, launches_per_step, per_step_ms)
    peak, peak_kind = hbm_peak()
    achieved = eff / (kern_ms / 1e3) / 1e9
    traffic = recorded_traffic(args.workload)

    # end to end through the public API: pinned H2D of the batch, the call, D2H of
    # the indices (and values), every step
    e2e_steps = max(3, min(args.steps, 50))
    host_idx = torch.empty_like(idx_out, device="cpu").pin_memory()
    host_val = None if val_out is None else torch.empty_like(val_out, device="cpu").pin_memory()
    x_e2e = copies[0]
    xv = x_e2e.view(torch.bfloat16 if eb == 2 else torch.float32)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record()
        for i in range(e2e_steps):
            x_e2e.copy_(host, non_blocking=True)
            if sampling:
                tok, _ = T.topk_sample(xv, w.k, u_dev, temperature=SAMPLE_T, top_p=SAMPLE_P, end=end_dev,
                                       nan_mode=w.nan_mode, stream=sptr)
                host_idx.view(-1)[: w.rows].copy_(tok, non_blocking=True)
            else:
                T.topk(xv, w.k, end=end_dev, sorted_index=w.sorted_index,
                       return_value=bool(w.return_value), index_dtype=itorch, nan_mode=w.nan_mode,
                       out=(val_out, idx_out), stream=sptr)
                host_idx.copy_(idx_out, non_blocking=True)
                if host_val is not None:
                    host_val.copy_(val_out, non_blocking=True)
        e1.record()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev) / e2e_steps
    h2d = in_bytes
    if sampling:
        d2h = w.rows * 8
    else:
        d2h = idx_out.numel() * idx_out.element_size() + (0 if val_out is None else val_out.numel() * val_out.element_size())
    e2e_value = world * eff / (e2e_ms / 1e3) / 1e9

    torch_ctx = torch_topk_context(args, w, copies, stream, eff, ms_per_step, sampling) if args.torch_topk else None

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        gbs1, rps1, nrows1, secs1 = cpu_oracle_throughput(w, args.cpu_seconds)
        pool = OraclePool(w, sampling)
        try:
            gbs, rps, nrows, secs = pool.throughput(args.cpu_seconds)
        finally:
            pool.close()
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": pool.cores, "kind": "oracle",
               "sample": f"{nrows} whole rows of {w.name} on {pool.cores} worker processes "
                         f"({secs:.1f} s wall, numpy)",
               "rows_per_s": round(rps, 2),
               "single_core": {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1, "rows_per_s": round(rps1, 2),
                               "sample": f"{nrows1} whole rows of {w.name} ({secs1:.1f} s, one thread, numpy)"}}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "rows_per_s": round(rows_per_s, 1),
        "n_gpus": world, "steps": steps, "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5), "timed_ms": round(elapsed_ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic", "config": workload_config(args, w, world),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_kind,
                     "kernel": kernel_name(T, plan, launches_per_step),
                     "launch_ms": round(kern_ms, 5),
                     "launch_ms_isolated": {"mean": round(statistics.mean(per_step_ms), 5),
                                            "median": round(statistics.median(per_step_ms), 5),
                                            "min": round(min(per_step_ms), 5)}},
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_value, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": launches_per_step * steps,
        "clocks": clocks,
        "plan": {k_: plan[k_] for k_ in ("kernel", "threads", "cluster", "groups", "stages", "smem_bytes")},
        "input_copies": n_copies,
    }
    if torch_ctx is not None:
        line["context_torch_topk"] = torch_ctx
    print(json.dumps(line), flush=True)


def torch_topk_context(args, w, copies, stream, eff, ms_per_step, sampling):
    """Context only (the pages compare their kernel with torch.topk): torch.topk with
    sorted=False on the same input copies, eager launches on the same stream, timed
    with CUDA events over at least 20 calls and about half a second.  Whole rows
    only: torch.topk has no per-row valid length."""
    import torch
    if sampling or w.end is not None:
        return {"skipped": "per-row end or sampling: torch.topk has no counterpart"}
    try:
        dtype = torch.bfloat16 if w.elem_bytes == 2 else torch.float32
        views = [c.view(dtype) for c in copies]
        with torch.cuda.stream(stream):
            for i in range(3):
                torch.topk(views[i % len(views)], w.k, dim=-1, largest=True, sorted=False)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record()
            torch.topk(views[0], w.k, dim=-1, largest=True, sorted=False)
            b.record()
        torch.cuda.synchronize()
        reps = int(max(20, min(2000, 500.0 / max(a.elapsed_time(b), 1e-3))))
        with torch.cuda.stream(stream):
            a.record()
            for i in range(reps):
                torch.topk(views[i % len(views)], w.k, dim=-1, largest=True, sorted=False)
            b.record()
        torch.cuda.synchronize()
        t_ms = a.elapsed_time(b) / reps
    except Exception as e:   # context only: never costs the line
        return {"skipped": f"torch.topk failed: {type(e).__name__}"}
    return {"call": f"torch.topk(x, {w.k}, dim=-1, sorted=False)", "calls": reps, "ms_per_call": round(t_ms, 5),
            "value": round(eff / (t_ms / 1e3) / 1e9, 2), "unit": "GB/s",
            "ratio_of_ours": round(t_ms / ms_per_step, 2), "torch": torch.__version__,
            "note": "eager launches; same effective bytes as the line's value"}


def kernel_name(T, plan, launches_per_step):
    if plan.get("kernel") == T.DSEL_KERNEL_RESIDENT:
        return "topk_resident_kernel"
    if plan.get("kernel") == T.DSEL_KERNEL_SLICE:
        return "topk_slice_kernel"
    return "topk_stream_kernel" + ("+topk_merge_kernel" if launches_per_step > 1 else "")


def run_long_split(args, world, rank, local, pg):
    """One 2^28-element float32 row split over the ranks (columns), TopK of the whole
    row through ``sharded.topk_row_split``: a local TopK per shard, one NCCL
    all-gather of the k candidates per rank, and the final TopK of the stacked
    candidates, timed end to end per step (strong scaling: the row is fixed, each
    rank holds 1 / N of it).  Each rank's shard is drawn on the host from its own
    seeded generator (U[-1, 1], the long-row workload's distribution)."""
    import torch
    import row_wise_topk_b200 as T
    from row_wise_topk_b200 import sharded

    k = int(args.workload.split("_")[2])
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    n = LONG_SPLIT_N
    if n % (world * 16):
        raise SystemExit("the long_split row must split into shards of whole 16-element units")
    shard_len = n // world
    rng = np.random.default_rng(4 + rank)
    host = torch.from_numpy(rng.uniform(-1.0, 1.0, size=(1, shard_len)).astype(np.float32)).pin_memory()
    x = host.to(dev)
    group = pg.group.WORLD if pg is not None else None

    def step():
        return sharded.topk_row_split(x, k, shard_len=shard_len, group=group, sorted_index=T.DSEL_ORDER_INDEX,
                                      return_value=True, index_dtype=torch.int64, nan_mode="trap")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    p0.record()
    step()
    p1.record()
    torch.cuda.synchronize(dev)
    est_ms = max(p0.elapsed_time(p1), 1e-3)
    steps = int(max(args.steps, -(-args.min_seconds * 1000.0 // est_ms)))
    steps = int(max_over_ranks(float(steps), pg, dev))
    sampler = ClockSampler(physical_gpu_index(local))
    sampler.start()
    time.sleep(0.3)
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler.mark("t0")
    t0.record()
    for _ in range(steps):
        step()
    t1.record()
    torch.cuda.synchronize(dev)
    sampler.mark("t1")
    if pg is not None:
        pg.barrier()
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), pg, dev)
    time.sleep(0.2)
    clocks = sampler.stop()

    # the dominant kernel: this rank's local TopK of its shard, timed alone
    be = sharded.CudaBackend()
    reps = max(3, min(50, steps))
    l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0.record()
    for _ in range(reps):
        be.local_topk(x, k, "trap")
    l1.record()
    torch.cuda.synchronize(dev)
    local_ms = l0.elapsed_time(l1) / reps
    plan = T.dsel_plan_device(T.DSEL_F32, 1, shard_len, k, T.DSEL_ORDER_INDEX)[1]
    local_launches = 1 + (1 if plan["groups"] > 1 else 0)
    shard_bytes = shard_len * 4 + k * (4 + 8)
    peak, peak_kind = hbm_peak()
    achieved = shard_bytes / (local_ms / 1e3) / 1e9

    # end to end: the shard from pinned host memory, the split TopK, the result to the host
    host_i = torch.empty((1, k), dtype=torch.int64).pin_memory()
    host_v = torch.empty((1, k), dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    torch.cuda.synchronize(dev)
    if pg is not None:
        pg.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        x.copy_(host, non_blocking=True)
        v, i = step()
        host_i.copy_(i, non_blocking=True)
        host_v.copy_(v, non_blocking=True)
    e1.record()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev) / e2e_steps
    if rank != 0:
        return
    total = n * 4 + k * (4 + 8)   # the row read once, the k (value, index) pairs written
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        wsub = W.long_rows(1, 1 << 24, k, "uniform")
        gbs1, rps1, nrows1, secs1 = cpu_oracle_throughput(wsub, args.cpu_seconds)
        cpu = {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": f"{nrows1} rows of 2^24 float32 (1/16 of the row), U[-1, 1], k = {k} "
                         f"({secs1:.1f} s, one thread, numpy)"}
    line = {
        "metric": METRIC, "value": round(total * steps / (elapsed_ms / 1e3) / 1e9, 2), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "steps_requested": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / steps, 5), "timed_ms": round(elapsed_ms, 3),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": f"long_split_f32_1x{n}_k{k}", "rows": 1, "row_length": n, "k": k,
                   "shard_len": shard_len, "sorted_index": 1, "return_value": 1, "index_dtype": "i64",
                   "parallelism": f"row split over {world} rank(s): local TopK, NCCL all-gather, final TopK",
                   "l2": "the 1 GiB row (1 / N per rank) exceeds L2 at N <= 8"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": None, "peak_source": peak_kind,
                     "kernel": kernel_name(T, plan, local_launches) + " (local shard TopK)",
                     "launch_ms": round(local_ms / local_launches, 5)},
        "cpu_baseline": cpu,
        "e2e": {"value": round(total / (e2e_ms / 1e3) / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": shard_len * 4, "d2h_bytes_per_step": k * (4 + 8),
                "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": (local_launches + 3) * steps,   # local TopK, stack, final TopK, index take
        "clocks": clocks,
        "plan": {k_: plan[k_] for k_ in ("kernel", "threads", "cluster", "groups", "stages", "smem_bytes")},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="indexer")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="the timed region runs at least this long (more steps than --steps if needed)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--torch-topk", action="store_true",
                    help="also time torch.topk on the same inputs (context only, not part of the line's value)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local, pg = dist_setup(args)
    if args.impl == "ours" and args.workload.startswith("long_split"):
        try:
            run_long_split(args, world, rank, local, pg)
        finally:
            if pg is not None:
                pg.destroy_process_group()
        return
    if args.impl == "reference" and rank != 0:
        w = None   # only rank 0 runs the reference arm
    else:
        w = make_workload(args.workload)
    try:
        if args.impl == "reference":
            run_reference(args, w, world, rank)
        else:
            run_ours(args, w, world, rank, local, pg)
    finally:
        if pg is not None:
            pg.destroy_process_group()


if __name__ == "__main__":
    main()
