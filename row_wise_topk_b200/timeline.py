"""Phase timeline of the slice kernel (or the streaming kernel's counters), from the
counter build of the library.

Run with the counter build selected, for example::

    ROW_WISE_TOPK_LIB=libdsel_stats.so python -m row_wise_topk_b200.timeline indexer

It replays a CUDA graph of back-to-back calls on one workload (the shapes of
``bench.py``), then reads the phase timestamps that thread 0 of every CTA of the
last launch kept (the SM's cycle counter, converted at the device's clock rate)
and prints, per phase, the median and the maximum over CTAs of the time since the
CTA passed its grid-dependency wait:

- issue: the slice's bulk copies issued;
- landed: the last chunk of the slice arrived and its vector maxima were counted;
- sync #1: the cluster barrier after the vector-maximum histograms;
- threshold: the cluster-wide search for T;
- filter: candidate vectors and elements collected;
- boundary: the cluster barrier after the candidate histograms and the level
  searches down to the boundary key;
- counts: the per-block counts and the cluster barrier that publishes them;
- ranks: the block prefix sums;
- written: the outputs stored.

Also printed: the chunk arrival times of the first CTAs and, per CTA, the
threshold summary and the candidate-list length.  The counter build only adds
timestamps kept in shared memory and written out when each CTA ends.  For a
workload that takes the streaming kernel it prints that kernel's counters
instead: time in the stream of rounds (and in block waits and compactions), in
the final phase, rounds, compactions, candidates appended, vectors given the
exact test and restarted passes.
"""
from __future__ import annotations

import os
import statistics
import sys

import numpy as np

PHASES = [(2, "issue"), (3, "landed"), (4, "sync #1"), (5, "threshold"), (6, "filter"), (7, "boundary"),
          (10, "counts"), (8, "ranks"), (9, "written")]
STATS_CTAS = 8192


def sm_clock_ghz(default: float = 1.965) -> float:
    """The current SM clock of GPU 0 from NVML (the B200's 1965 MHz when unavailable)."""
    try:
        import pynvml
        pynvml.nvmlInit()
        h = pynvml.nvmlDeviceGetHandleByIndex(0)
        mhz = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
        pynvml.nvmlShutdown()
        return mhz / 1000.0 if mhz > 0 else default
    except Exception:
        return default


def stream_counters(T, w, plan, per_launch_us, ghz):
    """The streaming kernel's per-CTA counters of the last launch: medians over CTAs."""
    n = min(w.rows * plan["cluster"] * plan["groups"], STATS_CTAS)
    st = np.array(T.dsel_debug_stats(n), dtype=np.int64)
    us = lambda c: c / ghz / 1000.0
    print(f"{w.name}: streaming kernel, {plan['threads']} threads, clusters of {plan['cluster']}, "
          f"{plan['groups']} cluster(s) per row; {per_launch_us:.2f} us per launch in a graph of back-to-back "
          f"launches; {n} CTAs (medians over CTAs)")
    rows = [("stream phase (rounds) us", us(st[:, 0])), ("  of it waiting for blocks us", us(st[:, 14])),
            ("  of it compacting us", us(st[:, 2])), ("final phase us", us(st[:, 1])), ("total us", us(st[:, 15])),
            ("rounds", st[:, 6]), ("compactions", st[:, 3]), ("candidates appended", st[:, 4]),
            ("vectors given the exact test", st[:, 5]), ("passes restarted (uncertified seed)", st[:, 7])]
    for name, v in rows:
        print(f"{name:<38} {statistics.median(v.tolist()):>12.2f} {max(v.tolist()):>12.2f} (max)")
    # per-round steps of CTA 0 (lane 0 of each warp): [warp][round][event], cycles since its start
    import ctypes
    buf = (ctypes.c_uint64 * (16 * 12 * 10))()
    if T.lib.dsel_debug_stats(ctypes.cast(buf, ctypes.c_void_p), -1, None) != 0:
        return
    tr = np.array(buf[:], dtype=np.uint64).astype(np.int64).reshape(16, 12, 10)
    steps = [(0, 8, "wait"), (8, 1, "screen"), (7, 6, "exact test"), (6, 2, "append"),
             (2, 3, "refill + count barrier"), (3, 4, "overflow"), (4, 5, "compaction")]
    print("CTA 0, rounds 1..9, median over warps (us):")
    print("round " + " ".join(f"{nm:>14}" for _, _, nm in steps))
    for r in range(1, 10):
        cols = []
        for a, b, _ in steps:
            d = [tr[wp, r, b] - tr[wp, r, a] for wp in range(16) if tr[wp, r, a] > 0 and tr[wp, r, b] > 0]
            cols.append(f"{us(statistics.median(d)):>14.2f}" if d else f"{'-':>14}")
        print(f"{r:>5} " + " ".join(cols))


def main(argv=None):
    import torch

    argv = sys.argv[1:] if argv is None else argv
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import row_wise_topk_b200 as T

    name = argv[0] if argv else "indexer"
    w = bench.make_workload(name)
    signed = w.x.view(np.int16) if w.elem_bytes == 2 else w.x.view(np.int32)
    copies = [torch.from_numpy(np.ascontiguousarray(signed)).cuda() for _ in range(8)]
    itorch = torch.int32 if w.index_dtype == "i32" else torch.int64
    idx = torch.empty((w.rows, w.k), dtype=itorch, device="cuda")
    val = torch.empty((w.rows, w.k), dtype=copies[0].dtype, device="cuda") if w.return_value else None
    end = None if w.end is None else torch.from_numpy(w.end).cuda()
    dt = T.DSEL_BF16 if w.dtype == "bf16" else T.DSEL_F32
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    st, plan = T.dsel_plan_for(dt, w.rows, w.row_stride, w.k, w.sorted_index, num_sms=sms)
    if plan["kernel"] not in (T.DSEL_KERNEL_SLICE, T.DSEL_KERNEL_STREAM):
        raise SystemExit(f"{w.name} takes neither the slice nor the streaming kernel (plan {plan})")
    s = torch.cuda.Stream()

    def call(i):
        r = T.dsel_topk(copies[i % len(copies)].data_ptr(), dt, w.rows, w.row_stride,
                        None if end is None else end.data_ptr(), w.k, w.sorted_index, w.return_value,
                        T.DSEL_I32 if w.index_dtype == "i32" else T.DSEL_I64, T.DSEL_NAN_TRAP,
                        None if val is None else val.data_ptr(), idx.data_ptr(), s.cuda_stream)
        if r != 0:
            raise T.DselError(r)

    with torch.cuda.stream(s):
        for i in range(3):
            call(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        for i in range(24):
            call(i)
    g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    per_launch_us = e0.elapsed_time(e1) / 24 * 1000.0

    ghz = sm_clock_ghz()   # cycles per ns
    if plan["kernel"] == T.DSEL_KERNEL_STREAM:
        stream_counters(T, w, plan, per_launch_us, ghz)
        return
    n = min(w.rows * plan["cluster"], STATS_CTAS // 2)
    allst = np.array(T.dsel_debug_stats(STATS_CTAS), dtype=np.int64)
    marks, chunks = allst[:n], allst[STATS_CTAS // 2:STATS_CTAS // 2 + n]
    t0 = marks[:, 1]   # each CTA's grid-dependency wait
    print(f"{w.name}: plan {plan['threads']} threads, clusters of {plan['cluster']}, {plan['stages']} chunks "
          f"per slice; {per_launch_us:.2f} us per launch in a graph of back-to-back launches; {n} CTAs")
    print(f"{'phase':<10} {'median us':>10} {'max us':>10}   (since each CTA's dependency wait)")
    for i, nm in PHASES:
        d = [(marks[c, i] - t0[c]) / ghz / 1000.0 for c in range(n) if marks[c, i] > 0]
        if d:
            print(f"{nm:<10} {statistics.median(d):>10.2f} {max(d):>10.2f}")
    for c in range(min(n, 4)):
        land = [round(float(v - t0[c]) / ghz / 1000.0, 2) for v in chunks[c, 8:16] if v > 0]
        print(f"cta {c}: chunks landed at {land} us; threshold summary {int(marks[c, 14])}, "
              f"list entries {int(marks[c, 15])}, chunk-wait polls (lane 0 of each warp) {int(marks[c, 13])}")


if __name__ == "__main__":
    main()
