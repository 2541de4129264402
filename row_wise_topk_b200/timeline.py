"""Phase timeline of the slice kernel, from the counter build of the library.

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
timestamps kept in shared memory and written out when each CTA ends.
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
    if plan["kernel"] != T.DSEL_KERNEL_SLICE:
        raise SystemExit(f"{w.name} does not take the slice kernel (plan {plan})")
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

    n = min(w.rows * plan["cluster"], STATS_CTAS // 2)
    allst = np.array(T.dsel_debug_stats(STATS_CTAS), dtype=np.int64)
    marks, chunks = allst[:n], allst[STATS_CTAS // 2:STATS_CTAS // 2 + n]
    t0 = marks[:, 1]   # each CTA's grid-dependency wait
    ghz = sm_clock_ghz()   # cycles per ns
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
              f"list entries {int(marks[c, 15])}")


if __name__ == "__main__":
    main()
