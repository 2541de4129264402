"""Helpers shared by the GPU tests: run a workload through the C ABI and compare
with the CPU oracle.  Device memory comes from torch; the call itself is the raw
``dsel_topk`` entry point."""
import numpy as np
import torch

import oracle.topk_oracle as O
import row_wise_topk_b200 as T
import workloads as W


def to_device_bits(x: np.ndarray) -> torch.Tensor:
    signed = x.view(np.int16) if x.dtype == np.uint16 else x.view(np.int32)
    return torch.from_numpy(np.ascontiguousarray(signed)).cuda()


def run_gpu(w: W.Workload, *, order=None, return_value=None, index_dtype=None, nan_mode=None,
            x_dev=None, end_dev=None, sync=True):
    order = w.sorted_index if order is None else order
    rv = w.return_value if return_value is None else return_value
    idt = w.index_dtype if index_dtype is None else index_dtype
    nm = w.nan_mode if nan_mode is None else nan_mode
    if x_dev is None:
        x_dev = to_device_bits(w.x)
    if end_dev is None and w.end is not None:
        end_dev = torch.from_numpy(w.end.astype(np.int32)).cuda()
    itorch = torch.int32 if idt == "i32" else torch.int64
    vtorch = torch.int16 if w.dtype == "bf16" else torch.int32
    idx = torch.full((w.rows, w.k), 12345, dtype=itorch, device="cuda")
    val = torch.full((w.rows, w.k), 77, dtype=vtorch, device="cuda") if rv else None
    st = T.dsel_topk(x_dev.data_ptr(), T.DSEL_BF16 if w.dtype == "bf16" else T.DSEL_F32, w.rows,
                     w.row_stride, None if end_dev is None else end_dev.data_ptr(), w.k, order, rv,
                     T.DSEL_I32 if idt == "i32" else T.DSEL_I64,
                     T.DSEL_NAN_FLAG if nm == "flag" else T.DSEL_NAN_TRAP,
                     None if val is None else val.data_ptr(), idx.data_ptr(),
                     torch.cuda.current_stream().cuda_stream)
    assert st == 0, T.dsel_status_string(st)
    if sync:
        torch.cuda.synchronize()
    bits_t = np.uint16 if w.dtype == "bf16" else np.uint32
    out_idx = idx.cpu().numpy()
    out_val = None if val is None else val.cpu().numpy().view(bits_t)
    return out_idx, out_val


def expected(w: W.Workload, rows=None, *, return_value=None, index_dtype=None, nan_mode=None):
    sub = w.x if rows is None else w.x[rows]
    end = w.end if (w.end is None or rows is None) else w.end[rows]
    return O.oracle_topk(sub, w.dtype, w.k, end=end, sorted_index=1,
                         return_value=w.return_value if return_value is None else return_value,
                         index_dtype=w.index_dtype if index_dtype is None else index_dtype,
                         nan_mode=w.nan_mode if nan_mode is None else nan_mode)


def compare(w: W.Workload, got_idx, got_val, exp: O.OracleResult, order, rows=None):
    """Element-by-element comparison; index order is canonicalised when the
    requested order leaves it unspecified, and value order is checked against the
    oracle's set sorted by (value desc, index asc)."""
    rows = np.arange(w.rows) if rows is None else np.asarray(rows)
    gi = got_idx[rows].astype(np.int64)
    gv = None if got_val is None else got_val[rows]
    ei = exp.indices.astype(np.int64)
    ev = exp.values
    for n, r in enumerate(rows):
        if exp.status[n] == O.ROW_SELECTED and order == T.DSEL_ORDER_NONE:
            perm = np.argsort(gi[n], kind="stable")
            gi_r = gi[n][perm]
            gv_r = None if gv is None else gv[n][perm]
            ei_r, ev_r = ei[n], None if ev is None else ev[n]
        elif exp.status[n] in (O.ROW_SELECTED, O.ROW_SHORT) and order == T.DSEL_ORDER_VALUE:
            # value order: the oracle's entries (a short row's real ones; its padding
            # stays at the end) put in value order by the oracle's value_order
            m = int((ei[n] >= 0).sum())
            bits = ev[n][:m] if ev is not None else w.x[r][ei[n][:m]]
            perm = np.concatenate([O.value_order(bits, ei[n][:m], w.dtype), np.arange(m, ei.shape[1])])
            ei_r = ei[n][perm]
            ev_r = None if ev is None else ev[n][perm]
            gi_r, gv_r = gi[n], None if gv is None else gv[n]
        else:
            gi_r, gv_r = gi[n], None if gv is None else gv[n]
            ei_r, ev_r = ei[n], None if ev is None else ev[n]
        if not np.array_equal(gi_r, ei_r):
            bad = np.flatnonzero(gi_r != ei_r)[:8]
            raise AssertionError(f"{w.name} row {r}: index mismatch at {bad.tolist()} "
                                 f"got {gi_r[bad].tolist()} want {ei_r[bad].tolist()} "
                                 f"(status {exp.status[n]})")
        if gv_r is not None and not np.array_equal(gv_r, ev_r):
            bad = np.flatnonzero(gv_r != ev_r)[:8]
            raise AssertionError(f"{w.name} row {r}: value mismatch at {bad.tolist()}")


def check(w: W.Workload, order=None, rows=None, **kw):
    order = w.sorted_index if order is None else order
    gi, gv = run_gpu(w, order=order, **kw)
    exp = expected(w, rows, return_value=kw.get("return_value"), index_dtype=kw.get("index_dtype"),
                   nan_mode=kw.get("nan_mode"))
    compare(w, gi, gv, exp, order, rows)
    return gi, gv
