"""B200 (sm_100a) batched row-wise TopK.

A thin ctypes binding over the in-tree CUDA library ``libdsel.so`` (C ABI in
``include/dsel.h``).  Every step of the selection runs in the library's kernels;
this module only marshals arguments.  Importing it fails loudly when the
library has not been built: there is no CPU fallback.

``dsel_topk`` mirrors the C entry point argument for argument (raw device
pointers as integers); ``topk`` is the torch-tensor convenience wrapper.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_HERE = os.path.dirname(os.path.abspath(__file__))
# ROW_WISE_TOPK_LIB may name another build of this same library (for example the
# counter-instrumented libdsel_stats.so); it must sit in this package directory.
LIB_PATH = os.path.join(_HERE, os.path.basename(os.environ.get("ROW_WISE_TOPK_LIB", "libdsel.so")))

# Constants of include/dsel.h
DSEL_BF16, DSEL_F32 = 0, 1
DSEL_I32, DSEL_I64 = 0, 1
DSEL_NAN_TRAP, DSEL_NAN_FLAG = 0, 1
DSEL_ORDER_NONE, DSEL_ORDER_INDEX, DSEL_ORDER_VALUE = 0, 1, 2
DSEL_IDX_PAD, DSEL_IDX_NAN, DSEL_IDX_BAD_END = -1, -2, -3
DSEL_KERNEL_STREAM, DSEL_KERNEL_RESIDENT, DSEL_KERNEL_SLICE = 0, 1, 2
DSEL_OK = 0
DSEL_ERR_SCRATCH_LIMIT = -16
DSEL_NOALLOC_SCRATCH_BYTES = 512 * 1024


class DselPlan(ctypes.Structure):
    _fields_ = [
        ("threads", ctypes.c_int32),
        ("cluster", ctypes.c_int32),
        ("groups", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("b2", ctypes.c_int32),
        ("round", ctypes.c_int32),
        ("capacity", ctypes.c_int32),
        ("stages", ctypes.c_int32),
        ("idx_bits", ctypes.c_int32),
        ("smem_bytes", ctypes.c_int32),
        ("workspace_bytes", ctypes.c_int64),
        ("kernel", ctypes.c_int32),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class DselError(RuntimeError):
    def __init__(self, status: int):
        self.status = status
        super().__init__(f"dsel status {status}: {status_string(status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python row_wise_topk_b200/build.py` "
            "(the CUDA library is required; there is no fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    c_int, c_i64, vp = ctypes.c_int, ctypes.c_int64, ctypes.c_void_p
    lib.dsel_topk.restype = c_int
    lib.dsel_topk.argtypes = [vp, c_int, c_i64, c_i64, vp, ctypes.c_int32, c_int, c_int, c_int, c_int,
                              vp, vp, vp]
    lib.dsel_topk_noalloc.restype = c_int
    lib.dsel_topk_noalloc.argtypes = list(lib.dsel_topk.argtypes)
    lib.dsel_topk_sample.restype = c_int
    lib.dsel_topk_sample.argtypes = [vp, c_i64, c_i64, vp, ctypes.c_int32, ctypes.c_float, ctypes.c_float, vp, c_int,
                                     vp, vp, vp, vp, vp]
    lib.dsel_shard_stack.restype = c_int
    lib.dsel_shard_stack.argtypes = [vp, vp, c_int, c_i64, ctypes.c_int32, ctypes.c_int32, c_i64, c_i64, vp, vp, vp]
    lib.dsel_take_index.restype = c_int
    lib.dsel_take_index.argtypes = [vp, c_i64, vp, c_int, c_i64, ctypes.c_int32, c_int, vp, vp]
    lib.dsel_stride_requirement.restype = c_i64
    lib.dsel_stride_requirement.argtypes = [c_int]
    lib.dsel_status_string.restype = ctypes.c_char_p
    lib.dsel_status_string.argtypes = [c_int]
    lib.dsel_plan_for.restype = c_int
    lib.dsel_plan_for.argtypes = [c_int, c_i64, c_i64, ctypes.c_int32, c_int, ctypes.c_int32, ctypes.c_int32,
                                  ctypes.c_int32, ctypes.POINTER(DselPlan)]
    lib.dsel_plan_device.restype = c_int
    lib.dsel_plan_device.argtypes = [c_int, c_i64, c_i64, ctypes.c_int32, c_int, ctypes.c_void_p]
    lib.dsel_plan_fit.argtypes = [c_int, c_i64, c_i64, ctypes.c_int32, c_int, ctypes.c_int32, ctypes.c_int32,
                                  ctypes.c_void_p, ctypes.c_void_p]
    lib.dsel_plan_fit.restype = c_int
    lib.dsel_plan.restype = c_int
    lib.dsel_plan.argtypes = [c_int, c_i64, c_i64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                              ctypes.c_int32, ctypes.POINTER(DselPlan)]
    lib.dsel_device_status.restype = c_int
    lib.dsel_device_status.argtypes = [ctypes.POINTER(c_int), vp]
    lib.dsel_debug_stats.restype = c_int
    lib.dsel_debug_stats.argtypes = [ctypes.c_void_p, c_i64, vp]
    lib.dsel_version.restype = ctypes.c_char_p
    lib.dsel_version.argtypes = []
    return lib


lib = _load()


# --------------------------------------------------------------------------- #
# Same names as the C ABI
# --------------------------------------------------------------------------- #
def dsel_topk(x: int, dtype: int, rows: int, row_stride: int, end: Optional[int], k: int,
              sorted_index: int, return_value: int, index_dtype: int, nan_mode: int,
              values_out: Optional[int], indices_out: int, stream: Optional[int]) -> int:
    """Raw entry point: pointers are integers (device addresses), returns the status."""
    return lib.dsel_topk(x, dtype, rows, row_stride, end, k, sorted_index, return_value,
                         index_dtype, nan_mode, values_out, indices_out, stream)


def dsel_topk_noalloc(x: int, dtype: int, rows: int, row_stride: int, end: Optional[int], k: int,
                      sorted_index: int, return_value: int, index_dtype: int, nan_mode: int,
                      values_out: Optional[int], indices_out: int, stream: Optional[int]) -> int:
    """Raw allocation-free entry point (same arguments as dsel_topk): for callers
    that cannot let the library allocate device memory.  Uses a static per-device
    scratch of DSEL_NOALLOC_SCRATCH_BYTES; returns DSEL_ERR_SCRATCH_LIMIT when a
    call needs more, and calls that overlap on the GPU must be ordered."""
    return lib.dsel_topk_noalloc(x, dtype, rows, row_stride, end, k, sorted_index, return_value,
                                 index_dtype, nan_mode, values_out, indices_out, stream)


def dsel_topk_sample(x: int, rows: int, row_stride: int, end: Optional[int], k: int, temperature: float,
                     top_p: float, u: int, nan_mode: int, values_out: Optional[int], indices_out: Optional[int],
                     token_out: int, prob_out: Optional[int], stream: Optional[int]) -> int:
    """Raw entry point of TopK + sampling draw on float32 logits (see include/dsel.h):
    pointers are integers (device addresses), returns the status."""
    return lib.dsel_topk_sample(x, rows, row_stride, end, k, temperature, top_p, u, nan_mode, values_out,
                                indices_out, token_out, prob_out, stream)


def dsel_stride_requirement(dtype: int) -> int:
    return lib.dsel_stride_requirement(dtype)


def dsel_status_string(status: int) -> str:
    return lib.dsel_status_string(status).decode()


status_string = dsel_status_string


def dsel_plan(dtype: int, rows: int, row_stride: int, k: int, num_sms: int = 148,
              smem_optin: int = 232448, max_cluster: int = 8) -> Tuple[int, dict]:
    p = DselPlan()
    st = lib.dsel_plan(dtype, rows, row_stride, k, num_sms, smem_optin, max_cluster, ctypes.byref(p))
    return st, p.as_dict()


def dsel_plan_for(dtype: int, rows: int, row_stride: int, k: int, sorted_index: int, num_sms: int = 148,
                  smem_optin: int = 232448, max_cluster: int = 8) -> Tuple[int, dict]:
    p = DselPlan()
    st = lib.dsel_plan_for(dtype, rows, row_stride, k, sorted_index, num_sms, smem_optin, max_cluster,
                           ctypes.byref(p))
    return st, p.as_dict()


def dsel_plan_fit(dtype: int, rows: int, row_stride: int, k: int, sorted_index: int, cluster_fit,
                  num_sms: int = 148, smem_optin: int = 232448) -> Tuple[int, dict]:
    """dsel_plan_for with a given cluster capacity: cluster_fit[c] (c = 0..16) clusters
    of c streaming CTAs fit the device at once (host only)."""
    fit = (ctypes.c_int32 * 17)(*[int(v) for v in cluster_fit])
    p = DselPlan()
    st = lib.dsel_plan_fit(dtype, rows, row_stride, k, sorted_index, num_sms, smem_optin,
                           ctypes.cast(fit, ctypes.c_void_p), ctypes.byref(p))
    return st, p.as_dict()


def dsel_plan_device(dtype: int, rows: int, row_stride: int, k: int, sorted_index: int) -> Tuple[int, dict]:
    """The plan dsel_topk uses on the current device (DSEL_ORDER_VALUE: dsel_topk_sample's)."""
    p = DselPlan()
    st = lib.dsel_plan_device(dtype, rows, row_stride, k, sorted_index, ctypes.byref(p))
    return st, p.as_dict()


def dsel_device_status(stream: Optional[int] = None) -> int:
    out = ctypes.c_int(0)
    st = lib.dsel_device_status(ctypes.byref(out), stream)
    if st != DSEL_OK:
        raise DselError(st)
    return out.value


def dsel_debug_stats(n_ctas: int, stream: Optional[int] = None):
    """Per-CTA counters of the last streaming launch (counter builds only), as a
    list of 16-tuples; raises DselError(DSEL_ERR_UNAVAILABLE) otherwise."""
    buf = (ctypes.c_uint64 * (16 * n_ctas))()
    st = lib.dsel_debug_stats(ctypes.cast(buf, ctypes.c_void_p), n_ctas, stream)
    if st != DSEL_OK:
        raise DselError(st)
    return [tuple(buf[16 * i: 16 * i + 16]) for i in range(n_ctas)]


def dsel_version() -> str:
    return lib.dsel_version().decode()


# --------------------------------------------------------------------------- #
# torch convenience wrapper
# --------------------------------------------------------------------------- #
def topk(x, k: int, *, end=None, sorted_index: int = DSEL_ORDER_INDEX, return_value: bool = True,
         index_dtype=None, nan_mode: str = "trap", out=None, stream=None):
    """Row-wise TopK of a 2-D CUDA tensor (bfloat16 or float32).

    ``x`` must be contiguous in its last dimension with a row stride that is a
    multiple of ``dsel_stride_requirement``; its columns may exceed the valid
    length given by ``end`` (int32 CUDA tensor, one entry per row).  Returns
    ``(values, indices)``; ``values`` is None when ``return_value`` is False.
    ``out`` may supply preallocated ``(values, indices)`` tensors.
    """
    import torch

    if x.dim() != 2:
        raise ValueError("x must be 2-D [rows, row_stride]")
    if x.dtype == torch.bfloat16:
        dt = DSEL_BF16
    elif x.dtype == torch.float32:
        dt = DSEL_F32
    else:
        raise TypeError("x must be bfloat16 or float32")
    if x.stride(1) != 1:
        raise ValueError("x must be contiguous in the last dimension")
    if not x.is_cuda:
        raise ValueError("x must be a CUDA tensor (there is no CPU path)")
    rows = x.shape[0]
    row_stride = x.stride(0) if rows > 1 else x.shape[1]
    if end is None and x.shape[1] != row_stride:
        raise ValueError("rows narrower than their stride need end= (valid length per row)")
    if index_dtype is None:
        index_dtype = torch.int32
    idt = DSEL_I32 if index_dtype == torch.int32 else DSEL_I64
    if out is not None:
        values, indices = out
    else:
        indices = torch.empty((rows, k), dtype=index_dtype, device=x.device)
        values = torch.empty((rows, k), dtype=x.dtype, device=x.device) if return_value else None
    if end is not None:
        if end.dtype != torch.int32 or not end.is_cuda or end.numel() != rows:
            raise ValueError("end must be an int32 CUDA tensor with one entry per row")
        end = end.contiguous()
    if stream is None:
        stream = torch.cuda.current_stream(x.device).cuda_stream
    st = dsel_topk(x.data_ptr(), dt, rows, row_stride, None if end is None else end.data_ptr(), k,
                   sorted_index, 1 if return_value else 0, idt,
                   DSEL_NAN_FLAG if nan_mode == "flag" else DSEL_NAN_TRAP,
                   None if values is None else values.data_ptr(), indices.data_ptr(), stream)
    if st != DSEL_OK:
        raise DselError(st)
    return values, indices


def topk_sample(logits, k: int, u, *, temperature: float = 1.0, top_p: float = 1.0, end=None,
                return_topk: bool = False, nan_mode: str = "trap", stream=None):
    """Sampling draw among the k largest float32 logits of each row.

    ``u`` is a float32 CUDA tensor with one uniform in [0, 1) per row (the caller's
    random numbers).  Returns ``(token, prob)``, int64 and float32 tensors of one
    entry per row, plus ``(values, indices)`` of the TopK in value order when
    ``return_topk`` is set.
    """
    import torch

    if logits.dim() != 2 or logits.dtype != torch.float32 or not logits.is_cuda or logits.stride(1) != 1:
        raise ValueError("logits must be a 2-D float32 CUDA tensor, contiguous in the last dimension")
    rows = logits.shape[0]
    row_stride = logits.stride(0) if rows > 1 else logits.shape[1]
    if end is None and logits.shape[1] != row_stride:
        raise ValueError("rows narrower than their stride need end= (valid length per row)")
    if u.dtype != torch.float32 or not u.is_cuda or u.numel() != rows:
        raise ValueError("u must be a float32 CUDA tensor with one entry per row")
    u = u.contiguous()
    token = torch.empty(rows, dtype=torch.int64, device=logits.device)
    prob = torch.empty(rows, dtype=torch.float32, device=logits.device)
    values = indices = None
    if return_topk:
        values = torch.empty((rows, k), dtype=torch.float32, device=logits.device)
        indices = torch.empty((rows, k), dtype=torch.int64, device=logits.device)
    if end is not None:
        if end.dtype != torch.int32 or not end.is_cuda or end.numel() != rows:
            raise ValueError("end must be an int32 CUDA tensor with one entry per row")
        end = end.contiguous()
    if stream is None:
        stream = torch.cuda.current_stream(logits.device).cuda_stream
    st = dsel_topk_sample(logits.data_ptr(), rows, row_stride, None if end is None else end.data_ptr(), k,
                          float(temperature), float(top_p), u.data_ptr(),
                          DSEL_NAN_FLAG if nan_mode == "flag" else DSEL_NAN_TRAP,
                          None if values is None else values.data_ptr(),
                          None if indices is None else indices.data_ptr(), token.data_ptr(), prob.data_ptr(),
                          stream)
    if st != DSEL_OK:
        raise DselError(st)
    if return_topk:
        return token, prob, (values, indices)
    return token, prob
