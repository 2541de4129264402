"""Row TopK with each row split over the ranks of a process group, one GPU each.

A row too long for one GPU (the 1 x 2^28 and 16 x 2^24 sampler stress rows, or
longer) is cut into contiguous column shards, one per rank.  The exchange is
one collective:

1. every rank selects the k largest of its shard (``dsel_topk``, index order,
   with values, int64 indices relative to the shard);
2. one all-gather of those k (value, index) pairs per row, shard-major
   ``[ranks][rows][k]`` (NCCL over NVLink / NVSwitch);
3. ``dsel_shard_stack`` lays them out as one row of ranks * k candidates per
   input row (indices made global, -inf padding to the stride requirement);
4. ``dsel_topk`` on that row; ``dsel_take_index`` maps its positions back to
   indices in the whole row.

Correctness: none of a row's k largest can be missing from the k largest of its
own shard, and the stacked row keeps the candidates in global index order, so
step 4 breaks ties exactly as a TopK of the whole row would.  Every rank ends
with the same result.  Each shard must hold at least k elements.

The pages keep a row on one device (their multi-CTA split is the within-GPU
case, "DeepSeek releases DeepSelect, a TopK kernel for sparse attention and
sampling", method paragraph); this module is the library's multi-GPU
extension of it.  The steps that touch data run in the library's kernels and
in the collective; this module only sequences them.
"""
from __future__ import annotations

from typing import Optional


def _round_up(v: int, m: int) -> int:
    return (v + m - 1) // m * m


class CudaBackend:
    """The product steps: library kernels and a NCCL all-gather."""

    def local_topk(self, x_shard, k: int, nan_mode: str):
        import torch
        from . import DSEL_ORDER_INDEX, topk

        values, indices = topk(x_shard, k, sorted_index=DSEL_ORDER_INDEX, return_value=True,
                               index_dtype=torch.int64, nan_mode=nan_mode)
        return values, indices

    def all_gather(self, values, indices, group):
        import torch
        import torch.distributed as dist

        if not dist.is_initialized():   # a single process: the gather is the identity
            return values.unsqueeze(0), indices.unsqueeze(0)
        world = dist.get_world_size(group)
        vg = torch.empty((world,) + tuple(values.shape), dtype=values.dtype, device=values.device)
        ig = torch.empty((world,) + tuple(indices.shape), dtype=indices.dtype, device=indices.device)
        dist.all_gather_into_tensor(vg, values.contiguous(), group=group)
        dist.all_gather_into_tensor(ig, indices.contiguous(), group=group)
        return vg, ig

    def stack(self, vals_g, idx_g, k: int, shard_len: int, out_stride: int):
        import torch
        from . import DSEL_BF16, DSEL_F32, DselError, lib

        shards, rows = vals_g.shape[0], vals_g.shape[1]
        vs = torch.empty((rows, out_stride), dtype=vals_g.dtype, device=vals_g.device)
        ix = torch.empty((rows, out_stride), dtype=torch.int64, device=vals_g.device)
        dt = DSEL_BF16 if vals_g.dtype == torch.bfloat16 else DSEL_F32
        st = lib.dsel_shard_stack(vals_g.data_ptr(), idx_g.data_ptr(), dt, rows, k, shards, shard_len, out_stride,
                                  vs.data_ptr(), ix.data_ptr(), torch.cuda.current_stream(vals_g.device).cuda_stream)
        if st != 0:
            raise DselError(st)
        return vs, ix

    def final_topk(self, stacked, k: int, sorted_index: int, return_value: bool, nan_mode: str):
        import torch
        from . import topk

        return topk(stacked, k, sorted_index=sorted_index, return_value=return_value, index_dtype=torch.int64,
                    nan_mode=nan_mode)

    def take(self, table, pos, index_dtype):
        import torch
        from . import DSEL_I32, DSEL_I64, DselError, lib

        rows, k = pos.shape
        out = torch.empty((rows, k), dtype=index_dtype, device=pos.device)
        st = lib.dsel_take_index(table.data_ptr(), table.shape[1], pos.data_ptr(),
                                 DSEL_I64 if pos.dtype == torch.int64 else DSEL_I32, rows, k,
                                 DSEL_I32 if index_dtype == torch.int32 else DSEL_I64, out.data_ptr(),
                                 torch.cuda.current_stream(pos.device).cuda_stream)
        if st != 0:
            raise DselError(st)
        return out


def topk_row_split(x_shard, k: int, *, shard_len: int, group=None, sorted_index: int = 1,
                   return_value: bool = True, index_dtype=None, nan_mode: str = "trap",
                   backend: Optional[object] = None):
    """TopK of rows whose columns are split over the ranks of ``group``.

    ``x_shard`` is this rank's ``[rows, shard_len]`` block: columns
    ``[rank * shard_len, (rank + 1) * shard_len)`` of every row (bfloat16 or
    float32, contiguous, stride meeting the stride requirement).  Returns
    ``(values, indices)`` of the whole rows, identical on every rank; indices are
    relative to the row start.  Collective: every rank of ``group`` must call it
    with the same ``k``, ``shard_len`` and options, in the same order.
    """
    import torch
    import torch.distributed as dist

    be = backend if backend is not None else CudaBackend()
    if index_dtype is None:
        index_dtype = torch.int64
    if shard_len < k:
        raise ValueError("every shard must hold at least k elements")
    if x_shard.shape[1] != shard_len:
        raise ValueError("x_shard must be [rows, shard_len]")
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    values, indices = be.local_topk(x_shard, k, nan_mode)
    vals_g, idx_g = be.all_gather(values, indices, group)
    stride = _round_up(world * k, 16)
    stacked, table = be.stack(vals_g, idx_g, k, shard_len, stride)
    fvals, pos = be.final_topk(stacked, k, sorted_index, return_value, nan_mode)
    findex = be.take(table, pos, index_dtype)
    return fvals, findex
