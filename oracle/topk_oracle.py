"""CPU oracle for batched row-wise TopK.  TEST INFRASTRUCTURE, NOT PRODUCT.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its ``cpu_baseline``
leg and ``--impl reference``) may import this module.  The CUDA library never
calls it and shares no code, table or helper with it: this file compares decoded
float64 values, while the GPU path compares order-preserving unsigned keys.

What it computes (plain definition, not the streaming algorithm)
-----------------------------------------------------------------
"DeepSeek releases DeepSelect, a TopK kernel for sparse attention and sampling"
(narracomm), method paragraph: the kernel keeps a rising threshold and a candidate
buffer, and a radix select cuts the buffer back to k.  The threshold only discards
elements that can no longer be among the k largest, so the method reaches exactly
the k largest entries of each row.  The oracle therefore writes out that
definition directly:

* each element is decoded exactly to float64 (bfloat16 by placing its 16 bits in
  the high half of a float32 pattern; float32 as is);
* the k entries that come first in the total order "value descending, then index
  ascending" are selected, with -0.0 equal to +0.0 and both infinities ordinary
  values (reading: the pages only promise stable, repeatable results -- "DeepSeek
  开源DeepSelect：比torch.topk快二十倍！", section "DeepSelect 的差异化设计" and its
  Q&A on 结果稳定 -- so ties are broken by the smaller index);
* output order: ascending index (the pages' ``sorted_index`` orders by index:
  narracomm, paragraph on install and switches).  With ``sorted_index=0`` the
  order is unspecified and parity compares the set, so the oracle's ascending
  order serves both.

Interface rules taken from the pages
------------------------------------
* Rows of valid length n <= k return all n entries and skip the NaN check
  (narracomm, NaN paragraph; "DeepSeek 在 GitHub 发布 DeepSelect v1.0.0", section
  "PyTorch 接口与 CUDA 环境要求").  Reading: slots n..k-1 are padding, index -1
  and value -inf.
* NaN checking is always on and by default aborts (same passages).  Reading:
  the trap mode reports ``would_trap``; the flag mode marks the row, writes index
  -2 in every slot and a quiet NaN in every value slot.
* ``end`` gives each row's valid range [0, end) inside one batched call (aifluxnews
  section above).  Reading: end < 0 or end > row_stride is invalid; the flag mode
  writes index -3 (and quiet-NaN values), the trap mode clamps end to
  [0, row_stride].
* Values are returned in the input dtype with their original bits (so -0.0 stays
  -0.0); indices are int32 or int64, relative to the row start.

Selection step
--------------
``select_row`` finds the k-th largest value t (``np.partition``, a library
selection), then takes every element greater than t plus the lowest-index
elements equal to t until k are taken.  That is the set the total order picks,
stated directly; ``brute_force_row`` (a full sort under the same total order) pins
it on small rows in the tests.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# row status codes
ROW_SELECTED = 0
ROW_SHORT = 1
ROW_NAN = 2
ROW_BAD_END = 3

IDX_PAD = -1
IDX_NAN = -2
IDX_BAD_END = -3

BF16_NEG_INF = np.uint16(0xFF80)
F32_NEG_INF = np.uint32(0xFF800000)
BF16_QNAN = np.uint16(0x7FC0)
F32_QNAN = np.uint32(0x7FC00000)


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns -> exact float64 (the 16 bits are the high half of a float32)."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):          # NaN patterns stay NaN
        return u32.view(np.float32).astype(np.float64)


def decode_f32(bits: np.ndarray) -> np.ndarray:
    """float32 bit patterns -> exact float64."""
    with np.errstate(invalid="ignore"):
        return np.ascontiguousarray(bits, dtype=np.uint32).view(np.float32).astype(np.float64)


def decode(bits: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return decode_bf16(bits)
    if dtype == "f32":
        return decode_f32(bits)
    raise ValueError(f"unknown dtype {dtype!r}")


def select_row(v: np.ndarray, k: int) -> np.ndarray:
    """Indices (ascending) of the k first entries of ``v`` under value-desc, index-asc.

    ``v`` is float64 without NaN and ``len(v) > k >= 1``.
    """
    n = v.shape[0]
    assert 1 <= k < n
    t = np.partition(v, n - k)[n - k]          # the k-th largest value
    above = np.flatnonzero(v > t)              # fewer than k of these
    tied = np.flatnonzero(v == t)[: k - above.shape[0]]   # smallest indices first
    return np.sort(np.concatenate([above, tied]))


def brute_force_row(v, k: int) -> list:
    """Full sort under (value descending, index ascending); first k, by index.

    Pure Python, for small rows only.  -0.0 == +0.0 in the key comparison.
    """
    order = sorted(range(len(v)), key=lambda i: (-float(v[i]), i))
    return sorted(order[:k])


def value_order(bits: np.ndarray, idx: np.ndarray, dtype: str) -> np.ndarray:
    """Permutation that lists the entries (bits[i], idx[i]) in value order.

    Value order (``sorted_index=2``, float32 only: narracomm, paragraph on install
    and switches) is value descending, ties by ascending index, -0.0 equal to +0.0.
    Reading for the rows no longer than k, which skip the NaN check and so may hold
    a NaN: such a row is put in value order too (as torch.topk would order it), a
    NaN taking its IEEE 754 totalOrder place -- sign bit clear: above +inf, a larger
    payload higher; sign bit set: below -inf, a larger payload lower.
    """
    bits = np.asarray(bits)
    v = decode(bits, dtype)
    nan = np.isnan(v)
    neg = np.signbit(v)
    payload = bits.astype(np.int64) & (0x7F if dtype == "bf16" else 0x7FFFFF)
    cls = np.where(nan, np.where(neg, 0, 2), 1)                  # -NaN < numbers < +NaN
    within = np.where(nan, np.where(neg, payload, -payload), 0)  # rank inside a NaN class
    num = np.where(nan, 0.0, -v) + 0.0                           # value descending, -0.0 == +0.0
    return np.lexsort((np.asarray(idx), num, within, -cls))


@dataclasses.dataclass
class OracleResult:
    indices: np.ndarray                 # [rows, k] int32 | int64
    values: Optional[np.ndarray]        # [rows, k] uint16 | uint32 bits, or None
    status: np.ndarray                  # [rows] int8 (ROW_*)
    would_trap: bool                    # trap mode met a NaN in a row longer than k


def oracle_topk(x_bits: np.ndarray, dtype: str, k: int, *, end: Optional[np.ndarray] = None,
                sorted_index: int = 1, return_value: int = 1, index_dtype: str = "i64",
                nan_mode: str = "trap") -> OracleResult:
    """Row-wise TopK of ``x_bits`` ([rows, row_stride] raw bits) per the pages' rules."""
    if dtype not in ("bf16", "f32"):
        raise ValueError(dtype)
    if not 1 <= k <= 4096:
        raise ValueError("k must be in [1, 4096]")
    rows, stride = x_bits.shape
    idx_t = np.int32 if index_dtype == "i32" else np.int64
    bits_t = np.uint16 if dtype == "bf16" else np.uint32
    neg_inf = BF16_NEG_INF if dtype == "bf16" else F32_NEG_INF
    qnan = BF16_QNAN if dtype == "bf16" else F32_QNAN
    indices = np.full((rows, k), IDX_PAD, dtype=idx_t)
    values = np.full((rows, k), neg_inf, dtype=bits_t) if return_value else None
    status = np.zeros(rows, dtype=np.int8)
    would_trap = False
    for r in range(rows):
        n = stride if end is None else int(end[r])
        if n < 0 or n > stride:
            if nan_mode == "flag":
                status[r] = ROW_BAD_END
                indices[r, :] = IDX_BAD_END
                if values is not None:
                    values[r, :] = qnan
                continue
            n = min(max(n, 0), stride)
        row_bits = x_bits[r, :n]
        if n <= k:
            status[r] = ROW_SHORT
            indices[r, :n] = np.arange(n)
            if values is not None:
                values[r, :n] = row_bits
            continue
        v = decode(row_bits, dtype)
        if np.isnan(v).any():
            if nan_mode == "trap":
                would_trap = True
            status[r] = ROW_NAN
            indices[r, :] = IDX_NAN
            if values is not None:
                values[r, :] = qnan
            continue
        sel = select_row(v, k)
        indices[r, :] = sel
        if values is not None:
            values[r, :] = row_bits[sel]
    return OracleResult(indices, values, status, would_trap)
