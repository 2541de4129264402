"""Seeded synthetic inputs for batched row-wise TopK.

This module only draws numbers: it holds none of the selection arithmetic, so both
the CPU oracle (``oracle/``) and the CUDA path (``row_wise_topk_b200``) can be fed
the very same buffers without sharing any code with one another.

Every generator returns a :class:`Workload`: the raw element bits as a 2-D numpy
array ``[rows, row_stride]`` (``uint16`` holding bfloat16 patterns, or ``uint32``
holding float32 patterns), an optional per-row valid length ``end`` (int32), and
the call options that go with the shape.

The shapes follow the two cases the DeepSelect pages describe ("Inside DeepSeek
V4.1's New Open Inference Toolkit", section "DeepSelect: a fast, deliberately
narrow TopK"; "DeepSeek releases DeepSelect, a TopK kernel for sparse attention
and sampling", coverage paragraph): bfloat16 Lightning-Indexer scores with
k = 512, and float32 sampler logits over a 129,280-token vocabulary, both with
k <= 4096.  The pages print no data, so the value distributions are synthetic:
normal scores, quantised (tie-heavy) scores, boosted "hot" logits, uniform long
rows, sorted and all-equal rows, and rows with one injected NaN.

RNG: numpy ``default_rng(seed)`` (PCG64).  Floats are drawn in float32 (or
float64 and then cast to float32), and bfloat16 inputs are the float32 values
rounded to nearest-even.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

BF16 = "bf16"
F32 = "f32"

SAMPLER_VOCAB = 129_280          # the sampler benchmark's vocabulary length
INDEXER_CONTEXT = 131_072        # indexer context positions per row
BF16_POS_INF = 0x7F80
BF16_QNAN = 0x7FC0
F32_QNAN = 0x7FC00000


@dataclasses.dataclass
class Workload:
    name: str
    dtype: str                       # "bf16" | "f32"
    x: np.ndarray                    # uint16 / uint32 bits, shape [rows, row_stride]
    end: Optional[np.ndarray]        # int32 [rows] or None (every row is row_stride long)
    k: int
    sorted_index: int
    return_value: int
    index_dtype: str                 # "i32" | "i64"
    nan_mode: str = "trap"           # "trap" | "flag"
    nan_rows: Optional[np.ndarray] = None   # rows that received an injected NaN

    @property
    def rows(self) -> int:
        return int(self.x.shape[0])

    @property
    def row_stride(self) -> int:
        return int(self.x.shape[1])

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == BF16 else 4

    def valid_lengths(self) -> np.ndarray:
        if self.end is None:
            return np.full(self.rows, self.row_stride, dtype=np.int64)
        return np.clip(self.end.astype(np.int64), 0, self.row_stride)

    def effective_bytes(self) -> int:
        """Valid input read once + outputs written (+ the end array when given)."""
        idx_b = 4 if self.index_dtype == "i32" else 8
        val_b = self.elem_bytes if self.return_value else 0
        b = int(self.valid_lengths().sum()) * self.elem_bytes
        b += self.rows * self.k * (idx_b + val_b)
        if self.end is not None:
            b += 4 * self.rows
        return b


def bf16_bits_rne(f32: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest, ties to even.

    Inputs here are finite or +-inf, never NaN.
    """
    u = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    rounded = u + np.uint32(0x7FFF) + lsb
    return (rounded >> np.uint32(16)).astype(np.uint16)


def f32_bits(f: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(f, dtype=np.float32).view(np.uint32)


# --------------------------------------------------------------------------- #
# The five workload families
# --------------------------------------------------------------------------- #
def pr1_duplicates(seed: int = 0, rows: int = 4, n: int = 8192, k: int = 64,
                   dup_frac: float = 0.05) -> Workload:
    """float32 N(0,1) rows where 5% of positions are overwritten by exact copies of
    other positions of the same row (forces ties at the selection boundary)."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((rows, n), dtype=np.float32)
    n_dup = int(round(dup_frac * n))
    for r in range(rows):
        tgt = rng.choice(n, size=n_dup, replace=False)
        src = rng.integers(0, n, size=n_dup)
        z[r, tgt] = z[r, src].copy()
    return Workload("pr1_f32_4x8192_k64", F32, f32_bits(z), None, k,
                    sorted_index=1, return_value=1, index_dtype="i64")


def indexer_drift(seed: int = 1, rows: int = 64, n: int = INDEXER_CONTEXT, k: int = 512,
                  sorted_index: int = 0, return_value: int = 0,
                  index_dtype: str = "i32") -> Workload:
    """bfloat16 indexer scores: N(0,1) plus a linear drift of +2 sigma along the row
    (an ascending layout that defeats an in-order threshold)."""
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((rows, n), dtype=np.float32)
    drift = (2.0 * np.arange(n, dtype=np.float64) / max(n - 1, 1)).astype(np.float32)
    x = bf16_bits_rne(z + drift[None, :])
    return Workload(f"indexer_bf16_{rows}x{n}_k{k}", BF16, x, None, k,
                    sorted_index, return_value, index_dtype)


def indexer_varlen(seed: int = 2, rows: int = 4096, stride: int = 16384, k: int = 512,
                   end_lo: int = 256, return_value: int = 0, sorted_index: int = 1) -> Workload:
    """bfloat16 indexer, many rows of variable valid length ``end ~ U{end_lo..stride}``.
    Values are a 256-level uniform quantiser of clip(N(0,1), -4, 4) (heavy ties);
    the padding past ``end`` is +inf so any read past ``end`` would win the top-k."""
    rng = np.random.default_rng(seed)
    end = rng.integers(end_lo, stride + 1, size=rows).astype(np.int32)
    z = rng.standard_normal((rows, stride), dtype=np.float32).astype(np.float64)
    j = np.rint((np.clip(z, -4.0, 4.0) + 4.0) * (255.0 / 8.0))
    q = (-4.0 + j * (8.0 / 255.0)).astype(np.float32)
    x = bf16_bits_rne(q)
    cols = np.arange(stride)[None, :]
    x[cols >= end[:, None]] = BF16_POS_INF
    return Workload(f"indexer_varlen_bf16_{rows}x{stride}_k{k}", BF16, x, end, k,
                    sorted_index, return_value, "i32")


def sampler_logits(batch: int, k: int, seed: int = 3, vocab: int = SAMPLER_VOCAB,
                   n_hot: int = 20, hot_boost: float = 15.0) -> Workload:
    """float32 sampler logits 3*N(0,1) with ``n_hot`` distinct positions per row boosted
    by +15; the row stride is the vocabulary rounded up to 16 elements."""
    rng = np.random.default_rng(seed)
    stride = (vocab + 15) // 16 * 16
    x = np.zeros((batch, stride), dtype=np.float32)
    x[:, :vocab] = 3.0 * rng.standard_normal((batch, vocab), dtype=np.float32)
    for r in range(batch):
        hot = rng.choice(vocab, size=n_hot, replace=False)
        x[r, hot] += np.float32(hot_boost)
    end = None if stride == vocab else np.full(batch, vocab, dtype=np.int32)
    return Workload(f"sampler_f32_{batch}x{vocab}_k{k}", F32, f32_bits(x), end, k,
                    sorted_index=1, return_value=1, index_dtype="i64")


def uniforms(rows: int, seed: int = 5) -> np.ndarray:
    """One float32 uniform in [0, 1) per row: the random numbers of a sampling draw,
    passed to the draw as an input."""
    rng = np.random.default_rng(seed)
    return rng.random(rows, dtype=np.float32)


def long_rows(rows: int, n: int, k: int, variant: str = "uniform", seed: int = 4,
              inject_nan: bool = False) -> Workload:
    """float32 long rows, U[-1, 1] (``uniform``), sorted descending (``desc``) or all
    equal to 0.5 (``equal``).  With ``inject_nan`` one quiet NaN goes to a seeded
    position of each odd row (of row 0 when there is a single row), and the call
    uses the flag-returning NaN mode."""
    rng = np.random.default_rng(seed)
    if variant == "uniform":
        x = rng.uniform(-1.0, 1.0, size=(rows, n)).astype(np.float32)
    elif variant == "desc":
        x = rng.uniform(-1.0, 1.0, size=(rows, n)).astype(np.float32)
        x = -np.sort(-x, axis=1)
    elif variant == "equal":
        x = np.full((rows, n), 0.5, dtype=np.float32)
    else:
        raise ValueError(variant)
    bits = f32_bits(x)
    nan_rows = None
    if inject_nan:
        nan_rows = np.arange(1, rows, 2) if rows > 1 else np.array([0])
        pos = rng.integers(0, n, size=len(nan_rows))
        bits[nan_rows, pos] = np.uint32(F32_QNAN)
    return Workload(f"long_f32_{rows}x{n}_k{k}_{variant}{'_nan' if inject_nan else ''}",
                    F32, bits, None, k, sorted_index=1, return_value=1, index_dtype="i64",
                    nan_mode="flag" if inject_nan else "trap", nan_rows=nan_rows)


def random_small(seed: int, dtype: str, rows: int, stride: int, k: int, *,
                 dist: str = "normal", with_end: bool = False, end_lo: int = 0,
                 sorted_index: int = 1, return_value: int = 1, index_dtype: str = "i64",
                 nan_rows: Optional[np.ndarray] = None, nan_mode: str = "flag") -> Workload:
    """Small mixed cases for parity tests.

    ``dist``: ``normal`` | ``ties`` (values from a handful of levels, +-0 and +-inf
    included) | ``ascending`` | ``equal``.
    """
    rng = np.random.default_rng(seed)
    if dist == "normal":
        f = rng.standard_normal((rows, stride), dtype=np.float32)
    elif dist == "ties":
        levels = np.array([-np.inf, -2.0, -1.0, -0.0, 0.0, 0.5, 1.0, 3.0, np.inf], dtype=np.float32)
        f = levels[rng.integers(0, len(levels), size=(rows, stride))]
    elif dist == "ascending":
        f = np.tile(np.linspace(-3, 3, stride, dtype=np.float32), (rows, 1))
    elif dist == "equal":
        f = np.full((rows, stride), 1.25, dtype=np.float32)
    else:
        raise ValueError(dist)
    bits = bf16_bits_rne(f) if dtype == BF16 else f32_bits(f)
    end = None
    if with_end:
        end = rng.integers(end_lo, stride + 1, size=rows).astype(np.int32)
    if nan_rows is not None and len(nan_rows):
        lens = np.full(rows, stride) if end is None else end
        for r in nan_rows:
            if lens[r] > 0:
                p = int(rng.integers(0, lens[r]))
                bits[r, p] = BF16_QNAN if dtype == BF16 else F32_QNAN
    return Workload(f"small_{dtype}_{rows}x{stride}_k{k}_{dist}", dtype, bits, end, k,
                    sorted_index, return_value, index_dtype, nan_mode=nan_mode,
                    nan_rows=None if nan_rows is None else np.asarray(nan_rows))
