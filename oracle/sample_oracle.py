"""CPU oracle for the sampling step that follows TopK on fp32 sampler logits.
TEST INFRASTRUCTURE, NOT PRODUCT.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may import this
module.  The CUDA library never calls it and shares no code with it.

What the pages fix
------------------
"DeepSeek releases DeepSelect, a TopK kernel for sparse attention and sampling"
(narracomm), paragraph "Why rewrite TopK at all?": during sampling, TopK picks
the candidate tokens out of a large vocabulary.  The deepseek-recipe page
(section "deepseek-recipe: the protocol layer is real engineering") lists
temperature and top-p among the generation settings.  The pages print no formula
for the draw itself, so this oracle takes the plainest reading:

1. candidates: the row's top-k (``oracle_topk``), in value-descending order with
   ties by ascending index -- the TopK total order;
2. temperature t > 0: weights e_i = exp((z_i - z_1) / t), z_1 the largest logit,
   and e_i = 1 wherever z_i equals z_1 (the limit; it keeps +-inf logits
   meaningful: a row whose candidates are all -inf draws uniformly among them);
   t <= 0 means greedy, the first candidate;
3. top-p: keep the shortest prefix of c candidates whose weight sum E_c reaches
   top_p * E_m (m = number of candidates); top_p >= 1 keeps all m;
4. draw: with the caller's uniform u in [0, 1), the token is the first kept
   candidate i whose prefix sum E_i exceeds u * E_c;
5. the reported probability is e_token / E_c.

Row rules follow the TopK ones: a row of valid length n <= k samples among its n
entries; a NaN row (flag mode) gives token -2, an invalid ``end`` -3, an empty row
(n = 0) -1, each with probability NaN.  Reading: TopK skips the NaN check on rows
of length <= k, but a softmax over a NaN logit has no meaning, so the sampling
step checks every row it draws from: a NaN among the candidates gives -2 (flag
mode) or a trap (trap mode, reported as ``would_trap``).

The arithmetic here is float64; the GPU computes in float32 (``expf``, float32
prefix sums), so its token can differ only where u * E_c or top_p * E_m lies
within rounding distance of a prefix sum.  ``SampleResult.prefix`` carries the
float64 prefix sums so that a test can recognise those boundary cases.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

from .topk_oracle import IDX_BAD_END, IDX_NAN, IDX_PAD, ROW_BAD_END, ROW_NAN, decode_f32, oracle_topk


@dataclasses.dataclass
class SampleResult:
    token: np.ndarray                 # int64 [rows]
    prob: np.ndarray                  # float64 [rows]
    kept: np.ndarray                  # int64 [rows]: c, candidates left after the top-p cut (0 if none)
    would_trap: bool                  # trap mode met a NaN
    order: List[Optional[np.ndarray]]   # per row: candidate indices in value order (None if no draw)
    prefix: List[Optional[np.ndarray]]  # per row: float64 prefix sums E_1..E_m of the weights


def sample_row(z: np.ndarray, temperature: float, top_p: float, u: float):
    """Steps 2-5 on candidate logits ``z`` already in value order (float64).

    Returns (position in ``z``, probability, c, prefix sums)."""
    m = len(z)
    if m == 0:
        raise ValueError("no candidates")
    if temperature <= 0.0:
        e = np.zeros(m)
        e[0] = 1.0
    else:
        with np.errstate(invalid="ignore", over="ignore"):
            e = np.where(z == z[0], 1.0, np.exp((z - z[0]) / temperature))
    prefix = np.cumsum(e)
    total = prefix[-1]
    if top_p >= 1.0:
        c = m
    else:
        c = int(np.searchsorted(prefix, top_p * total, side="left")) + 1   # first E_c >= top_p * E_m
        c = min(max(c, 1), m)
    target = u * prefix[c - 1]
    pos = int(np.searchsorted(prefix[:c], target, side="right"))          # first E_i > target
    pos = min(pos, c - 1)
    return pos, float(e[pos] / prefix[c - 1]), c, prefix


def oracle_sample(x_bits: np.ndarray, k: int, temperature: float, top_p: float, u: np.ndarray, *,
                  end: Optional[np.ndarray] = None, nan_mode: str = "flag") -> SampleResult:
    """Token per row of fp32 logits ``x_bits`` ([rows, row_stride] uint32 bits)."""
    rows = x_bits.shape[0]
    top = oracle_topk(x_bits, "f32", k, end=end, sorted_index=1, return_value=1, index_dtype="i64",
                      nan_mode=nan_mode)
    token = np.full(rows, IDX_PAD, dtype=np.int64)
    prob = np.full(rows, np.nan)
    kept = np.zeros(rows, dtype=np.int64)
    order: List[Optional[np.ndarray]] = [None] * rows
    prefix: List[Optional[np.ndarray]] = [None] * rows
    would_trap = top.would_trap
    for r in range(rows):
        if top.status[r] == ROW_NAN:
            token[r] = IDX_NAN
            continue
        if top.status[r] == ROW_BAD_END:
            token[r] = IDX_BAD_END
            continue
        idx = top.indices[r]
        idx = idx[idx >= 0]
        if len(idx) == 0:
            continue
        z = decode_f32(x_bits[r, idx].astype(np.uint32))
        if np.isnan(z).any():   # only possible on a short row: TopK did not check it
            token[r] = IDX_NAN
            would_trap = would_trap or nan_mode == "trap"
            continue
        # value order: value descending, then index ascending (-0.0 == +0.0)
        perm = sorted(range(len(idx)), key=lambda i: (-z[i], int(idx[i])))
        idx_o = idx[perm]
        z_o = z[perm].astype(np.float64)
        pos, p, c, pre = sample_row(z_o, temperature, top_p, float(u[r]))
        token[r] = int(idx_o[pos])
        prob[r] = p
        kept[r] = c
        order[r] = idx_o
        prefix[r] = pre
    return SampleResult(token, prob, kept, would_trap, order, prefix)
