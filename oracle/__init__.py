"""CPU oracle for batched row-wise TopK (test infrastructure; see topk_oracle)."""
from .topk_oracle import (  # noqa: F401
    IDX_BAD_END, IDX_NAN, IDX_PAD, ROW_BAD_END, ROW_NAN, ROW_SELECTED, ROW_SHORT,
    OracleResult, brute_force_row, decode, decode_bf16, decode_f32, oracle_topk, select_row,
)
