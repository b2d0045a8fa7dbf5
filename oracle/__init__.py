"""CPU oracle (test infrastructure only; see msa_oracle.py)."""
from .msa_oracle import (  # noqa: F401
    to_f64, token_scores, block_max_pool, select_blocks, index_select_rows,
    selected_tokens, sdpa, attend_rows, prefill_rows, decode_rows,
)
