"""Work accounting for measurement: useful FLOPs and each kernel's algorithmic bytes/FLOPs.

Useful work (the counting rule of the prefill/decode study): 2 * d_idx FLOPs per
causally visible token per (query, group) for the Index Branch, plus 4 * d FLOPs per
selected token per (query, head) for the Main Branch (QK^T and PV). For query i with
local block b = i // Bk: it selects i + 1 tokens when b + 1 <= k, else
(k - 1) * Bk + (i mod Bk) + 1 (k - 1 full blocks plus the causal part of its own).
"""
from __future__ import annotations

import numpy as np


def _selected_tokens(pos: np.ndarray, Bk: int, k: int) -> np.ndarray:
    bl = pos // Bk
    return np.where(bl + 1 <= k, pos + 1, (k - 1) * Bk + (pos % Bk) + 1).astype(np.float64)


def prefill_useful_flops(N: int, Hq: int, G: int, d: int, d_idx: int, Bk: int, k: int) -> tuple[float, float]:
    i = np.arange(N, dtype=np.int64)
    idx = 2.0 * d_idx * G * float((i + 1).sum())
    main = 4.0 * d * Hq * float(_selected_tokens(i, Bk, k).sum())
    return idx, main


def decode_useful_flops(lengths, Hq: int, G: int, d: int, d_idx: int, Bk: int, k: int) -> tuple[float, float]:
    L = np.asarray(lengths, dtype=np.int64)
    idx = 2.0 * d_idx * G * float(L.sum())
    main = 4.0 * d * Hq * float(_selected_tokens(L - 1, Bk, k).sum())
    return idx, main


def index_kernel_flops(qb_begin: int, qb_end: int, G: int, d_idx: int, Bk: int = 128) -> float:
    """Index Branch score kernels (index_topk, and index_blockmax on the two-kernel path):
    every (query, key) pair whose key block lies before the query's own block, i.e.
    Bk * Bk * qb pairs for query block qb, 2 * d_idx FLOPs each."""
    qb = np.arange(qb_begin, qb_end, dtype=np.float64)
    return 2.0 * d_idx * G * Bk * Bk * float(qb.sum())


def index_kernel_bytes(qb_begin: int, qb_end: int, G: int, d_idx: int, Bk: int = 128) -> float:
    """Compulsory HBM bytes of index_blockmax: the query and key index rows once, the
    packed maxima once (4 bytes per (row, earlier block))."""
    rows = (qb_end - qb_begin) * Bk
    keys = max(qb_end - 1, 0) * Bk
    qb = np.arange(qb_begin, qb_end, dtype=np.float64)
    return 2.0 * G * d_idx * (rows + keys) + 4.0 * G * Bk * float(qb.sum())


def kvouter_flops(N: int, Hq: int, d: int, Bk: int, k: int) -> float:
    """kvouter: per (query, head, selected block) a full 128-key QK^T and PV (the causal
    mask inside the local block does not save tensor work): 4 * d * Bk per block."""
    i = np.arange(N, dtype=np.int64)
    nsel = np.minimum(i // Bk + 1, k).astype(np.float64)
    return 4.0 * d * Bk * Hq * float(nsel.sum())


def main_branch_bytes(N: int, Hq: int, G: int, d: int, Bk: int, k: int) -> dict:
    """Compulsory HBM bytes of the KV-outer pass and of the merge, for N queries."""
    i = np.arange(N, dtype=np.int64)
    nsel = float(np.minimum(i // Bk + 1, k).sum())       # (query, slot) pairs per group
    R = Hq // G
    partial = nsel * G * R * (d * 2 + 8)                 # bf16 partial row + fp32 (m, l) pair
    q_bytes = N * Hq * d * 2
    kv_bytes = 2 * N * G * d * 2
    return {"kvouter": q_bytes + kv_bytes + partial,
            "merge": partial + N * G * k * 4 + N * Hq * d * 2}


def decode_scan_bytes(lengths, G: int, d_idx: int, Bk: int = 128) -> float:
    """decode_scan: every index key of the full blocks before each local block, once."""
    L = np.asarray(lengths, dtype=np.int64)
    return float((((L - 1) // Bk) * Bk).sum()) * G * d_idx * 2
