"""Algorithmic byte model of the ALHR inference path (what the algorithm must touch).

Per query at position i of the fused forward (head dimension d, window w, M = i - w + 1 keys
before the window, rowB(level) = d for a key row and 4d for a tree row):
  q row                         d
  causal sum G_i (predictor)    the tree rows of the binary decomposition of [0, i+1)
  remaining descent roots       the blocks of [0, M) not shared with that decomposition (all of
                                them without the predictor), only when the descent runs (r > 0)
  selected window keys          nsel_win * d
  descent                       exp_hi * 4d + exp_l1 * d: one left-child row per expansion (the
                                right child's score is parent - left)
  value rows                    count * 2d (bf16)
  output row                    4d (fp32)
plus the predictor weights (64 d) once per launch. Routed keys' rows are not re-read.
The tree build reads K once and writes every tree row once: n d + (n-1) 4d per (b,h).
The counts come from the run's own outputs (count, expansions, budget), which match the
oracle's bit for bit, so the byte total is exact for the run.
"""
from __future__ import annotations

import numpy as np


def _rows_bytes(bits: np.ndarray, d: int) -> np.ndarray:
    """Sum of rowB over the set bits of each value (bit b = a block of level b)."""
    bits = np.asarray(bits, dtype=np.int64)
    total = np.zeros_like(bits)
    for b in range(0, 40):
        total += ((bits >> b) & 1) * (d if b == 0 else 4 * d)
    return total


def _highest_bit(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.int64)
    out = np.full(x.shape, -1, dtype=np.int64)
    for b in range(0, 40):
        out = np.where((x >> b) & 1, b, out)
    return out


def forward_bytes(positions, d: int, window: int, count, expansions, budget,
                  predictor: bool, max_keys: int = 96) -> int:
    """Algorithmic bytes of one alhr_forward launch over the given queries.

    positions: query positions i (any shape); count, budget: same shape; expansions: [..., 2]."""
    i = np.asarray(positions, dtype=np.int64).ravel()
    count = np.asarray(count, dtype=np.int64).ravel()
    budget = np.asarray(budget, dtype=np.int64).ravel()
    exp = np.asarray(expansions, dtype=np.int64).reshape(-1, 2)
    nwin = np.minimum(window, i + 1)
    b_eff = np.minimum(np.minimum(np.maximum(budget, 1), i + 1), max_keys)
    nsel_win = np.minimum(b_eff, nwin)
    r = b_eff - nsel_win
    A = i + 1
    M = np.maximum(i - window + 1, 0)
    if predictor:
        p = np.where(M > 0, _highest_bit(A ^ M), 62)
        low = (np.int64(2) << np.minimum(p, 61)) - 1
        g_rows = _rows_bytes(A, d)
        rest = M & low
    else:
        g_rows = np.zeros_like(i)
        rest = M
    root_rows = np.where(r > 0, _rows_bytes(rest, d), 0)
    per_q = (d + g_rows + root_rows + nsel_win * d + exp[:, 0] * 4 * d + exp[:, 1] * d
             + count * 2 * d + 4 * d)
    return int(per_q.sum()) + (64 * d if predictor else 0)


def tree_bytes(bh: int, n: int, d: int) -> int:
    return int(bh) * (n * d + (n - 1) * 4 * d)
