"""Algorithmic byte model of the ALHR inference path (what the algorithm must touch).

Per query of the fused forward (one (b,h) with head dimension d, window w):
  q row                     d bytes
  window key rows           nwin * d, nwin = min(w, i+1) with the predictor (G_i needs them
                            all), else the selected window keys only
  roots of [0, i-w]         4d per tree root, d for a key root; read with the predictor (G_i)
                            or when the descent runs
  descent                   exp_hi * 4d + exp_l1 * d: one left-child row per expansion (the
                            right child's score is parent - left)
  value rows                count * 2d (bf16)
  output row                4d (fp32)
plus the predictor weights 64 d once per launch. Routed keys' score rows are not re-read.
The tree build touches K once and writes every tree row once: n d + (n-1) 4d per (b,h).
These counts come from the run's own outputs (count, expansions), which match the oracle's
bit for bit, so the byte total is exact for the run.
"""
from __future__ import annotations

import numpy as np


def root_row_bytes(m: np.ndarray, d: int) -> np.ndarray:
    """Bytes of the roots of [0, m) for each m (0 where m <= 0)."""
    m = np.maximum(np.asarray(m, dtype=np.int64), 0)
    total = np.zeros_like(m)
    for b in range(0, 40):
        bit = (m >> b) & 1
        total += bit * (d if b == 0 else 4 * d)
    return total


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
    m = i - window + 1
    win_rows = nwin if predictor else nsel_win
    roots = root_row_bytes(m, d)
    if not predictor:
        roots = np.where(r > 0, roots, 0)
    per_q = (d + win_rows * d + roots + exp[:, 0] * 4 * d + exp[:, 1] * d
             + count * 2 * d + 4 * d)
    return int(per_q.sum()) + (64 * d if predictor else 0)


def tree_bytes(bh: int, n: int, d: int) -> int:
    return int(bh) * (n * d + (n - 1) * 4 * d)
