"""Algorithmic byte model of the ALHR inference path (what the algorithm must touch).

Row sizes: a key row d bytes, a tree row of a narrow level (at d = 128, value_bound * 2^l <=
32767, stored as int16) 2d bytes, any other tree row 4d bytes. Per query at position i of the
fused forward (window w, M = i - w + 1 keys before the window):
  q row                         d
  forest roots                  the blocks of [0, M), one row each: always with the predictor
                                (they and the window keys give the causal sum G_i), else only
                                when the descent runs (r > 0)
  window keys                   all min(w, i+1) of them with the predictor (G_i), else only the
                                nsel_win selected ones: d each
(g_from_blocks: the warp-per-query kernel at d = 64 forms G_i from the blocks of the binary
decomposition of [0, i+1) instead; it then reads those rows, the roots below the blocks they
share only when the descent runs, and only the nsel_win selected window keys.)
  descent                       one left-child row per expanded node (the right child's score
                                is parent - left): exp_wide * 4d + (exp_hi - exp_wide) * 2d +
                                exp_l1 * d
  value rows                    count * 2d (bf16)
  output row                    4d (fp32)
plus the predictor weights (64 d) once per launch. Routed keys' rows are not re-read, except
under the leaf-bucket variant, where the kept buckets' keys are read once to be scored.
The tree build reads K once and writes every tree row once. The counters (count, the three
expansion counters, budgets) come from the run's own outputs, which match the oracle's, so the
byte total is exact for the run.
"""
from __future__ import annotations

import numpy as np


def narrow_levels(n: int, d: int, value_bound: int = 16) -> int:
    """At d = 128: the largest l with value_bound * 2^l <= 32767, capped at log2 n; at d = 64:
    0 (every level int32)."""
    if d != 128:
        return 0
    vb = 16 if value_bound == 0 else value_bound
    L = int(n).bit_length() - 1
    nl = 0
    while nl < L and (vb << (nl + 1)) <= 32767:
        nl += 1
    return nl


def row_bytes(level: int, d: int, narrow: int) -> int:
    if level == 0:
        return d
    return 2 * d if level <= narrow else 4 * d


def _rows_bytes(bits: np.ndarray, d: int, narrow: int) -> np.ndarray:
    """Sum of row bytes over the set bits of each value (bit b = a block of level b)."""
    bits = np.asarray(bits, dtype=np.int64)
    total = np.zeros_like(bits)
    for b in range(0, 40):
        total += ((bits >> b) & 1) * row_bytes(b, d, narrow)
    return total


def _highest_bit(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, dtype=np.int64)
    out = np.full(x.shape, -1, dtype=np.int64)
    for b in range(0, 40):
        out = np.where((x >> b) & 1, b, out)
    return out


def forward_bytes(positions, n: int, d: int, window: int, count, expansions, budget,
                  predictor: bool, max_keys: int = 96, value_bound: int = 16,
                  bucket_log: int = 0, g_from_blocks: bool = False) -> int:
    """Algorithmic bytes of one alhr_forward launch over the given queries.

    positions: query positions i (any shape); count, budget: same shape; expansions: [..., 3]
    (level >= 2 expanded, level 1 expanded, expanded with an int32 child row). With leaf
    buckets (bucket_log > 0) the descent runs only when r >> bucket_log > 0, and the keys of the
    kept buckets are read once more to be scored. g_from_blocks: the rows the d = 64
    warp-per-query kernel reads for G_i (see the module docstring)."""
    narrow = narrow_levels(n, d, value_bound)
    i = np.asarray(positions, dtype=np.int64).ravel()
    count = np.asarray(count, dtype=np.int64).ravel()
    budget = np.asarray(budget, dtype=np.int64).ravel()
    exp = np.asarray(expansions, dtype=np.int64).reshape(-1, 3)
    nwin = np.minimum(window, i + 1)
    b_eff = np.minimum(np.minimum(np.maximum(budget, 1), i + 1), max_keys)
    nsel_win = np.minimum(b_eff, nwin)
    r = b_eff - nsel_win
    M = np.maximum(i - window + 1, 0)
    descends = (r >> bucket_log) > 0
    if predictor and g_from_blocks:
        A = i + 1
        p = np.where(M > 0, _highest_bit(A ^ M), 62)
        low = (np.int64(2) << np.minimum(p, 61)) - 1
        g_rows = _rows_bytes(A, d, narrow) + np.where(descends, _rows_bytes(M & low, d, narrow), 0)
        win_keys = nsel_win * d
    elif predictor:
        g_rows = _rows_bytes(M, d, narrow)
        win_keys = nwin * d
    else:
        g_rows = np.where(descends, _rows_bytes(M, d, narrow), 0)
        win_keys = nsel_win * d
    descent = exp[:, 2] * 4 * d + (exp[:, 0] - exp[:, 2]) * 2 * d + exp[:, 1] * d
    if bucket_log > 0:
        descent = descent + (count - nsel_win) * d
    per_q = d + g_rows + win_keys + descent + count * 2 * d + 4 * d
    return int(per_q.sum()) + (64 * d if predictor else 0)


def tree_block_bytes(n: int, d: int, value_bound: int = 16) -> int:
    narrow = narrow_levels(n, d, value_bound)
    L = int(n).bit_length() - 1
    return sum((n >> l) * row_bytes(l, d, narrow) for l in range(1, L + 1))


def tree_bytes(bh: int, n: int, d: int, value_bound: int = 16) -> int:
    """Algorithmic bytes of one tree build: K read once, every tree row written once."""
    return int(bh) * (n * d + tree_block_bytes(n, d, value_bound))
