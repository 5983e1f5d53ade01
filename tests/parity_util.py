"""Helpers shared by the GPU parity tests: run the oracle on the same seeded inputs."""
import numpy as np
import torch

from oracle import oracle as orc
from tree_routed_sparse_b200 import metrics


def decode_tree(block: np.ndarray, n: int, d: int, value_bound: int = 16) -> np.ndarray:
    """One (b,h) block of the tree bytes -> level-major int32 rows [n-1, d], read with the
    layout documented in include/alhr.h (levels in order; at d = 128 int16 rows for
    value_bound * 2^l <= 32767, int32 otherwise), independently of the library's unpack kernel."""
    block = np.ascontiguousarray(block, dtype=np.uint8)
    narrow = metrics.narrow_levels(n, d, value_bound)
    out = np.zeros((n - 1, d), dtype=np.int32)
    off, row0 = 0, 0
    for lev in range(1, n.bit_length()):
        rows = n >> lev
        if lev <= narrow:
            part = block[off: off + rows * 2 * d].view(np.int16).reshape(rows, d)
            off += rows * 2 * d
        else:
            part = block[off: off + rows * 4 * d].view(np.int32).reshape(rows, d)
            off += rows * 4 * d
        out[row0: row0 + rows] = part
        row0 += rows
    assert off == len(block)
    return out


def v_bits(V: torch.Tensor) -> np.ndarray:
    return V.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_slice(inp_cpu: dict, wl, b: int, h: int, rows=None, nodes=None, score_norm=False,
                 bucket_log=0) -> dict:
    """Oracle results for the (b, h) block of a workload's inputs (host tensors); score_norm /
    bucket_log select the descent variants."""
    K = inp_cpu["K"][b, h].numpy()
    Q = inp_cpu["Q"][b, h].numpy()
    V = v_bits(inp_cpu["V"][b, h])
    if nodes is None:
        nodes = orc.build_tree(K)
    W = None if inp_cpu["W"] is None else inp_cpu["W"].numpy()
    bo = None if inp_cpu["budget_override"] is None else inp_cpu["budget_override"][b, h].numpy()
    res = orc.forward(Q, K, V, nodes, W, bo, q_start=wl.q_start, window=wl.window,
                      max_keys=wl.max_keys, rows=rows, score_norm=score_norm,
                      bucket_log=bucket_log)
    res["nodes"] = nodes
    res["narrow"] = metrics.narrow_levels(wl.n, wl.d, max(-wl.qk_lo, wl.qk_hi))
    return res


def compare_rows(gpu: dict, ref: dict, b: int, h: int, rows, tol=1e-3, what=""):
    """Bit-exact idx/count/expansions/budget and |out - oracle| <= tol on the given rows."""
    rows = np.asarray(rows)
    for key in ("idx", "count", "expansions", "budget"):
        if key in gpu:
            g = gpu[key][b, h].cpu().numpy()[rows]
            r = ref[key][rows]
            if key == "expansions":
                # GPU: {level >= 2, level 1, children stored as int32 rows}; the oracle gives the
                # first two and a per-level histogram for the third
                wide = ref["by_level"][rows][:, ref["narrow"] + 2:].sum(1)
                r = np.concatenate([r, wide[:, None]], axis=1).astype(np.int32)
            if not np.array_equal(g, r):
                bad = np.nonzero((g != r).reshape(len(rows), -1).any(1))[0][:5]
                raise AssertionError(f"{what} {key} differs at rows {rows[bad].tolist()}:\n"
                                     f"gpu {g[bad].tolist()}\noracle {r[bad].tolist()}")
    if "out" in gpu:
        g = gpu["out"][b, h].cpu().numpy()[rows].astype(np.float64)
        err = np.abs(g - ref["out"][rows]).max() if len(rows) else 0.0
        assert err <= tol, f"{what} max |out - oracle| = {err:.3e} > {tol}"
        return float(err)
    return 0.0
