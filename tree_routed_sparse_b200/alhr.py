"""Thin ctypes binding of libalhr.so (the C ABI declared in include/alhr.h).

Argument marshalling only: shapes are read from the torch tensors, outputs are allocated with
torch on the inputs' device, raw pointers and the current CUDA stream are passed to the C entry
points, and a non-OK status raises AlhrError. Every step of the path runs in the library's CUDA
kernels; there is no fallback of any kind. Loading fails loudly when the library has not been
built (python -m tree_routed_sparse_b200.build).
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libalhr.so")

ALHR_OK = 0
STATUS = {0: "ALHR_OK", 1: "ALHR_ERR_INVALID_ARG", 2: "ALHR_ERR_UNSUPPORTED",
          3: "ALHR_ERR_OVERFLOW", 4: "ALHR_ERR_CUDA"}
DEVERR_BUDGET_LOW = 0x1
DEVERR_VALUE_RANGE = 0x2
DEVERR_INDEX = 0x4
DEVERR_TIMEOUT = 0x8
LAUNCH_MODES = {"auto": 0, "throughput": 1, "latency": 2}

EXPORTS = ["alhr_tree_rows", "alhr_tree_narrow_levels", "alhr_tree_bytes",
           "alhr_tree_level_offset", "alhr_score_bits", "alhr_status_string", "alhr_build_info",
           "alhr_build_tree", "alhr_update_tree", "alhr_tree_unpack", "alhr_predict_budget",
           "alhr_route", "alhr_attend", "alhr_forward", "alhr_set_launch_mode",
           "alhr_get_launch_mode", "alhr_topk_labels", "alhr_tree_pack"]


class AlhrError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


class Dims(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in
                ("batch", "heads", "n", "d", "q_start", "nq", "window", "max_keys",
                 "score_bits", "value_bound", "score_norm", "bucket_log")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library with argument types set. Raises if it was never built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libalhr.so is not built ({LIB_PATH}); run "
                               "`python -m tree_routed_sparse_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        DP = ctypes.POINTER(Dims)
        L.alhr_tree_rows.argtypes, L.alhr_tree_rows.restype = [I32], SZ
        L.alhr_tree_narrow_levels.argtypes = [I32, I32, I32]
        L.alhr_tree_narrow_levels.restype = I32
        L.alhr_tree_bytes.argtypes, L.alhr_tree_bytes.restype = [I32, I32, I32], SZ
        L.alhr_tree_level_offset.argtypes = [I32, I32, I32, I32]
        L.alhr_tree_level_offset.restype = SZ
        L.alhr_score_bits.argtypes, L.alhr_score_bits.restype = [DP], I32
        L.alhr_status_string.argtypes, L.alhr_status_string.restype = [I32], ctypes.c_char_p
        L.alhr_build_info.argtypes, L.alhr_build_info.restype = [], ctypes.c_char_p
        L.alhr_build_tree.argtypes = [DP, P, P, P, P]
        L.alhr_update_tree.argtypes = [DP, P, P, I32, I32, P, P]
        L.alhr_tree_unpack.argtypes = [DP, P, P, P]
        L.alhr_tree_pack.argtypes = [DP, P, P, P, P]
        L.alhr_predict_budget.argtypes = [DP, P, P, P, P, P, P, P]
        L.alhr_route.argtypes = [DP, P, P, P, P, P, P, P, P, P]
        L.alhr_attend.argtypes = [DP, P, P, P, P, P, P, P, P]
        L.alhr_forward.argtypes = [DP, P, P, P, P, P, P, P, P, P, P, P, P, P]
        L.alhr_topk_labels.argtypes = [DP, P, P, I32, P, P, P, P]
        L.alhr_set_launch_mode.argtypes = [I32]
        L.alhr_get_launch_mode.argtypes, L.alhr_get_launch_mode.restype = [], I32
        for f in ("alhr_build_tree", "alhr_update_tree", "alhr_tree_unpack", "alhr_tree_pack",
                  "alhr_predict_budget", "alhr_route", "alhr_attend", "alhr_forward",
                  "alhr_set_launch_mode", "alhr_topk_labels"):
            getattr(L, f).restype = I32
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != ALHR_OK:
        raise AlhrError(status, where)


def set_launch_mode(mode: str) -> None:
    """Process-wide launch shape of the per-query kernels: "auto", "throughput" or "latency"."""
    if mode not in LAUNCH_MODES:
        raise ValueError(f"launch mode {mode!r}: one of {sorted(LAUNCH_MODES)}")
    _check(lib().alhr_set_launch_mode(LAUNCH_MODES[mode]), "alhr_set_launch_mode")


def get_launch_mode() -> str:
    code = lib().alhr_get_launch_mode()
    return {v: k for k, v in LAUNCH_MODES.items()}[code]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def make_dims(Q, K, q_start=0, window=16, max_keys=96, score_bits=0, value_bound=16,
              score_norm=False, bucket_log=0) -> Dims:
    B, H, n, d = K.shape
    nq = 0 if Q is None else Q.shape[2]
    return Dims(B, H, n, d, q_start, nq, window, max_keys, score_bits, value_bound,
                int(bool(score_norm)), int(bucket_log))


def _want(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")


def tree_rows(n: int) -> int:
    return int(lib().alhr_tree_rows(n))


def tree_bytes(n: int, d: int, value_bound: int = 16) -> int:
    """Bytes of one (b,h) block of the tree."""
    return int(lib().alhr_tree_bytes(n, d, value_bound))


def tree_narrow_levels(n: int, d: int, value_bound: int = 16) -> int:
    return int(lib().alhr_tree_narrow_levels(n, d, value_bound))


def tree_level_offset(n: int, d: int, value_bound: int, level: int) -> int:
    return int(lib().alhr_tree_level_offset(n, d, value_bound, level))


def score_bits(dims: Dims) -> int:
    return int(lib().alhr_score_bits(ctypes.byref(dims)))


def build_tree(K: torch.Tensor, tree: torch.Tensor | None = None, value_bound: int = 16,
               dev_err: torch.Tensor | None = None) -> torch.Tensor:
    """K int8 [B,H,n,d] -> the tree, uint8 [B,H,tree_bytes(n,d,value_bound)] (the block
    layout of include/alhr.h: int16 rows for the narrow levels, int32 above)."""
    B, H, n, d = K.shape
    _want(K, torch.int8, (B, H, n, d), "K")
    tb = tree_bytes(n, d, value_bound)
    if tree is None:
        tree = torch.empty((B, H, tb), dtype=torch.uint8, device=K.device)
    _want(tree, torch.uint8, (B, H, tb), "tree")
    dims = make_dims(None, K, value_bound=value_bound)
    _check(lib().alhr_build_tree(ctypes.byref(dims), _ptr(K), _ptr(tree), _ptr(dev_err),
                                 _stream(K.device)), "alhr_build_tree")
    return tree


def update_tree(K: torch.Tensor, tree: torch.Tensor, lo: int, hi: int, value_bound: int = 16,
                dev_err: torch.Tensor | None = None) -> torch.Tensor:
    """After rows [lo, hi) of K changed (e.g. appended keys): updates `tree` in place to equal
    build_tree(K), given that it was the tree of K before the change. Returns `tree`."""
    B, H, n, d = K.shape
    _want(K, torch.int8, (B, H, n, d), "K")
    _want(tree, torch.uint8, (B, H, tree_bytes(n, d, value_bound)), "tree")
    dims = make_dims(None, K, value_bound=value_bound)
    _check(lib().alhr_update_tree(ctypes.byref(dims), _ptr(K), _ptr(tree), int(lo), int(hi),
                                  _ptr(dev_err), _stream(K.device)), "alhr_update_tree")
    return tree


def tree_unpack(tree: torch.Tensor, n: int, d: int, value_bound: int = 16) -> torch.Tensor:
    """The tree as plain level-major int32 rows [B,H,n-1,d] (alhr_tree_unpack)."""
    B, H, tb = tree.shape
    _want(tree, torch.uint8, (B, H, tree_bytes(n, d, value_bound)), "tree")
    nodes = torch.empty((B, H, n - 1, d), dtype=torch.int32, device=tree.device)
    dims = Dims(B, H, n, d, 0, 0, 16, 96, 0, value_bound)
    _check(lib().alhr_tree_unpack(ctypes.byref(dims), _ptr(tree), _ptr(nodes),
                                  _stream(tree.device)), "alhr_tree_unpack")
    return nodes


def tree_pack(nodes: torch.Tensor, value_bound: int = 16, tree: torch.Tensor | None = None,
              dev_err: torch.Tensor | None = None) -> torch.Tensor:
    """Plain level-major int32 rows [B,H,n-1,d] into the tree layout (alhr_tree_pack)."""
    B, H, rows, d = nodes.shape
    n = rows + 1
    _want(nodes, torch.int32, (B, H, rows, d), "nodes")
    tb = tree_bytes(n, d, value_bound)
    if tree is None:
        tree = torch.empty((B, H, tb), dtype=torch.uint8, device=nodes.device)
    _want(tree, torch.uint8, (B, H, tb), "tree")
    dims = Dims(B, H, n, d, 0, 0, 16, 96, 0, value_bound)
    _check(lib().alhr_tree_pack(ctypes.byref(dims), _ptr(nodes), _ptr(tree), _ptr(dev_err),
                                _stream(nodes.device)), "alhr_tree_pack")
    return tree


def predict_budget(Q, K, tree, W, q_start=0, window=16, max_keys=96, score_bits=0,
                   value_bound=16, budget=None, dev_err=None) -> torch.Tensor:
    dims = make_dims(Q, K, q_start, window, max_keys, score_bits, value_bound)
    B, H, nq, d = Q.shape
    if budget is None:
        budget = torch.empty((B, H, nq), dtype=torch.int32, device=Q.device)
    _want(Q, torch.int8, (B, H, nq, d), "Q")
    _want(W, torch.int8, (32, 2 * d), "W")
    _want(budget, torch.int32, (B, H, nq), "budget")
    _check(lib().alhr_predict_budget(ctypes.byref(dims), _ptr(Q), _ptr(K), _ptr(tree), _ptr(W),
                                     _ptr(budget), _ptr(dev_err), _stream(Q.device)),
           "alhr_predict_budget")
    return budget


def route(Q, K, tree, budget, q_start=0, window=16, max_keys=96, score_bits=0,
          value_bound=16, with_expansions=True, idx=None, count=None, dev_err=None,
          score_norm=False, bucket_log=0) -> dict:
    """The descent alone (score_norm / bucket_log select the descent variants)."""
    dims = make_dims(Q, K, q_start, window, max_keys, score_bits, value_bound, score_norm,
                     bucket_log)
    B, H, nq, d = Q.shape
    _want(budget, torch.int32, (B, H, nq), "budget")
    if idx is None:
        idx = torch.empty((B, H, nq, max_keys), dtype=torch.int32, device=Q.device)
    if count is None:
        count = torch.empty((B, H, nq), dtype=torch.int32, device=Q.device)
    _want(idx, torch.int32, (B, H, nq, max_keys), "idx")
    _want(count, torch.int32, (B, H, nq), "count")
    exp = (torch.empty((B, H, nq, 3), dtype=torch.int32, device=Q.device)
           if with_expansions else None)
    _check(lib().alhr_route(ctypes.byref(dims), _ptr(Q), _ptr(K), _ptr(tree), _ptr(budget),
                            _ptr(idx), _ptr(count), _ptr(exp), _ptr(dev_err), _stream(Q.device)),
           "alhr_route")
    return dict(idx=idx, count=count, expansions=exp)


def attend(Q, K, V, idx, count, q_start=0, window=16, max_keys=96, value_bound=16,
           out=None, dev_err=None) -> torch.Tensor:
    dims = make_dims(Q, K, q_start, window, max_keys, 0, value_bound)
    B, H, nq, d = Q.shape
    _want(V, torch.bfloat16, K.shape, "V")
    _want(idx, torch.int32, (B, H, nq, max_keys), "idx")
    if out is None:
        out = torch.empty((B, H, nq, d), dtype=torch.float32, device=Q.device)
    _check(lib().alhr_attend(ctypes.byref(dims), _ptr(Q), _ptr(K), _ptr(V), _ptr(idx),
                             _ptr(count), _ptr(out), _ptr(dev_err), _stream(Q.device)),
           "alhr_attend")
    return out


def forward(Q, K, V, tree, W=None, budget_override=None, q_start=0, window=16, max_keys=96,
            score_bits=0, value_bound=16, out=None, want_idx=False, want_count=False,
            want_expansions=False, want_budget=False, dev_err=None, score_norm=False,
            bucket_log=0) -> dict:
    """The fused path. Returns a dict with `out` and the optional outputs asked for.
    score_norm / bucket_log select the descent variants (include/alhr.h)."""
    dims = make_dims(Q, K, q_start, window, max_keys, score_bits, value_bound, score_norm,
                     bucket_log)
    B, H, nq, d = Q.shape
    dev = Q.device
    _want(Q, torch.int8, (B, H, nq, d), "Q")
    _want(K, torch.int8, (B, H, K.shape[2], d), "K")
    _want(V, torch.bfloat16, K.shape, "V")
    _want(tree, torch.uint8, (B, H, tree_bytes(K.shape[2], d, value_bound)), "tree")
    if W is not None:
        _want(W, torch.int8, (32, 2 * d), "W")
    if budget_override is not None:
        _want(budget_override, torch.int32, (B, H, nq), "budget_override")
    if out is None:
        out = torch.empty((B, H, nq, d), dtype=torch.float32, device=dev)
    res = dict(out=out)
    mk = lambda shape: torch.empty(shape, dtype=torch.int32, device=dev)
    if want_idx:
        res["idx"] = mk((B, H, nq, max_keys))
    if want_count:
        res["count"] = mk((B, H, nq))
    if want_expansions:
        res["expansions"] = mk((B, H, nq, 3))
    if want_budget:
        res["budget"] = mk((B, H, nq))
    _check(lib().alhr_forward(ctypes.byref(dims), _ptr(Q), _ptr(K), _ptr(V), _ptr(tree),
                              _ptr(W), _ptr(budget_override), _ptr(out), _ptr(res.get("idx")),
                              _ptr(res.get("count")), _ptr(res.get("expansions")),
                              _ptr(res.get("budget")), _ptr(dev_err), _stream(dev)),
           "alhr_forward")
    return res


def topk_labels(Q, K, k: int = 16, q_start: int = 0, with_scores: bool = True,
                labels=None, scores=None, dev_err=None) -> dict:
    """Phase-2 labels: for every query, its k best causal keys by exact q . k (best first,
    -1 padded), computed on the tensor cores. Q int8 [B,H,nq,d], K int8 [B,H,n,d]."""
    dims = make_dims(Q, K, q_start)
    B, H, nq, d = Q.shape
    _want(Q, torch.int8, (B, H, nq, d), "Q")
    _want(K, torch.int8, (B, H, K.shape[2], d), "K")
    if labels is None:
        labels = torch.empty((B, H, nq, k), dtype=torch.int32, device=Q.device)
    if scores is None and with_scores:
        scores = torch.empty((B, H, nq, k), dtype=torch.int32, device=Q.device)
    _want(labels, torch.int32, (B, H, nq, k), "labels")
    if scores is not None:
        _want(scores, torch.int32, (B, H, nq, k), "scores")
    _check(lib().alhr_topk_labels(ctypes.byref(dims), _ptr(Q), _ptr(K), int(k), _ptr(labels),
                                  _ptr(scores), _ptr(dev_err), _stream(Q.device)),
           "alhr_topk_labels")
    return dict(labels=labels, scores=scores)
