"""ctypes front end of the C++ oracle (oracle/alhr_oracle.cpp).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's CPU-baseline
arm are the only users. The library's product path never imports this module, and this
module imports nothing from the library.

All arrays are numpy arrays on the host; one call handles one (batch, head) block.
"""
from __future__ import annotations

import contextlib
import ctypes
import hashlib
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "alhr_oracle.cpp")
_BUILD = os.path.join(_HERE, "_build")


def _so_path() -> str:
    with open(_SRC, "rb") as f:
        digest = hashlib.sha1(f.read()).hexdigest()[:12]
    return os.path.join(_BUILD, f"liboracle_{digest}.so")


def build() -> str:
    """Compile the oracle (g++, -O2, no target-specific flags) if its source changed."""
    so = _so_path()
    if not os.path.exists(so):
        os.makedirs(_BUILD, exist_ok=True)
        tmp = so + f".tmp{os.getpid()}"
        subprocess.run(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-o", tmp, _SRC],
                       check=True)
        os.replace(tmp, so)
    return so


_lib = None


def _configure(L):
    P = ctypes.c_void_p
    I = ctypes.c_int
    L.oracle_build_tree.argtypes = [I, I, P, P]
    L.oracle_build_tree.restype = I
    L.oracle_causal_sum.argtypes = [I, P, I, P]
    L.oracle_causal_sum.restype = None
    L.oracle_predict.argtypes = [I, P, P, P, P]
    L.oracle_predict.restype = I
    L.oracle_route.argtypes = [I, I, P, P, P, I, I, I, I, I, I, P, P, P]
    L.oracle_route.restype = I
    L.oracle_attend.argtypes = [I, P, P, P, P, I, P]
    L.oracle_attend.restype = None
    L.oracle_forward.argtypes = [I, I, I, I, I, I, I, I, P, P, P, P, P, P, P, I, P, P, P, P, P,
                                 P]
    L.oracle_forward.restype = None
    L.oracle_topk_labels.argtypes = [I, I, P, P, I, I, I, P, P]
    L.oracle_topk_labels.restype = None
    L.oracle_time_block.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P, I, P, P, P, P, P, P]
    L.oracle_time_block.restype = ctypes.c_double
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = _configure(ctypes.CDLL(build()))
    return _lib


@contextlib.contextmanager
def use_library(path: str):
    """Run the wrappers against another build of the oracle (used to plant mistakes in a
    copy of the oracle and check that the pins catch them)."""
    global _lib
    saved = _lib
    _lib = _configure(ctypes.CDLL(path))
    try:
        yield
    finally:
        _lib = saved


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def build_tree(K: np.ndarray) -> np.ndarray:
    """K int8 [n, d] -> level-major int32 tree [n-1, d]."""
    K = _c(K, np.int8)
    n, d = K.shape
    nodes = np.zeros((n - 1, d), dtype=np.int32)
    bad = lib().oracle_build_tree(n, d, _p(K), _p(nodes))
    if bad:
        raise OverflowError("tree sum outside int32")
    return nodes


def causal_sum(K: np.ndarray, i: int) -> np.ndarray:
    K = _c(K, np.int8)
    G = np.zeros(K.shape[1], dtype=np.int64)
    lib().oracle_causal_sum(K.shape[1], _p(K), i, _p(G))
    return G


def predict(q: np.ndarray, G: np.ndarray, W: np.ndarray):
    """-> (class c*, logits int64 [32])."""
    q = _c(q, np.int8)
    G = _c(G, np.int64)
    W = _c(W, np.int8)
    logits = np.zeros(32, dtype=np.int64)
    c = lib().oracle_predict(q.shape[0], _p(q), _p(G), _p(W), _p(logits))
    return c, logits


def route(K, nodes, q, i: int, budget: int, window: int, max_keys: int, by_level=False,
          score_norm: bool = False, bucket_log: int = 0):
    """-> (selected positions ascending, (exp_hi, exp_l1)[, expanded nodes per level [32]]).
    score_norm / bucket_log: the mean-normalised and leaf-bucket descent variants."""
    K = _c(K, np.int8)
    nodes = _c(nodes, np.int32)
    q = _c(q, np.int8)
    n, d = K.shape
    sel = np.zeros(max(max_keys, 1), dtype=np.int32)
    exp = np.zeros(2, dtype=np.int32)
    lv = np.zeros(32, dtype=np.int32) if by_level else None
    c = lib().oracle_route(n, d, _p(K), _p(nodes), _p(q), i, budget, window, max_keys,
                           int(bool(score_norm)), int(bucket_log), _p(sel), _p(exp), _p(lv))
    if by_level:
        return sel[:c].copy(), (int(exp[0]), int(exp[1])), lv
    return sel[:c].copy(), (int(exp[0]), int(exp[1]))


def attend(q, K, V_bits, sel) -> np.ndarray:
    """V_bits: uint16 bf16 bit patterns [n, d]; -> float64 [d]."""
    q = _c(q, np.int8)
    K = _c(K, np.int8)
    V_bits = _c(V_bits, np.uint16)
    sel = _c(sel, np.int32)
    out = np.zeros(K.shape[1], dtype=np.float64)
    lib().oracle_attend(K.shape[1], _p(q), _p(K), _p(V_bits), _p(sel), len(sel), _p(out))
    return out


def forward(Q, K, V_bits, nodes, W, budget_override, q_start: int, window: int,
            max_keys: int, rows=None, score_norm: bool = False, bucket_log: int = 0) -> dict:
    """The whole path for one (b,h) block. Q int8 [nq, d]; K int8 [n, d]; V_bits uint16
    [n, d]; nodes int32 [n-1, d] (from build_tree); W int8 [32, 2d] or None; budget_override
    int32 [nq] or None; rows: query rows to compute (None = all).
    -> dict of out float64 [nq,d], idx int32 [nq,max_keys], count, expansions [nq,2], budget,
    by_level int32 [nq,32] (expanded nodes per level)."""
    Q = _c(Q, np.int8)
    K = _c(K, np.int8)
    V_bits = _c(V_bits, np.uint16)
    nodes = _c(nodes, np.int32)
    W = None if W is None else _c(W, np.int8)
    bo = None if budget_override is None else _c(budget_override, np.int32)
    nq, d = Q.shape
    n = K.shape[0]
    rws = None if rows is None else _c(rows, np.int32)
    out = np.zeros((nq, d), dtype=np.float64)
    idx = np.full((nq, max_keys), -1, dtype=np.int32)
    count = np.zeros(nq, dtype=np.int32)
    exp = np.zeros((nq, 2), dtype=np.int32)
    bud = np.zeros(nq, dtype=np.int32)
    lv = np.zeros((nq, 32), dtype=np.int32)
    lib().oracle_forward(n, d, q_start, nq, window, max_keys, int(bool(score_norm)),
                         int(bucket_log), _p(Q), _p(K), _p(V_bits),
                         _p(nodes), _p(W), _p(bo), _p(rws), 0 if rws is None else len(rws),
                         _p(out), _p(idx), _p(count), _p(exp), _p(bud), _p(lv))
    return dict(out=out, idx=idx, count=count, expansions=exp, budget=bud, by_level=lv)


def topk_labels(Q, K, q_start: int, k: int = 16):
    """Phase-2 labels of one (b,h) block: Q int8 [nq, d], K int8 [n, d] -> (labels int32
    [nq, k] best first, -1 padded; scores int32 [nq, k], 0 padded)."""
    Q = _c(Q, np.int8)
    K = _c(K, np.int8)
    nq, d = Q.shape
    labels = np.full((nq, k), -1, dtype=np.int32)
    scores = np.zeros((nq, k), dtype=np.int32)
    lib().oracle_topk_labels(K.shape[0], d, _p(Q), _p(K), q_start, nq, k, _p(labels),
                             _p(scores))
    return labels, scores


def time_block(Q, K, V_bits, W, budget_override, q_start: int, window: int, max_keys: int,
               rows=None) -> tuple[float, dict]:
    """Tree build plus the whole path over the listed query rows (None = all) of one (b,h)
    block, timed inside the oracle library with std::chrono::steady_clock on the calling thread.
    -> (seconds, outputs as forward() without by_level)."""
    Q = _c(Q, np.int8)
    K = _c(K, np.int8)
    V_bits = _c(V_bits, np.uint16)
    W = None if W is None else _c(W, np.int8)
    bo = None if budget_override is None else _c(budget_override, np.int32)
    nq, d = Q.shape
    n = K.shape[0]
    rws = None if rows is None else _c(rows, np.int32)
    nodes = np.empty((n - 1, d), dtype=np.int32)
    out = np.zeros((nq, d), dtype=np.float64)
    idx = np.full((nq, max_keys), -1, dtype=np.int32)
    count = np.zeros(nq, dtype=np.int32)
    exp = np.zeros((nq, 2), dtype=np.int32)
    bud = np.zeros(nq, dtype=np.int32)
    t = lib().oracle_time_block(n, d, q_start, nq, window, max_keys, _p(Q), _p(K), _p(V_bits),
                                _p(W), _p(bo), _p(rws), 0 if rws is None else len(rws),
                                _p(nodes), _p(out), _p(idx), _p(count), _p(exp), _p(bud))
    if t < 0:
        raise OverflowError("tree sum outside int32")
    return float(t), dict(out=out, idx=idx, count=count, expansions=exp, budget=bud)
