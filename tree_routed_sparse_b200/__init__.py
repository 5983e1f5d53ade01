"""B200 (sm_100a) inference path of ALHR tree attention.

Importing the package loads nothing native. The compute entry points live in
`tree_routed_sparse_b200.alhr` (a thin ctypes binding of libalhr.so); the first access to
them loads the library and raises if it has not been built. Seeded synthetic inputs live in
`tree_routed_sparse_b200.synth`.
"""
import importlib

__all__ = ["alhr", "synth", "build_tree", "predict_budget", "route", "attend", "forward"]

_LAZY = {"build_tree", "predict_budget", "route", "attend", "forward", "Dims", "AlhrError"}


def __getattr__(name):
    if name in ("alhr", "synth", "metrics"):
        return importlib.import_module(f"{__name__}.{name}")
    if name in _LAZY:
        return getattr(importlib.import_module(f"{__name__}.alhr"), name)
    raise AttributeError(name)
