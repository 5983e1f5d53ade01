"""The C ABI without a GPU: the library loads, exports every symbol include/*.h declares, and
its host-side checks return the documented status codes before touching the device."""
import ctypes
import glob
import os
import re

import pytest

from conftest import ROOT


@pytest.fixture(scope="module")
def A():
    from tree_routed_sparse_b200 import build
    build.build()
    from tree_routed_sparse_b200 import alhr
    alhr.lib()
    return alhr


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(alhr_[a-z0-9_]+)\s*\(", text))
    return names


def test_every_declared_symbol_is_exported(A):
    declared = _declared()
    assert {"alhr_build_tree", "alhr_predict_budget", "alhr_route", "alhr_attend",
            "alhr_forward"} <= declared
    L = A.lib()
    for name in sorted(declared):
        assert hasattr(L, name), name
    assert set(A.EXPORTS) == declared


def test_only_abi_symbols_are_exported(A):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", A.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert _declared() <= exported
    assert not [s for s in exported if "oracle" in s]


def test_tree_layout_helpers(A):
    L = A.lib()
    assert L.alhr_tree_rows(8) == 7 and L.alhr_tree_rows(1 << 20) == (1 << 20) - 1
    assert L.alhr_tree_rows(6) == 0 and L.alhr_tree_rows(1) == 0 and L.alhr_tree_rows(1 << 21) == 0
    # n = 8, d = 128, value_bound 16: every level narrow (int16 rows of 256 bytes); at d = 64
    # every level is int32 (rows of 256 bytes too)
    assert [L.alhr_tree_level_offset(8, 128, 16, l) for l in (1, 2, 3)] == [0, 4 * 256, 6 * 256]
    assert [L.alhr_tree_level_offset(8, 64, 16, l) for l in (1, 2, 3)] == [0, 4 * 256, 6 * 256]
    assert L.alhr_tree_level_offset(8, 64, 16, 0) == 2**64 - 1
    assert L.alhr_tree_level_offset(8, 64, 16, 4) == 2**64 - 1
    assert L.alhr_tree_level_offset(8, 96, 16, 1) == 2**64 - 1
    assert L.alhr_tree_narrow_levels(16384, 128, 16) == 10
    assert L.alhr_tree_narrow_levels(16384, 128, 0) == 10
    assert L.alhr_tree_narrow_levels(16384, 64, 16) == 0
    assert L.alhr_tree_narrow_levels(1024, 128, 127) == 8 and L.alhr_tree_narrow_levels(8, 128, 1) == 3
    assert L.alhr_tree_narrow_levels(1000, 128, 16) == -1
    assert L.alhr_tree_narrow_levels(8, 128, 128) == -1 and L.alhr_tree_narrow_levels(8, 32, 16) == -1
    assert L.alhr_tree_bytes(6, 64, 16) == 0 and L.alhr_tree_bytes(8, 32, 16) == 0
    assert b"sm_100a" in L.alhr_build_info()


def test_launch_mode_setting(A):
    """The process-wide launch shape: default auto, the three documented values accepted,
    anything else refused without changing the setting."""
    L = A.lib()
    assert A.get_launch_mode() == "auto"
    try:
        for name in ("latency", "throughput", "auto"):
            A.set_launch_mode(name)
            assert A.get_launch_mode() == name
        A.set_launch_mode("latency")
        for bad in (-1, 3, 1 << 30):
            assert L.alhr_set_launch_mode(bad) == 1
            assert A.get_launch_mode() == "latency"
        with pytest.raises(ValueError):
            A.set_launch_mode("fast")
    finally:
        A.set_launch_mode("auto")


@pytest.mark.parametrize("n,d,vb", [(16384, 64, 16), (262144, 128, 16), (1024, 128, 127),
                                    (4096, 128, 3), (2, 64, 0), (2, 128, 0), (1 << 20, 128, 1)])
def test_tree_layout_matches_documented_layout(A, n, d, vb):
    """Level offsets and block size follow the layout of include/alhr.h (levels in order,
    int16 rows up to the narrow level, int32 above), computed here independently."""
    from tree_routed_sparse_b200 import metrics
    L = A.lib()
    narrow = (0 if d == 64 else
              max([l for l in range(0, n.bit_length()) if (vb or 16) << l <= 32767]))
    assert metrics.narrow_levels(n, d, vb) == narrow
    assert L.alhr_tree_narrow_levels(n, d, vb) == narrow
    off = 0
    for lev in range(1, n.bit_length()):
        assert L.alhr_tree_level_offset(n, d, vb, lev) == off
        off += (n >> lev) * (2 * d if lev <= narrow else 4 * d)
    assert L.alhr_tree_bytes(n, d, vb) == off == metrics.tree_block_bytes(n, d, vb)
    assert off % 128 == 0


def _dims(A, **kw):
    base = dict(batch=2, heads=8, n=16384, d=64, q_start=0, nq=16384, window=16, max_keys=96,
                score_bits=0, value_bound=16, score_norm=0, bucket_log=0)
    base.update(kw)
    return A.Dims(*[base[f] for f, _ in A.Dims._fields_])


def test_score_width_choice(A):
    L = A.lib()
    sb = lambda **kw: L.alhr_score_bits(ctypes.byref(_dims(A, **kw)))
    assert sb() == 32                                  # 64 * 16^2 * 8192 < 2^31
    assert sb(d=128) == 32                             # 128 * 256 * 8192 = 2^28
    assert sb(n=262144, d=128) == 64                   # 128 * 256 * 2^17 = 2^32
    assert sb(n=262144, d=128, score_bits=32) == -3   # ALHR_ERR_OVERFLOW
    assert sb(value_bound=127) == 64
    assert sb(score_bits=64) == 64
    assert sb(d=96) == -2 and sb(n=1000) == -1 and sb(window=33) == -2 and sb(max_keys=97) == -2
    assert sb(max_keys=0) == -1 and sb(q_start=1) == -1 and sb(score_bits=16) == -1
    assert sb(batch=65536, heads=32768) == -2         # batch * heads must stay below 2^31
    assert sb(batch=65535, heads=32768) == 32
    # ranked by means, a key's ranking value is q . k * n: the bound doubles
    assert sb(n=65536, d=128) == 32                    # 128 * 256 * 2^15 = 2^30
    assert sb(n=65536, d=128, score_norm=1) == 64      # 128 * 256 * 2^16 = 2^31
    assert sb(n=65536, d=128, score_norm=1, score_bits=32) == -3
    assert sb(score_norm=1) == 32 and sb(bucket_log=4) == 32
    assert sb(score_norm=2) == -1 and sb(bucket_log=-1) == -1 and sb(bucket_log=16) == -1


def test_entry_points_reject_bad_arguments_before_launch(A):
    L = A.lib()
    fake = ctypes.c_void_p(0x10000)     # never dereferenced: every call below fails its checks
    odd = ctypes.c_void_p(0x10008)      # not 16-byte aligned
    odd32 = ctypes.c_void_p(0x10010)    # 16-byte but not 32-byte aligned (enough but for a tree)
    null = None
    d = ctypes.byref(_dims(A))
    assert L.alhr_build_tree(None, fake, fake, null, null) == 1
    assert L.alhr_build_tree(ctypes.byref(_dims(A, n=1000)), fake, fake, null, null) == 1
    assert L.alhr_build_tree(ctypes.byref(_dims(A, d=32)), fake, fake, null, null) == 2
    assert L.alhr_build_tree(d, null, fake, null, null) == 1
    assert L.alhr_build_tree(d, odd, fake, null, null) == 1
    assert L.alhr_forward(d, fake, fake, fake, fake, null, null, fake, null, null, null, null,
                          null, null) == 1            # neither W nor a budget
    assert L.alhr_forward(ctypes.byref(_dims(A, window=0)), fake, fake, fake, fake, fake, null,
                          fake, null, null, null, null, null, null) == 1
    assert L.alhr_forward(ctypes.byref(_dims(A, n=262144, d=128, nq=1, q_start=262143,
                                              score_bits=32)),
                          fake, fake, fake, fake, fake, null, fake, null, null, null, null,
                          null, null) == 3
    assert L.alhr_forward(d, fake, fake, odd, fake, fake, null, fake, null, null, null, null,
                          null, null) == 1
    assert L.alhr_route(d, fake, fake, fake, fake, null, fake, null, null, null) == 1
    assert L.alhr_attend(d, fake, fake, fake, fake, fake, null, null, null) == 1
    assert L.alhr_predict_budget(d, fake, fake, fake, null, fake, null, null) == 1
    n = _dims(A).n
    for lo, hi in ((-1, 1), (3, 2), (0, n + 1), (n, n + 1)):
        assert L.alhr_update_tree(d, fake, fake, lo, hi, null, null) == 1, (lo, hi)
    assert L.alhr_update_tree(d, null, fake, 0, 1, null, null) == 1
    assert L.alhr_update_tree(d, fake, odd, 0, 1, null, null) == 1
    # the tree is read 32 bytes at a time: a 16-byte aligned tree is refused everywhere
    assert L.alhr_build_tree(d, fake, odd32, null, null) == 1
    assert L.alhr_update_tree(d, fake, odd32, 0, 1, null, null) == 1
    assert L.alhr_tree_unpack(d, odd32, fake, null) == 1
    assert L.alhr_tree_pack(d, fake, odd32, null, null) == 1
    assert L.alhr_tree_pack(d, odd, fake, null, null) == 1
    assert L.alhr_tree_pack(d, null, fake, null, null) == 1
    assert L.alhr_tree_pack(ctypes.byref(_dims(A, d=32)), fake, fake, null, null) == 2
    assert L.alhr_forward(d, fake, fake, fake, odd32, fake, null, fake, null, null, null, null,
                          null, null) == 1
    assert L.alhr_route(d, fake, fake, odd32, fake, fake, fake, null, null, null) == 1
    assert L.alhr_predict_budget(d, fake, fake, odd32, fake, fake, null, null) == 1
    assert L.alhr_update_tree(ctypes.byref(_dims(A, d=32)), fake, fake, 0, 1, null, null) == 2
    # nothing to do: no pointer is needed
    assert L.alhr_update_tree(d, null, null, 5, 5, null, null) == 0
    assert L.alhr_forward(ctypes.byref(_dims(A, nq=0)), null, null, null, null, null, null, null,
                          null, null, null, null, null, null) == 0
    assert L.alhr_status_string(3) == b"ALHR_ERR_OVERFLOW"
    assert L.alhr_status_string(99) == b"ALHR_ERR_UNKNOWN"


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from tree_routed_sparse_b200 import alhr
    monkeypatch.setattr(alhr, "_lib", None)
    monkeypatch.setattr(alhr, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        alhr.lib()
