"""The algorithmic byte model on hand-counted cases (N=8, d=2, w=2: the golden example), and
the tree layout sizes."""
import numpy as np
import pytest

from tree_routed_sparse_b200 import metrics

# d = 2 (not 128): every tree level is int32, a tree row is 4d bytes


def test_hand_counted_query_without_predictor():
    # i=7, B=5: q 2 + roots of [0,6) = levels 2 and 1 -> 2 tree rows 16 + window keys 2*2
    # + expansions 1*8 + 3*2 + values 5*4 + out 8 = 64
    assert metrics.forward_bytes([7], 8, 2, 2, [5], [[1, 3, 1]], [5], predictor=False) == 64


def test_hand_counted_query_with_predictor():
    # the causal sum is formed from the roots of [0,6) and the window keys, which the query
    # reads anyway (same 64 bytes as without the predictor) + W once (64*2)
    assert metrics.forward_bytes([7], 8, 2, 2, [5], [[1, 3, 1]], [5], predictor=True) == \
        64 + 128


def test_narrow_rows_at_d128():
    # value_bound 127 at d = 128: narrow levels 1..8 (127 * 256 <= 32767); at n = 1024 the
    # expansion of a level-10 node reads a level-9 int32 row (4d), of a level-9 node an int16
    # level-8 row (2d)
    assert metrics.narrow_levels(1024, 128, 127) == 8 and metrics.narrow_levels(1024, 64, 127) == 0
    base = metrics.forward_bytes([1000], 1024, 128, 2, [3], [[1, 0, 0]], [3], predictor=False,
                                 value_bound=127)
    wide = metrics.forward_bytes([1000], 1024, 128, 2, [3], [[1, 0, 1]], [3], predictor=False,
                                 value_bound=127)
    assert wide - base == 2 * 128


def test_no_descent_reads_no_roots():
    assert metrics.forward_bytes([7], 8, 2, 2, [2], [[0, 0, 0]], [2], predictor=False) == \
        2 + 2 * 2 + 2 * 4 + 8


def test_predictor_reads_every_root_and_window_key():
    # i = 20, w = 2, budget 1: no descent and one selected key, but the causal sum G_i still
    # needs every root of [0, 19) (19 = 10011b: levels 4, 1, 0) and both window keys
    d = 2
    got = metrics.forward_bytes([20], 32, d, 2, [1], [[0, 0, 0]], [1], predictor=True)
    roots = 4 * d + 4 * d + d
    assert got == d + roots + 2 * d + 1 * 2 * d + 4 * d + 64 * d
    # without the predictor the same query reads neither the roots nor the unselected key
    assert metrics.forward_bytes([20], 32, d, 2, [1], [[0, 0, 0]], [1], predictor=False) == \
        d + d + 2 * d + 4 * d


def test_g_from_blocks_counts_the_blocks_of_the_prefix():
    # i = 20, w = 2: i+1 = 21 = 10101b, i-w+1 = 19 = 10011b differ first at bit 2, so the
    # level-4 block [0,16) is read once for both; G needs bits 2 and 0 of 21 (a level-2 row, a
    # key), the descent also bits 1 and 0 of 19 (a level-1 row and a key); only the selected
    # window keys are read
    d = 2
    got = metrics.forward_bytes([20], 32, d, 2, [3], [[0, 0, 0]], [3], predictor=True,
                                g_from_blocks=True)
    g_rows = 4 * d + 4 * d + d          # [0,16), [16,20), [20,21)
    roots_rest = 4 * d + d              # [16,18), [18,19)
    assert got == d + g_rows + roots_rest + 2 * d + 3 * 2 * d + 4 * d + 64 * d
    # the algorithmic count of the same query (G_i from the roots and the window keys, which the
    # query reads anyway): the roots of [0,19) and both window keys
    plain = metrics.forward_bytes([20], 32, d, 2, [3], [[0, 0, 0]], [3], predictor=True)
    assert plain == d + (4 * d + 4 * d + d) + 2 * d + 3 * 2 * d + 4 * d + 64 * d


@pytest.mark.parametrize("n,d,vb", [(16384, 64, 16), (16384, 128, 16), (262144, 128, 16),
                                    (1024, 128, 127), (8, 128, 0), (2, 128, 1)])
def test_tree_block_bytes(n, d, vb):
    narrow = metrics.narrow_levels(n, d, vb)
    L = n.bit_length() - 1
    expect = sum((n >> l) * (2 * d if l <= narrow else 4 * d) for l in range(1, L + 1))
    assert metrics.tree_block_bytes(n, d, vb) == expect
    assert narrow == ({(16384, 128): 10, (262144, 128): 10}.get((n, d), narrow))
    if d == 64:
        assert narrow == 0


def test_bucket_keys_are_read_once_more():
    """Same counters, buckets of 4: the routed keys' rows (count - window keys) are read once
    more; a query whose routed budget holds no whole bucket reads no roots."""
    d, n, w = 64, 1024, 16
    pos = np.array([500])
    exp = np.array([[20, 0, 20]])
    base = metrics.forward_bytes(pos, n, d, w, [40], exp, [40], False)
    with_b = metrics.forward_bytes(pos, n, d, w, [40], exp, [40], False, bucket_log=2)
    assert with_b - base == (40 - 16) * d
    none = np.array([[0, 0, 0]])
    a = metrics.forward_bytes(pos, n, d, w, [16], none, [19], False, bucket_log=2)  # r = 3 < 4
    b = metrics.forward_bytes(pos, n, d, w, [16], none, [19], False)                # r = 3
    assert b - a == metrics._rows_bytes(np.array([500 - w + 1]), d, 0)[0]


def test_tree_build_launch_count_follows_the_build_plan():
    """bench.py's launch count of one alhr_build_tree: no streaming launch below 16 keys (one
    shared-memory launch of up to 7 levels), else a streaming launch of 5 levels (7 from 2^24
    keys in all) and one launch per further 7 levels."""
    import bench
    assert bench.tree_build_launches(1, 8) == 1           # 3 levels, one launch
    assert bench.tree_build_launches(1, 16) == 1          # 4 levels streamed at once
    assert bench.tree_build_launches(1, 32) == 1          # 5 levels streamed
    assert bench.tree_build_launches(64, 256) == 2        # 5 streamed + 3
    assert bench.tree_build_launches(16, 16384) == 3      # 5 + 7 + 2
    assert bench.tree_build_launches(512, 262144) == 3    # 2^27 keys: 7 + 7 + 4
    assert bench.tree_build_launches(1, 1 << 20) == 4     # 2^20 keys (small build): 5 + 7 + 7 + 1
