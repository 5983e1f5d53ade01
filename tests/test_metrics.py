"""The algorithmic byte model on hand-counted cases (N=8, d=2, w=2: the golden example)."""
from tree_routed_sparse_b200 import metrics


def test_hand_counted_query_without_predictor():
    # i=7, B=5: q 2 + roots of [0,6) = levels 2 and 1 -> 2 tree rows 16 + window keys 2*2
    # + expansions 1*8 + 3*2 + values 5*4 + out 8 = 64
    assert metrics.forward_bytes([7], 2, 2, [5], [[1, 3]], [5], predictor=False) == 64


def test_hand_counted_query_with_predictor():
    # causal sum: [0,8) is one block, the root row (8); the roots of [0,6) differ from it
    # (i+1 = 8 and i-w+1 = 6 differ at bit 3), so both are read (16) + W once (64*2)
    assert metrics.forward_bytes([7], 2, 2, [5], [[1, 3]], [5], predictor=True) == 64 + 8 + 128


def test_no_descent_reads_no_roots():
    # B = 2: the window fills the budget; without the predictor no tree row is read
    assert metrics.forward_bytes([7], 2, 2, [2], [[0, 0]], [2], predictor=False) == \
        2 + 2 * 2 + 2 * 4 + 8


def test_shared_blocks_counted_once():
    # i = 20, w = 2: i+1 = 21 = 10101b, i-w+1 = 19 = 10011b differ first at bit 2, so the
    # level-4 block [0,16) is read once for both; G needs bits 2 and 0 of 21 (one tree row of
    # level 2, one key), the descent also bits 1 and 0 of 19 (a level-1 row and a key)
    d = 2
    got = metrics.forward_bytes([20], d, 2, [3], [[0, 0]], [3], predictor=True)
    g_rows = 4 * d + 4 * d + d          # [0,16), [16,20), [20,21)
    roots_rest = 4 * d + d              # [16,18), [18,19)
    assert got == d + g_rows + roots_rest + 2 * d + 3 * 2 * d + 4 * d + 64 * d


def test_tree_bytes():
    assert metrics.tree_bytes(16, 16384, 64) == 16 * (16384 * 64 + 16383 * 256)
