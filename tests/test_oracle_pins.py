"""Pins of the oracle to facts that do not come from the oracle itself.

Sources of truth used here:
  * the hand-worked N=8, d=2 example in tests/golden/alhr_n8_d2.json (derived by hand from
    the ALHR README, sections "Inference stage" and "Training stage");
  * closed forms: the root is the sum of all keys; the causal sum telescopes; a planted key
    is always routed; with a beam at least as wide as the past, every past key is routed and
    every internal node of the forest is expanded exactly once;
  * a dense causal softmax attention written independently with numpy (the Monodratic-style
    check of a sparse selected-set attention against a dense masked one);
  * an independent range-based formulation of the descent (recursive halving of [lo, hi)
    intervals, node sums taken straight from K, a full Python sort) on small random inputs.
"""
import math

import numpy as np
import pytest

from oracle import oracle as orc


def _rng(seed):
    return np.random.default_rng(seed)


def _rand_qk(rng, shape, lo=-16, hi=16):
    return rng.integers(lo, hi + 1, size=shape).astype(np.int8)


def _rand_v_bits(rng, shape):
    v = rng.standard_normal(shape).astype(np.float32)
    bits = v.view(np.uint32)
    # round to nearest even bf16
    bits = ((bits + 0x7FFF + ((bits >> 16) & 1)) >> 16).astype(np.uint16)
    return bits


def _bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------- hand-worked example

def test_golden_tree(golden_n8):
    K = np.array(golden_n8["K"], dtype=np.int8)
    nodes = orc.build_tree(K)
    assert nodes.tolist() == golden_n8["tree_level_major"]


def test_golden_causal_sums(golden_n8):
    K = np.array(golden_n8["K"], dtype=np.int8)
    for case in golden_n8["causal_sums"]:
        assert orc.causal_sum(K, case["i"]).tolist() == case["G"], case["why"]


def test_golden_routes(golden_n8):
    K = np.array(golden_n8["K"], dtype=np.int8)
    nodes = orc.build_tree(K)
    for case in golden_n8["routes"]:
        sel, exp = orc.route(K, nodes, np.array(case["q"], dtype=np.int8), case["i"],
                             case["budget"], golden_n8["window"], golden_n8["max_keys"])
        assert sel.tolist() == case["selected"], case["why"]
        assert list(exp) == case["expansions"], case["why"]


def test_roots_not_pruned_before_the_first_expansion(golden_n8):
    """Hand-worked on the N=8, d=2 keys of the golden example, q = (1, 2), i = 7, w = 1, B = 2:
    the window is {7}, r = 1, and the forest of [0, 7) has three roots, more than the beam:
    [0,4) (sum (2,3), score 8), [4,6) (sum (1,3), score 7) and key 6 (score -4). The descent
    expands every non-leaf root before it prunes (reading R6): [0,2) 3, [2,4) 5, key 4 9, key 5
    -2, key 6 -4, of which key 4 is kept: selection {4, 7}, one level-2 and one level-1 node
    expanded. Pruning the roots first would follow [0,4) down to key 3 instead."""
    K = np.array(golden_n8["K"], dtype=np.int8)
    nodes = orc.build_tree(K)
    sel, exp = orc.route(K, nodes, np.array([1, 2], dtype=np.int8), 7, 2, 1, 96)
    assert sel.tolist() == [4, 7]
    assert list(exp) == [1, 1]


def test_golden_predictor(golden_n8):
    for case in golden_n8["predictor"]:
        W = np.zeros((32, 4), dtype=np.int8)
        for row, vals in case.get("W_rows", {}).items():
            W[int(row)] = vals
        c, _ = orc.predict(np.array(case["q"], dtype=np.int8),
                           np.array(case["G"], dtype=np.int64), W)
        assert c == case["class"], case["why"]
        assert 3 * (c + 1) == case["budget"]


def test_golden_forward_composition(golden_n8):
    """The slice entry point reproduces the hand-worked routes when given their budgets."""
    K = np.array(golden_n8["K"], dtype=np.int8)
    nodes = orc.build_tree(K)
    rng = _rng(1)
    V = _rand_v_bits(rng, (8, 2))
    cases = [c for c in golden_n8["routes"] if c["i"] == 7]
    for case in cases:
        Q = np.array([case["q"]], dtype=np.int8)
        res = orc.forward(Q, K, V, nodes, None, np.array([case["budget"]], dtype=np.int32),
                          q_start=7, window=2, max_keys=96)
        c = res["count"][0]
        assert res["idx"][0, :c].tolist() == case["selected"]
        assert (res["idx"][0, c:] == -1).all()
        assert res["expansions"][0].tolist() == case["expansions"]


# ---------------------------------------------------------------- tree closed forms

@pytest.mark.parametrize("n,d", [(2, 2), (8, 3), (64, 64), (1024, 64), (256, 128)])
def test_tree_root_and_children(n, d):
    rng = _rng(n + d)
    K = _rand_qk(rng, (n, d))
    nodes = orc.build_tree(K)
    L = int(math.log2(n))
    off = lambda l: n - (n >> (l - 1))
    # the root is the sum of every key
    assert (nodes[off(L)] == K.astype(np.int64).sum(0)).all()
    # level 1 holds key pairs, every higher node the sum of its two children
    lvl1 = nodes[off(1): off(1) + n // 2].astype(np.int64)
    assert (lvl1 == K[0::2].astype(np.int64) + K[1::2]).all()
    for l in range(2, L + 1):
        par = nodes[off(l): off(l) + (n >> l)].astype(np.int64)
        ch = nodes[off(l - 1): off(l - 1) + (n >> (l - 1))].astype(np.int64)
        assert (par == ch[0::2] + ch[1::2]).all()


def test_tree_planted_key_marks_its_ancestors():
    n, d = 256, 4
    for p in [0, 1, 77, 255]:
        K = np.zeros((n, d), dtype=np.int8)
        K[p] = [16, -16, 3, 0]
        nodes = orc.build_tree(K)
        for l in range(1, 9):
            off = n - (n >> (l - 1))
            for j in range(n >> l):
                expect = K[p] if j == (p >> l) else np.zeros(d, dtype=np.int8)
                assert (nodes[off + j] == expect).all()


def test_tree_extreme_values_exact():
    n, d = 4096, 64
    K = np.full((n, d), -16, dtype=np.int8)
    K[::3] = 16
    nodes = orc.build_tree(K)
    assert nodes[-1, 0] == int(K[:, 0].astype(np.int64).sum())


# ---------------------------------------------------------------- causal sum and predictor

def test_causal_sum_telescopes_and_ends_at_root():
    rng = _rng(5)
    n, d = 128, 16
    K = _rand_qk(rng, (n, d))
    nodes = orc.build_tree(K)
    prev = np.zeros(d, dtype=np.int64)
    for i in range(n):
        G = orc.causal_sum(K, i)
        assert (G - prev == K[i]).all()
        prev = G
    assert (prev == nodes[-1]).all()


def test_predictor_against_numpy_argmax():
    rng = _rng(7)
    for d in [2, 64, 128]:
        for _ in range(30):
            q = _rand_qk(rng, (d,))
            G = rng.integers(-16 * 5000, 16 * 5000, size=d).astype(np.int64)
            W = rng.integers(-4, 5, size=(32, 2 * d)).astype(np.int8)
            c, logits = orc.predict(q, G, W)
            x = np.concatenate([q.astype(np.int64), G])
            ref = W.astype(np.int64) @ x
            assert (logits == ref).all()
            assert c == int(np.argmax(ref))  # numpy argmax returns the first maximum


def test_predictor_ties_go_to_lowest_class():
    d = 8
    q = np.ones(d, dtype=np.int8)
    G = np.ones(d, dtype=np.int64)
    W = np.zeros((32, 2 * d), dtype=np.int8)
    assert orc.predict(q, G, W)[0] == 0
    W[[5, 9, 30]] = 1
    assert orc.predict(q, G, W)[0] == 5


# ---------------------------------------------------------------- route closed forms

def _forest_internal_counts(m):
    """(level>=2 internal nodes, level-1 internal nodes) of the forest of [0, m)."""
    hi = l1 = 0
    for b in range(64):
        if (m >> b) & 1 and b >= 1:
            l1 += 1 << (b - 1)
            hi += (1 << (b - 1)) - 1
    return hi, l1


@pytest.mark.parametrize("n,w", [(64, 16), (128, 1), (256, 5), (1024, 16)])
def test_wide_beam_routes_the_whole_past(n, w):
    rng = _rng(n * 31 + w)
    d = 8
    K = _rand_qk(rng, (n, d))
    nodes = orc.build_tree(K)
    for i in rng.choice(n, size=12, replace=False):
        i = int(i)
        q = _rand_qk(rng, (d,))
        sel, exp = orc.route(K, nodes, q, i, budget=n + 5, window=w, max_keys=n + 5)
        assert sel.tolist() == list(range(i + 1))
        m = i - w + 1
        assert exp == (_forest_internal_counts(m) if m > 0 else (0, 0))


@pytest.mark.parametrize("n,w", [(64, 4), (512, 16), (1024, 2)])
def test_planted_positive_key_is_routed(n, w):
    """K is zero except key p with q . k_p > 0: every node holding p scores above every other
    node (which all score 0), so p survives each pruning; the remaining r-1 places go to the
    lowest positions by the tie rule."""
    rng = _rng(n + w)
    d = 4
    q = np.array([1, 2, -1, 3], dtype=np.int8)
    for _ in range(25):
        i = int(rng.integers(w + 1, n))
        m = i - w + 1
        p = int(rng.integers(0, m))
        K = np.zeros((n, d), dtype=np.int8)
        K[p] = [5, 5, 1, 2]
        nodes = orc.build_tree(K)
        B = int(rng.integers(w + 1, w + 40))
        sel, _ = orc.route(K, nodes, q, i, B, w, max_keys=96)
        b_eff = min(B, i + 1, 96)
        r = b_eff - w
        others = [t for t in range(m) if t != p][: r - 1]
        expect = sorted(set(range(i - w + 1, i + 1)) | {p} | set(others))
        assert sel.tolist() == expect


def test_route_structure_random():
    rng = _rng(11)
    n, d = 512, 16
    K = _rand_qk(rng, (n, d))
    nodes = orc.build_tree(K)
    for _ in range(200):
        i = int(rng.integers(0, n))
        w = int(rng.integers(1, 33))
        B = int(rng.integers(-2, 110))
        mk = int(rng.integers(1, 97))
        q = _rand_qk(rng, (d,))
        sel, exp = orc.route(K, nodes, q, i, B, w, mk)
        b_eff = min(max(B, 1), i + 1, mk)
        assert len(sel) == b_eff  # min(B_eff, i+1) == B_eff
        assert (np.diff(sel) > 0).all()
        nwin = min(b_eff, w, i + 1)
        assert sel[-nwin:].tolist() == list(range(i - nwin + 1, i + 1))
        routed = sel[:-nwin]
        assert (routed <= i - w).all() and (routed >= 0).all()


def _alt_route(K, q, i, B, w, max_keys, norm=False, bucket_log=0):
    """Independent formulation: intervals [lo, hi) halved recursively, sums straight from K,
    roots as the largest aligned blocks taken greedily from the left. norm ranks intervals by
    their exact mean score (a Fraction); bucket_log makes intervals of at most 2^bucket_log keys
    leaves, the beam r >> bucket_log wide, and selects every key of the kept intervals."""
    from fractions import Fraction
    bsz = 1 << bucket_log
    b_eff = min(max(B, 1), i + 1, max_keys)
    win = [t for t in range(i, max(-1, i - w), -1)][:b_eff]
    r = b_eff - len(win)
    m = i - w + 1
    exp = [0, 0]
    routed = []
    if r // bsz > 0 and m > 0:
        F, lo = [], 0
        while lo < m:
            size = 1
            while lo % (2 * size) == 0 and lo + 2 * size <= m:
                size *= 2
            F.append((lo, lo + size))
            lo += size
        qq = q.astype(np.int64)

        def score(iv):
            s = int(K[iv[0]: iv[1]].astype(np.int64).sum(0) @ qq)
            return Fraction(s, iv[1] - iv[0]) if norm else s

        keep = r // bsz
        while True:
            if not any(hi - lo > bsz for lo, hi in F):
                if len(F) > keep:
                    F = sorted(F, key=lambda iv: (-score(iv), iv[0]))[:keep]
                break
            C = []
            for lo, hi in F:
                if hi - lo <= bsz:
                    C.append((lo, hi))
                    continue
                exp[0 if hi - lo >= 4 else 1] += 1
                mid = (lo + hi) // 2
                C += [(lo, mid), (mid, hi)]
            if len(C) > keep:
                C = sorted(C, key=lambda iv: (-score(iv), iv[0]))[:keep]
            F = C
        routed = [t for lo, hi in F for t in range(lo, hi)]
    return sorted(win + routed), tuple(exp)


@pytest.mark.parametrize("n,d", [(8, 2), (16, 4), (64, 64), (256, 8)])
def test_route_matches_independent_formulation(n, d):
    rng = _rng(n * 7 + d)
    for trial in range(60):
        # small value ranges make ties frequent, which exercises the tie rule
        lo, hi = (-16, 16) if trial % 2 else (-1, 1)
        K = _rand_qk(rng, (n, d), lo, hi)
        nodes = orc.build_tree(K)
        q = _rand_qk(rng, (d,), lo, hi)
        i = int(rng.integers(0, n))
        w = int(rng.integers(1, 6))
        B = int(rng.integers(1, n + 2))
        sel, exp = orc.route(K, nodes, q, i, B, w, 96)
        ref_sel, ref_exp = _alt_route(K, q, i, B, w, 96)
        assert sel.tolist() == ref_sel
        assert exp == ref_exp


@pytest.mark.parametrize("n,d", [(8, 2), (16, 4), (64, 8), (256, 8)])
@pytest.mark.parametrize("norm,bucket_log", [(True, 0), (False, 1), (False, 2), (True, 2),
                                             (True, 3)])
def test_descent_variants_match_independent_formulation(n, d, norm, bucket_log):
    rng = _rng(n * 13 + d + 101 * bucket_log + 7 * norm)
    for trial in range(40):
        lo, hi = (-16, 16) if trial % 2 else (-1, 1)
        K = _rand_qk(rng, (n, d), lo, hi)
        nodes = orc.build_tree(K)
        q = _rand_qk(rng, (d,), lo, hi)
        i = int(rng.integers(0, n))
        w = int(rng.integers(1, 6))
        B = int(rng.integers(1, n + 2))
        sel, exp = orc.route(K, nodes, q, i, B, w, 96, score_norm=norm, bucket_log=bucket_log)
        ref_sel, ref_exp = _alt_route(K, q, i, B, w, 96, norm=norm, bucket_log=bucket_log)
        assert sel.tolist() == ref_sel, (trial, i, w, B)
        assert exp == ref_exp


def test_variants_off_are_the_method():
    rng = _rng(5)
    n, d = 256, 8
    K = _rand_qk(rng, (n, d))
    nodes = orc.build_tree(K)
    for _ in range(50):
        q = _rand_qk(rng, (d,))
        i, B = int(rng.integers(0, n)), int(rng.integers(1, 97))
        a = orc.route(K, nodes, q, i, B, 16, 96)
        b = orc.route(K, nodes, q, i, B, 16, 96, score_norm=False, bucket_log=0)
        assert a[0].tolist() == b[0].tolist() and a[1] == b[1]


def test_mean_normalised_hand_example():
    """Worked by hand: keys 0..7 each score 1 against q, key 8 scores 3, window w = 1 at
    i = 9 (so the forest is [0, 8) and the key 8), one routed place (B = 2). Raw sums: [0, 8)
    (8) is expanded, its halves (4, 4) beat key 8 (3), and the descent ends on key 0 (ties go
    to the lower start). Means: the halves average 1, key 8 averages 3, so key 8 is kept."""
    d = 2
    K = np.zeros((16, d), dtype=np.int8)
    K[0:8] = [1, 0]
    K[8] = [3, 0]
    q = np.array([1, 0], dtype=np.int8)
    nodes = orc.build_tree(K)
    raw, _ = orc.route(K, nodes, q, 9, 2, 1, 96)
    mean, _ = orc.route(K, nodes, q, 9, 2, 1, 96, score_norm=True)
    assert raw.tolist() == [0, 9]
    assert mean.tolist() == [8, 9]


@pytest.mark.parametrize("n,w", [(64, 16), (256, 4)])
def test_mean_normalised_single_root_equals_raw(n, w):
    """When the past [0, i-w] is one aligned block, every frontier holds nodes of one level, so
    ranking by means and by sums is the same order: the two descents agree."""
    rng = _rng(n + w + 3)
    d = 8
    K = _rand_qk(rng, (n, d))
    nodes = orc.build_tree(K)
    for m in (1, 2, 4, 8, 16, 32):
        i = m + w - 1
        if i >= n:
            continue
        for _ in range(6):
            q = _rand_qk(rng, (d,))
            B = int(rng.integers(w + 1, w + 60))
            a = orc.route(K, nodes, q, i, B, w, 96)
            b = orc.route(K, nodes, q, i, B, w, 96, score_norm=True)
            assert a[0].tolist() == b[0].tolist() and a[1] == b[1]


@pytest.mark.parametrize("bucket_log", [1, 2, 4])
def test_buckets_wide_beam_route_the_whole_past(bucket_log):
    """When the past [0, m) is a whole number of buckets, a budget of every past key is a beam
    of exactly m >> bucket_log buckets: every key before the window is selected, and no node at
    or below the bucket level is expanded."""
    rng = _rng(bucket_log)
    n, d, w = 256, 4, 8
    K = _rand_qk(rng, (n, d))
    nodes = orc.build_tree(K)
    for t in (1, 3, 5, 10, 31):
        i = (t << bucket_log) + w - 1
        if i >= n:
            continue
        q = _rand_qk(rng, (d,))
        B = (n + 8) << bucket_log
        sel, _, lv = orc.route(K, nodes, q, i, B, w, B, by_level=True, bucket_log=bucket_log)
        assert sel.tolist() == list(range(i + 1))
        assert lv[: bucket_log + 1].sum() == 0


def test_bucket_hand_example():
    """Worked by hand: 16 past keys, buckets of 4, routed budget 8 -> 2 buckets. Key 9 alone
    scores 10, every other key 0, and the window is w = 1 at i = 16. Step 1 expands [0, 16)
    into [0, 8) (0) and [8, 16) (10); both stay. Step 2 expands them into four buckets scoring
    0, 0, 10, 0: [8, 12) first, then [0, 4) by the lower start. Selected: keys 0-3, 8-11, 16."""
    d = 2
    K = np.zeros((32, d), dtype=np.int8)
    K[9] = [5, 0]
    q = np.array([2, 1], dtype=np.int8)
    nodes = orc.build_tree(K)
    sel, exp = orc.route(K, nodes, q, 16, 9, 1, 96, bucket_log=2)
    assert sel.tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 16]
    assert exp == (3, 0)
    # a routed budget of 7 keys holds only one whole bucket
    sel, _ = orc.route(K, nodes, q, 16, 8, 1, 96, bucket_log=2)
    assert sel.tolist() == [8, 9, 10, 11, 16]
    # 3 routed keys hold no bucket: no beam, nothing expanded
    sel, exp = orc.route(K, nodes, q, 16, 4, 1, 96, bucket_log=2)
    assert sel.tolist() == [16] and exp == (0, 0)


def test_buckets_prune_roots_that_are_all_buckets():
    """i = 6, w = 1: the past [0, 6) is the forest [0, 4), [4, 6), both buckets of size <= 4.
    With one bucket allowed (budget 1 + 4), only the better root is kept, without expansion."""
    d = 1
    K = np.zeros((8, d), dtype=np.int8)
    K[5] = [3]
    q = np.array([1], dtype=np.int8)
    nodes = orc.build_tree(K)
    sel, exp = orc.route(K, nodes, q, 6, 5, 1, 96, bucket_log=2)
    assert sel.tolist() == [4, 5, 6]
    assert exp == (0, 0)


# ---------------------------------------------------------------- attention

def _dense_causal(Q, K, Vf, q_start):
    """Dense causal softmax attention in float64 (numpy), independent of the oracle."""
    nq, d = Q.shape
    S = Q.astype(np.float64) @ K.astype(np.float64).T / math.sqrt(d)
    pos = q_start + np.arange(nq)
    mask = np.arange(K.shape[0])[None, :] <= pos[:, None]
    S = np.where(mask, S, -np.inf)
    S = S - S.max(1, keepdims=True)
    P = np.exp(S)
    P /= P.sum(1, keepdims=True)
    return P @ Vf


@pytest.mark.parametrize("n,d,w", [(64, 8, 4), (256, 64, 16), (128, 128, 1)])
def test_full_budget_is_dense_causal_attention(n, d, w):
    rng = _rng(n + d + w)
    K = _rand_qk(rng, (n, d))
    Q = _rand_qk(rng, (n, d))
    V = _rand_v_bits(rng, (n, d))
    nodes = orc.build_tree(K)
    bud = np.full(n, n + 7, dtype=np.int32)
    res = orc.forward(Q, K, V, nodes, None, bud, q_start=0, window=w, max_keys=n)
    ref = _dense_causal(Q, K, _bits_to_f64(V), 0)
    assert np.abs(res["out"] - ref).max() <= 1e-12
    assert (res["count"] == np.arange(1, n + 1)).all()


def test_attention_closed_forms():
    rng = _rng(3)
    n, d = 32, 64
    K = _rand_qk(rng, (n, d))
    V = _rand_v_bits(rng, (n, d))
    Vf = _bits_to_f64(V)
    q = _rand_qk(rng, (d,))
    # one key: the output is that value row, exactly
    assert (orc.attend(q, K, V, np.array([9], dtype=np.int32)) == Vf[9]).all()
    # zero query: uniform weights -> mean of the selected rows
    sel = np.array([1, 4, 5, 30], dtype=np.int32)
    out = orc.attend(np.zeros(d, dtype=np.int8), K, V, sel)
    assert np.abs(out - Vf[sel].mean(0)).max() < 1e-15
    # two keys with a known score gap: weights 1/(1+e^-g) and e^-g/(1+e^-g)
    K2 = np.zeros((2, d), dtype=np.int8)
    K2[0, 0] = 8
    q2 = np.zeros(d, dtype=np.int8)
    q2[0] = 2  # score gap 16 / sqrt(64) = 2
    V2 = _rand_v_bits(rng, (2, d))
    out = orc.attend(q2, K2, V2, np.array([0, 1], dtype=np.int32))
    a = 1.0 / (1.0 + math.exp(-2.0))
    ref = a * _bits_to_f64(V2)[0] + (1 - a) * _bits_to_f64(V2)[1]
    assert np.abs(out - ref).max() < 1e-14
    # empty selection gives zeros
    assert (orc.attend(q, K, V, np.zeros(0, dtype=np.int32)) == 0).all()


def test_forward_budget_override_clamp_and_predictor():
    rng = _rng(21)
    n, d = 128, 64
    K = _rand_qk(rng, (n, d))
    Q = _rand_qk(rng, (n, d))
    V = _rand_v_bits(rng, (n, d))
    W = rng.integers(-4, 5, size=(32, 2 * d)).astype(np.int8)
    nodes = orc.build_tree(K)
    res = orc.forward(Q, K, V, nodes, W, None, q_start=0, window=16, max_keys=96)
    for i in [0, 5, 16, 17, 100, 127]:
        c, _ = orc.predict(Q[i], orc.causal_sum(K, i), W)
        assert res["budget"][i] == 3 * (c + 1)
        sel, exp = orc.route(K, nodes, Q[i], i, 3 * (c + 1), 16, 96)
        assert res["idx"][i, : res["count"][i]].tolist() == sel.tolist()
        assert tuple(res["expansions"][i]) == exp
        assert np.array_equal(res["out"][i], orc.attend(Q[i], K, V, sel))
    bud = np.array([0, -5] + [3] * (n - 2), dtype=np.int32)
    res = orc.forward(Q, K, V, nodes, None, bud, q_start=0, window=16, max_keys=96,
                      rows=np.array([0, 1, 2], dtype=np.int32))
    assert res["budget"][:3].tolist() == [1, 1, 3]
    assert res["count"][:3].tolist() == [1, 1, 3]


def test_expansions_by_level_add_up(golden_n8):
    """The per-level histogram sums to the two counters; the wide-beam case expands every
    internal node of the forest once, so level l holds the forest's level-l nodes."""
    K = np.array(golden_n8["K"], dtype=np.int8)
    nodes = orc.build_tree(K)
    for case in golden_n8["routes"]:
        sel, exp, lv = orc.route(K, nodes, np.array(case["q"], dtype=np.int8), case["i"],
                                 case["budget"], golden_n8["window"], 96, by_level=True)
        assert lv[0] == 0 and lv[2:].sum() == exp[0] and lv[1] == exp[1]
    rng = _rng(77)
    n, d, w = 256, 8, 5
    K = _rand_qk(rng, (n, d))
    nodes = orc.build_tree(K)
    for i in [200, 255, 77]:
        _, _, lv = orc.route(K, nodes, _rand_qk(rng, (d,)), i, n, w, n, by_level=True)
        m = i - w + 1
        expect = np.zeros(32, dtype=np.int64)
        for b in range(1, 20):
            if (m >> b) & 1:
                for l in range(1, b + 1):
                    expect[l] += 1 << (b - l)
        assert lv.tolist() == expect.tolist()


# ---------------------------------------------------------------- phase-2 labels (top-k)


def _labels_numpy(Q, K, q_start, k):
    """Independent formulation: the full causal score matrix with numpy, then per row a stable
    argsort of the negated scores (stable = equal scores keep ascending positions)."""
    S = Q.astype(np.int64) @ K.astype(np.int64).T
    nq = Q.shape[0]
    lab = np.full((nq, k), -1, dtype=np.int32)
    sc = np.zeros((nq, k), dtype=np.int32)
    for r in range(nq):
        i = q_start + r
        row = S[r, : i + 1]
        order = np.argsort(-row, kind="stable")[:k]
        lab[r, : len(order)] = order
        sc[r, : len(order)] = row[order]
    return lab, sc


@pytest.mark.parametrize("n,d,q_start,k", [(64, 8, 0, 16), (256, 64, 0, 16), (512, 16, 300, 16),
                                           (128, 128, 5, 4), (32, 4, 0, 32)])
def test_labels_match_numpy(n, d, q_start, k):
    rng = _rng(n + d + q_start + k)
    for lo, hi in ((-16, 16), (-1, 1)):  # the narrow range makes ties everywhere
        K = _rand_qk(rng, (n, d), lo, hi)
        Q = _rand_qk(rng, (n - q_start, d), lo, hi)
        lab, sc = orc.topk_labels(Q, K, q_start, k)
        ref_lab, ref_sc = _labels_numpy(Q, K, q_start, k)
        assert np.array_equal(lab, ref_lab) and np.array_equal(sc, ref_sc)


def test_labels_planted_keys_and_short_rows():
    """K is zero except 16 planted keys that score 1..16 against q: every row at or after the
    last planted key lists them from the best down; a row before it lists the planted keys
    already seen, then zero-score keys by position; rows with fewer than k keys are padded."""
    n, d = 256, 4
    q = np.array([1, 0, 0, 0], dtype=np.int8)
    K = np.zeros((n, d), dtype=np.int8)
    pos = np.array([3, 9, 17, 30, 31, 44, 60, 61, 77, 90, 101, 120, 140, 141, 150, 199])
    for v, p in enumerate(pos, start=1):
        K[p, 0] = v
    Q = np.tile(q, (n, 1))
    lab, sc = orc.topk_labels(Q, K, 0, 16)
    assert lab[255].tolist() == pos[::-1].tolist()
    assert sc[255].tolist() == list(range(16, 0, -1))
    seen = pos[pos <= 50][::-1].tolist()                       # 3, 9, 17, 30, 31, 44
    zeros = [t for t in range(51) if t not in pos][: 16 - len(seen)]
    assert lab[50].tolist() == seen + zeros
    assert lab[2].tolist() == [0, 1, 2] + [-1] * 13 and sc[2].tolist() == [0] * 16


def test_labels_top1_is_causal_argmax():
    rng = _rng(17)
    n, d = 300, 16
    K = _rand_qk(rng, (n, d))
    Q = _rand_qk(rng, (n, d))
    lab, sc = orc.topk_labels(Q, K, 0, 1)
    for i in range(n):
        s = K[: i + 1].astype(np.int64) @ Q[i].astype(np.int64)
        assert lab[i, 0] == int(np.argmax(s)) and sc[i, 0] == s.max()
