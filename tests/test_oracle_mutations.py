"""Planted mistakes: each test compiles a copy of the oracle with one plausible slip and checks
that the pins in test_oracle_pins.py reject it. The mistakes are planted in the oracle, on the
CPU; nothing here touches a GPU."""
import json
import os
import subprocess
import sys
import tempfile

import pytest

from oracle import oracle as orc
import test_oracle_pins as pins

_SRC = os.path.join(os.path.dirname(orc.__file__), "alhr_oracle.cpp")

MUTATIONS = {
    "tie_to_higher_start": ("return a.start < b.start;", "return a.start > b.start;"),
    "keep_lowest_scores": ("    return a.score > b.score;", "    return a.score < b.score;"),
    "window_one_too_wide": ("t > int64_t(i) - w &&", "t >= int64_t(i) - w &&"),
    "forest_covers_window_key": ("const int64_t m = int64_t(i) - w + 1;",
                                 "const int64_t m = int64_t(i) - w + 2;"),
    "forest_misses_a_key": ("const int64_t m = int64_t(i) - w + 1;",
                            "const int64_t m = int64_t(i) - w;"),
    "right_child_offset": ("right = nd.start + (int64_t(1) << cl);",
                           "right = nd.start + (int64_t(1) << nd.level);"),
    "level_offset_shifted": ("return n - (n >> (level - 1));", "return n - (n >> level);"),
    "exclusive_causal_sum": ("for (int u = 0; u <= i; ++u)", "for (int u = 0; u < i; ++u)"),
    "predictor_tie_to_higher_class": ("if (c == 0 || s > best_logit)",
                                      "if (c == 0 || s >= best_logit)"),
    "predictor_operands_swapped": ("s += int64_t(w[d + t]) * G[t];",
                                   "s += int64_t(w[t]) * G[t];"),
    "expansion_levels_misfiled": ("if (nd.level >= 2) ++exp_hi; else ++exp_l1;",
                                  "if (nd.level >= 1) ++exp_hi; else ++exp_l1;"),
    "no_score_scale": ("s[size_t(k)] = double(dot) * scale;",
                       "s[size_t(k)] = double(dot);"),
    "softmax_without_max_shift_sign": ("std::exp(s[size_t(k)] - mx)",
                                       "std::exp(mx - s[size_t(k)])"),
    "budget_not_clamped": ("budget = std::max(budget_override[row], 1);",
                           "budget = budget_override[row];"),
    "prune_keeps_one_less": ("cand.resize(size_t(keep));", "cand.resize(size_t(keep - 1));"),
    "mean_scaled_by_own_level": ("static_cast<__int128>(a.score) * (static_cast<__int128>(1) << b.level)",
                                 "static_cast<__int128>(a.score) * (static_cast<__int128>(1) << a.level)"),
    "mean_ignored": ("if (norm) {", "if (false) {"),
    "bucket_beam_in_keys": ("const int64_t keep = r >> bucket_log;", "const int64_t keep = r;"),
    "bucket_level_expanded": ("if (nd.level <= bucket_log) {", "if (nd.level < bucket_log) {"),
    "bucket_last_key_dropped": ("t < nd.start + (int64_t(1) << nd.level); ++t)",
                                "t + 1 < nd.start + (int64_t(1) << nd.level); ++t)"),
    "bucket_roots_not_pruned": ("if (int64_t(frontier.size()) > keep) {", "if (false) {"),
    "labels_exclude_own_key": ("for (int64_t t = 0; t <= i; ++t) {", "for (int64_t t = 0; t < i; ++t) {"),
    "labels_ties_to_higher_position": ("      return a.second < b.second;", "      return a.second > b.second;"),
    "labels_lowest_scores": ("      if (a.first != b.first) return a.first > b.first;",
                             "      if (a.first != b.first) return a.first < b.first;"),
    "window_cut_far_first": (
        "for (int64_t t = i; t >= 0 && t > int64_t(i) - w && int64_t(chosen.size()) < b_eff; --t)",
        "for (int64_t t = std::max<int64_t>(0, int64_t(i) - w + 1); "
        "t <= int64_t(i) && int64_t(chosen.size()) < b_eff; ++t)"),
    "roots_smallest_first": ("for (int b = 62; b >= 0; --b) {", "for (int b = 0; b <= 62; ++b) {"),
    "level_one_nodes_not_expanded": ("any_inner |= (nd.level > bucket_log);",
                                     "any_inner |= (nd.level > bucket_log + 1);"),
    "budget_classes_off_by_one": ("budget = 3 * (oracle_predict(d, q, G.data(), W, nullptr) + 1);",
                                  "budget = 3 * oracle_predict(d, q, G.data(), W, nullptr) + 1;"),
    "causal_sum_without_window": ("for (int u = 0; u <= i; ++u) s += K[int64_t(u) * d + t];",
                                  "for (int u = 0; u <= i - 16; ++u) s += K[int64_t(u) * d + t];"),
    "window_without_own_key": (
        "for (int64_t t = i; t >= 0 && t > int64_t(i) - w && int64_t(chosen.size()) < b_eff; --t)",
        "for (int64_t t = i - 1; t >= 0 && t >= int64_t(i) - w && int64_t(chosen.size()) < b_eff; --t)"),
    "value_row_of_the_previous_key": ("const uint16_t* v = V + int64_t(sel[k]) * d;",
                                  "const uint16_t* v = V + int64_t(sel[k] == 0 ? 0 : sel[k] - 1) * d;"),
    "roots_pruned_before_first_expansion": (
        "    const bool norm = score_norm != 0;\n",
        "    const bool norm = score_norm != 0;\n"
        "    if (int64_t(frontier.size()) > keep) {\n"
        "      std::sort(frontier.begin(), frontier.end(),\n"
        "                [norm](const Node& a, const Node& b) { return ranks_before(a, b, norm); });\n"
        "      frontier.resize(size_t(keep));\n"
        "    }\n"),
}

PIN_TESTS = [
    ("golden_tree", lambda g: pins.test_golden_tree(g)),
    ("golden_causal", lambda g: pins.test_golden_causal_sums(g)),
    ("golden_routes", lambda g: pins.test_golden_routes(g)),
    ("roots_not_pruned_first", lambda g: pins.test_roots_not_pruned_before_the_first_expansion(g)),
    ("golden_predictor", lambda g: pins.test_golden_predictor(g)),
    ("golden_forward", lambda g: pins.test_golden_forward_composition(g)),
    ("root_children", lambda g: pins.test_tree_root_and_children(64, 64)),
    ("telescoping", lambda g: pins.test_causal_sum_telescopes_and_ends_at_root()),
    ("numpy_argmax", lambda g: pins.test_predictor_against_numpy_argmax()),
    ("ties_lowest_class", lambda g: pins.test_predictor_ties_go_to_lowest_class()),
    ("wide_beam", lambda g: pins.test_wide_beam_routes_the_whole_past(256, 5)),
    ("planted", lambda g: pins.test_planted_positive_key_is_routed(512, 16)),
    ("dense", lambda g: pins.test_full_budget_is_dense_causal_attention(64, 8, 4)),
    ("attention_closed_forms", lambda g: pins.test_attention_closed_forms()),
    ("clamp", lambda g: pins.test_forward_budget_override_clamp_and_predictor()),
    ("mean_hand", lambda g: pins.test_mean_normalised_hand_example()),
    ("mean_single_root", lambda g: pins.test_mean_normalised_single_root_equals_raw(64, 16)),
    ("bucket_wide", lambda g: pins.test_buckets_wide_beam_route_the_whole_past(2)),
    ("bucket_hand", lambda g: pins.test_bucket_hand_example()),
    ("bucket_roots", lambda g: pins.test_buckets_prune_roots_that_are_all_buckets()),
    ("labels_numpy", lambda g: pins.test_labels_match_numpy(64, 8, 0, 16)),
    ("labels_planted", lambda g: pins.test_labels_planted_keys_and_short_rows()),
    ("labels_argmax", lambda g: pins.test_labels_top1_is_causal_argmax()),
]


def _compile_mutant(name, tmpdir):
    old, new = MUTATIONS[name]
    with open(_SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor for {name} must occur exactly once"
    path = os.path.join(tmpdir, f"{name}.cpp")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    so = os.path.join(tmpdir, f"lib{name}.so")
    subprocess.run(["g++", "-O1", "-std=c++17", "-shared", "-fPIC", "-o", so, path], check=True)
    return so


def run_pins_against(so_path: str) -> list:
    """Names of the pins that reject the oracle build at so_path."""
    import json as _json
    from conftest import ROOT
    with open(os.path.join(ROOT, "tests", "golden", "alhr_n8_d2.json")) as f:
        golden = _json.load(f)
    caught = []
    with orc.use_library(so_path):
        for pin, fn in PIN_TESTS:
            try:
                fn(golden)
            except (AssertionError, OverflowError):
                caught.append(pin)
    return caught


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    # each mutant runs in a child process: a slip that writes out of bounds may crash it,
    # which also counts as caught
    here = os.path.dirname(os.path.abspath(__file__))
    with tempfile.TemporaryDirectory() as tmp:
        so = _compile_mutant(name, tmp)
        code = ("import sys, json; sys.path[:0] = [%r, %r]; "
                "import test_oracle_mutations as m; print(json.dumps(m.run_pins_against(%r)))"
                % (here, os.path.dirname(here), so))
        proc = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True,
                              timeout=600)
        if proc.returncode != 0:
            return  # the mutant crashed the pins: caught
        caught = json.loads(proc.stdout.strip().splitlines()[-1])
        assert caught, f"no pin rejects the planted mistake {name}"


def test_unmutated_oracle_passes_every_pin(golden_n8):
    for _, fn in PIN_TESTS:
        fn(golden_n8)
