// alhr_oracle.cpp -- plain, single-threaded reference of the ALHR inference path.
//
// TEST INFRASTRUCTURE ONLY. This file is the oracle that the CUDA path is checked against.
// Only the test suite, the smoke check and the benchmark's CPU-baseline arm may load it; the
// library itself never calls it and shares no code with it.
//
// Every step restates the method as the ALHR project README ("ALHR (Adaptive learnable
// Hierarchical routing): sub-quadratic tree attention without meaningful accuracy loss,
// trained in three phases against a dense reference") describes it, in the order of its
// "Inference stage" section, with the numeric formats the library fixes (int8 Q/K, bf16 V).
// Integers are accumulated in int64 and attention runs in double precision. Nothing is
// blocked, fused or reordered beyond the definitions:
//   * tree sums are computed straight from their definition (a sum over each node's range),
//   * the causal key sum is a direct sum over the past keys,
//   * every candidate's routing score is a direct dot product with its stored sum row,
//   * pruning is a full sort of the candidates.
//
// Readings of points the README leaves open (each one is listed in the design notes):
//   R1  the predictor's sum over all key vectors is read causally: G_i = sum of keys 0..i.
//   R2  the budget predictor is linear: logits = W [q ; G_i], 32 classes, ties -> lower class,
//       class c asks for 3*(c+1) keys (32 classes, at most 96 keys, as in §Results and Variables).
//   R3  the budget counts the whole selection: the own key and the window keys come first
//       (nearest first) and the descent only fills what is left (the neighbour keys found are
//       taken off the predicted count, §Inference stage, fourth paragraph).
//   R4  the window is the own key plus the w-1 keys before it; when the budget is smaller
//       than the window, it is cut nearest first.
//   R5  causality (§Training stage, last paragraph) is the forest of maximal aligned
//       power-of-two blocks covering the keys before the window, [0, i-w], largest first.
//   R6  descent: every step expands all non-leaf frontier nodes into their two children and
//       then keeps the r best by exact integer q . node_sum (raw sums, not means), ties to
//       the lower start position; it ends when the frontier holds only keys. The number of
//       branches followed equals the keys still needed (§Inference stage, fourth paragraph).
//   R7  the reuse of what earlier queries found among their own neighbours (§Inference stage,
//       third paragraph) is read as a cache that changes no selected set; ignored.
//   R8  attention is softmax(q . k / sqrt(d)) . V over the selected keys, no temperature.
//   R11 phase-2 labels: the top-k keys of a query's causal attention row are its k largest
//       q . k, equal scores to the lower position (softmax keeps the order of the scores).
// Two descent variants (off by default; both off is the method above):
//   R9  mean-normalised scores: candidates are ranked by q . node_sum / 2^level, the mean of
//       the keys beneath them (what block-sparse methods rank blocks by; page "ALHR把注意力
//       变成树搜索", §"它和块稀疏、线性注意力有什么区别"). Compared exactly, as fractions with
//       power-of-two denominators; equal means go to the lower start.
//   R10 leaf buckets of 2^b keys (page "ALHR把注意力变成树搜索", §"次二次复杂度成立，需要满足三个
//       前提": the leaf bucket size must not grow with the sequence): a node of level <= b is
//       a bucket and is not expanded; the beam keeps r >> b nodes (the routed key budget r
//       counted in whole buckets, so at most r keys); the descent ends when the frontier holds
//       only buckets, and every key of every kept bucket is selected; when r >> b is 0 there is
//       no beam and no descent. b = 0 is the method above.
//       The frontier is pruned after every expansion step and also when the forest's roots are
//       all buckets already.

#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <utility>
#include <vector>

namespace {

// Row offset of tree level l (1 <= l <= log2 n) in the level-major layout: level 1 first
// (n/2 rows), then level 2 (n/4 rows), ..., the root last.
int64_t level_offset(int64_t n, int level) { return n - (n >> (level - 1)); }

int log2_exact(int64_t n) {
  int l = 0;
  while ((int64_t(1) << l) < n) ++l;
  return l;
}

struct Node {
  int level;      // 0 = a single key
  int64_t start;  // first key position covered; the node covers [start, start + 2^level)
  int64_t score;  // q . node_sum
};

// Candidate order: the larger score first (raw sums, or under R9 the larger mean
// score / 2^level, compared as a.score * 2^b.level against b.score * 2^a.level), then the
// lower start.
bool ranks_before(const Node& a, const Node& b, bool norm) {
  if (norm) {
    const __int128 x = static_cast<__int128>(a.score) * (static_cast<__int128>(1) << b.level);
    const __int128 y = static_cast<__int128>(b.score) * (static_cast<__int128>(1) << a.level);
    if (x != y) return x > y;
  } else if (a.score != b.score) {
    return a.score > b.score;
  }
  return a.start < b.start;
}

// The stored sum row of a node: K itself at level 0, the tree above.
int64_t node_score(int n, int d, const int8_t* K, const int32_t* nodes, const int8_t* q,
                   int level, int64_t start) {
  int64_t s = 0;
  if (level == 0) {
    const int8_t* row = K + start * d;
    for (int t = 0; t < d; ++t) s += int64_t(q[t]) * int64_t(row[t]);
  } else {
    const int32_t* row = nodes + (level_offset(n, level) + (start >> level)) * int64_t(d);
    for (int t = 0; t < d; ++t) s += int64_t(q[t]) * int64_t(row[t]);
  }
  return s;
}

double bf16_to_double(uint16_t bits) {
  uint32_t u = uint32_t(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return double(f);
}

}  // namespace

extern "C" {

// Tree over one (b,h) block of keys [README opening paragraph: each branch is indexed by the
// sum of all the key vectors beneath it; §Inference stage, first paragraph: built once on the
// key matrix and stored]. node(l, j) = sum over t in [j 2^l, (j+1) 2^l) of K[t], l = 1..log2 n.
// Returns 0, or 1 when a sum does not fit in int32 (nothing is clipped; the value is stored
// truncated and the caller must treat the tree as invalid).
int oracle_build_tree(int n, int d, const int8_t* K, int32_t* nodes) {
  const int L = log2_exact(n);
  int bad = 0;
  for (int l = 1; l <= L; ++l) {
    const int64_t rows = int64_t(n) >> l;
    for (int64_t j = 0; j < rows; ++j) {
      for (int t = 0; t < d; ++t) {
        int64_t s = 0;
        for (int64_t u = j << l; u < (j + 1) << l; ++u) s += K[u * d + t];
        if (s > INT32_MAX || s < INT32_MIN) bad = 1;
        nodes[(level_offset(n, l) + j) * d + t] = int32_t(s);
      }
    }
  }
  return bad;
}

// Causal global key sum, reading R1: G[t] = sum_{u <= i} K[u][t].
void oracle_causal_sum(int d, const int8_t* K, int i, int64_t* G) {
  for (int t = 0; t < d; ++t) {
    int64_t s = 0;
    for (int u = 0; u <= i; ++u) s += K[int64_t(u) * d + t];
    G[t] = s;
  }
}

// Budget predictor, reading R2 [README §Inference stage, second paragraph; §Results and
// Variables: 32 budget classes]. logits[c] = sum_t W[c][t] q[t] + sum_t W[c][d+t] G[t].
// Returns the class c* (smallest c among the largest logits); the budget is 3 (c* + 1).
int oracle_predict(int d, const int8_t* q, const int64_t* G, const int8_t* W, int64_t* logits) {
  int best = 0;
  int64_t best_logit = 0;
  for (int c = 0; c < 32; ++c) {
    const int8_t* w = W + int64_t(c) * 2 * d;
    int64_t s = 0;
    for (int t = 0; t < d; ++t) s += int64_t(w[t]) * int64_t(q[t]);
    for (int t = 0; t < d; ++t) s += int64_t(w[d + t]) * G[t];
    if (logits) logits[c] = s;
    if (c == 0 || s > best_logit) {
      best = c;
      best_logit = s;
    }
  }
  return best;
}

// Neighbour search and budget-limited descent for the query q at position i with budget B,
// readings R3..R7 [README §Inference stage, third and fourth paragraphs; §Training stage, last
// paragraph]. Writes the selection ascending into sel (room for min(B, i+1, max_keys) entries),
// {nodes of level >= 2 expanded, level-1 nodes expanded} into expansions (nullable) and the
// number of expanded nodes of each level l into by_level[l], l < 32 (nullable).
// Returns the selection size min(B_eff, i+1) with B_eff = min(max(B,1), i+1, max_keys).
// score_norm selects R9, bucket_log the bucket size 2^bucket_log of R10 (0: single keys).
int oracle_route(int n, int d, const int8_t* K, const int32_t* nodes, const int8_t* q, int i,
                 int budget, int w, int max_keys, int score_norm, int bucket_log, int32_t* sel,
                 int32_t* expansions, int32_t* by_level) {
  if (by_level)
    for (int l = 0; l < 32; ++l) by_level[l] = 0;
  int64_t b_eff = std::max(budget, 1);
  b_eff = std::min<int64_t>(b_eff, int64_t(i) + 1);
  b_eff = std::min<int64_t>(b_eff, max_keys);

  std::vector<int64_t> chosen;
  // own key first, then the neighbours before it, nearest first (R3, R4)
  for (int64_t t = i; t >= 0 && t > int64_t(i) - w && int64_t(chosen.size()) < b_eff; --t)
    chosen.push_back(t);

  int64_t exp_hi = 0, exp_l1 = 0;
  const int64_t r = b_eff - int64_t(chosen.size());
  const int64_t m = int64_t(i) - w + 1;  // keys strictly before the window: [0, m)
  const int64_t keep = r >> bucket_log;  // the beam: r keys, or r >> b whole buckets (R10)
  if (keep > 0 && m > 0) {
    // R5: the maximal aligned power-of-two blocks of [0, m), largest first
    std::vector<Node> frontier;
    int64_t s = 0;
    for (int b = 62; b >= 0; --b) {
      if ((m >> b) & 1) {
        frontier.push_back({b, s, node_score(n, d, K, nodes, q, b, s)});
        s += int64_t(1) << b;
      }
    }
    // R6: expand every non-leaf, then keep the r best, until only keys remain (R10: leaves
    // are the buckets, nodes of level <= bucket_log, and the beam keeps r >> bucket_log)
    const bool norm = score_norm != 0;
    for (;;) {
      bool any_inner = false;
      for (const Node& nd : frontier) any_inner |= (nd.level > bucket_log);
      if (!any_inner) {
        if (int64_t(frontier.size()) > keep) {  // roots that are all buckets (R10)
          std::sort(frontier.begin(), frontier.end(),
                    [norm](const Node& a, const Node& b) { return ranks_before(a, b, norm); });
          frontier.resize(size_t(keep));
        }
        break;
      }
      std::vector<Node> cand;
      for (const Node& nd : frontier) {
        if (nd.level <= bucket_log) {
          cand.push_back(nd);
          continue;
        }
        if (nd.level >= 2) ++exp_hi; else ++exp_l1;
        if (by_level) ++by_level[nd.level];
        const int cl = nd.level - 1;
        const int64_t left = nd.start, right = nd.start + (int64_t(1) << cl);
        cand.push_back({cl, left, node_score(n, d, K, nodes, q, cl, left)});
        cand.push_back({cl, right, node_score(n, d, K, nodes, q, cl, right)});
      }
      if (int64_t(cand.size()) > keep) {
        std::sort(cand.begin(), cand.end(),
                  [norm](const Node& a, const Node& b) { return ranks_before(a, b, norm); });
        cand.resize(size_t(keep));
      }
      frontier.swap(cand);
    }
    for (const Node& nd : frontier)
      for (int64_t t = nd.start; t < nd.start + (int64_t(1) << nd.level); ++t) chosen.push_back(t);
  }
  std::sort(chosen.begin(), chosen.end());
  for (size_t k = 0; k < chosen.size(); ++k) sel[k] = int32_t(chosen[k]);
  if (expansions) {
    expansions[0] = int32_t(exp_hi);
    expansions[1] = int32_t(exp_l1);
  }
  return int(chosen.size());
}

// Exact attention over the selected keys, reading R8 [README §Inference stage, fifth
// paragraph]: out = sum_j e^{s_j - m} V[j] / sum_j e^{s_j - m}, s_j = (q . K[j]) / sqrt(d),
// m = max_j s_j, all in double; V converted from bf16 exactly. count <= 0 gives zeros.
void oracle_attend(int d, const int8_t* q, const int8_t* K, const uint16_t* V,
                   const int32_t* sel, int count, double* out) {
  for (int t = 0; t < d; ++t) out[t] = 0.0;
  if (count <= 0) return;
  const double scale = 1.0 / std::sqrt(double(d));
  std::vector<double> s(static_cast<size_t>(count));
  double mx = -INFINITY;
  for (int k = 0; k < count; ++k) {
    int64_t dot = 0;
    const int8_t* row = K + int64_t(sel[k]) * d;
    for (int t = 0; t < d; ++t) dot += int64_t(q[t]) * int64_t(row[t]);
    s[size_t(k)] = double(dot) * scale;
    mx = std::max(mx, s[size_t(k)]);
  }
  double den = 0.0;
  for (int k = 0; k < count; ++k) {
    const double p = std::exp(s[size_t(k)] - mx);
    den += p;
    const uint16_t* v = V + int64_t(sel[k]) * d;
    for (int t = 0; t < d; ++t) out[t] += p * bf16_to_double(v[t]);
  }
  for (int t = 0; t < d; ++t) out[t] /= den;
}

// The whole path for a set of queries of one (b,h) block, in the README's order: causal sum
// and budget predictor (or the given budget), neighbour search and descent (with the R9 / R10
// variants as oracle_route), attention.
//   Q [nq][d], K [n][d], V [n][d], nodes [n-1][d] (this oracle's own tree), W [32][2d] or NULL,
//   budget_override [nq] or NULL, rows: the query rows to compute (NULL = all nq rows).
// Outputs (rows not listed are left untouched): out [nq][d], idx [nq][max_keys] (-1 padded),
// count [nq], expansions [nq][2], budget_out [nq] (the budget used, after the clamp to >= 1),
// by_level [nq][32] or NULL (expanded nodes per level).
void oracle_forward(int n, int d, int q_start, int nq, int w, int max_keys, int score_norm,
                    int bucket_log, const int8_t* Q,
                    const int8_t* K, const uint16_t* V, const int32_t* nodes, const int8_t* W,
                    const int32_t* budget_override, const int32_t* rows, int n_rows,
                    double* out, int32_t* idx, int32_t* count, int32_t* expansions,
                    int32_t* budget_out, int32_t* by_level) {
  std::vector<int64_t> G(static_cast<size_t>(d));
  std::vector<int32_t> sel(static_cast<size_t>(std::max(max_keys, 1)));
  const int total = rows ? n_rows : nq;
  for (int k = 0; k < total; ++k) {
    const int row = rows ? rows[k] : k;
    const int i = q_start + row;
    const int8_t* q = Q + int64_t(row) * d;
    int budget;
    if (budget_override) {
      budget = std::max(budget_override[row], 1);
    } else {
      oracle_causal_sum(d, K, i, G.data());
      budget = 3 * (oracle_predict(d, q, G.data(), W, nullptr) + 1);
    }
    const int c = oracle_route(n, d, K, nodes, q, i, budget, w, max_keys, score_norm,
                               bucket_log, sel.data(),
                               expansions + int64_t(row) * 2,
                               by_level ? by_level + int64_t(row) * 32 : nullptr);
    oracle_attend(d, q, K, V, sel.data(), c, out + int64_t(row) * d);
    for (int s = 0; s < max_keys; ++s) idx[int64_t(row) * max_keys + s] = s < c ? sel[size_t(s)] : -1;
    count[row] = c;
    budget_out[row] = budget;
  }
}

// Phase-2 labels [README §Training stage, Phase 2: the dense model's attention matrix gives the
// top-k keys of every query; §Results and Variables: k = 16]. Softmax is monotonic in the score,
// so the top-k of an attention row are the k largest q . K[t] over the causal keys t <= i, taken
// here as exact integers; equal scores go to the lower key position (R11). Writes, per query
// row, labels[row][0..k) (positions, best first, -1 when fewer than k keys exist) and
// scores[row][0..k) (the dot products, 0 in padded slots; scores may be NULL).
void oracle_topk_labels(int n, int d, const int8_t* Q, const int8_t* K, int q_start, int nq,
                        int k, int32_t* labels, int32_t* scores) {
  (void)n;
  std::vector<std::pair<int64_t, int64_t>> row;  // (score, position)
  for (int r = 0; r < nq; ++r) {
    const int i = q_start + r;
    const int8_t* q = Q + int64_t(r) * d;
    row.clear();
    for (int64_t t = 0; t <= i; ++t) {
      int64_t s = 0;
      for (int u = 0; u < d; ++u) s += int64_t(q[u]) * int64_t(K[t * d + u]);
      row.push_back({s, t});
    }
    std::sort(row.begin(), row.end(), [](const std::pair<int64_t, int64_t>& a,
                                         const std::pair<int64_t, int64_t>& b) {
      if (a.first != b.first) return a.first > b.first;
      return a.second < b.second;
    });
    for (int j = 0; j < k; ++j) {
      const bool ok = size_t(j) < row.size();
      labels[int64_t(r) * k + j] = ok ? int32_t(row[size_t(j)].second) : -1;
      if (scores) scores[int64_t(r) * k + j] = ok ? int32_t(row[size_t(j)].first) : 0;
    }
  }
}

// Timing harness of the CPU baseline (no arithmetic of its own): the wall time, measured with
// std::chrono::steady_clock on the calling thread, of oracle_build_tree on one block followed by
// oracle_forward over the listed query rows of that block (rows NULL: all nq rows). Outputs as
// oracle_forward; nodes is scratch of [n-1][d] int32. Returns seconds, or -1.0 when a tree sum
// leaves int32.
double oracle_time_block(int n, int d, int q_start, int nq, int w, int max_keys,
                         const int8_t* Q, const int8_t* K, const uint16_t* V, const int8_t* W,
                         const int32_t* budget_override, const int32_t* rows, int n_rows,
                         int32_t* nodes, double* out, int32_t* idx, int32_t* count,
                         int32_t* expansions, int32_t* budget_out) {
  const auto t0 = std::chrono::steady_clock::now();
  if (oracle_build_tree(n, d, K, nodes) != 0) return -1.0;
  oracle_forward(n, d, q_start, nq, w, max_keys, 0, 0, Q, K, V, nodes, W, budget_override, rows,
                 n_rows, out, idx, count, expansions, budget_out, nullptr);
  const auto t1 = std::chrono::steady_clock::now();
  return std::chrono::duration<double>(t1 - t0).count();
}

}  // extern "C"

