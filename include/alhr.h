/*
 * alhr.h -- C ABI of the B200 (sm_100a) inference path of ALHR tree attention.
 *
 * Source of the method: the project README "ALHR (Adaptive learnable Hierarchical
 * routing): sub-quadratic tree attention without meaningful accuracy loss, trained in
 * three phases against a dense reference" (GitHub project
 * Adaptive-Learnable-Hierarchical-Routing-), cited below as [README §<section>], and the
 * openai-hub analysis "ALHR把注意力变成树搜索", cited as [openai-hub §<section>].
 *
 * Problem statement fixed for this library (the README leaves the numeric formats open):
 *   - per (batch b, head h) there are n keys, n a power of two, head dimension d in {64,128};
 *   - Q and K are int8 with |value| <= value_bound (16 unless stated), so every tree sum and
 *     every routing score is an exact integer;
 *   - V is bf16 (passed as raw uint16 bit patterns); outputs are fp32;
 *   - budgets come from 32 classes, class c meaning 3*(c+1) keys, at most 96 keys
 *     [README §Results and Variables: the caps are 96 keys and 32 budget classes];
 *   - the neighbour window is w keys (16 in the README's setting).
 *
 * Memory layouts (all row-major, contiguous, device memory, 16-byte aligned base pointers; the
 * tree 32-byte aligned, since its rows are read 32 bytes at a time — cudaMalloc and torch
 * allocations are 256-byte aligned):
 *   Q      int8     [batch][heads][nq][d]        row t is the query at position q_start+t
 *   K      int8     [batch][heads][n][d]
 *   V      uint16   [batch][heads][n][d]         bf16 bit patterns
 *   tree   bytes    [batch][heads][alhr_tree_bytes(n, d, value_bound)]  the key tree, see below
 *   W      int8     [32][2d]                     budget-predictor weights, shared by all heads
 *   budget int32    [batch][heads][nq]           keys asked for by each query (>= 1)
 *   idx    int32    [batch][heads][nq][max_keys] selected key positions, ascending, -1 padded
 *   count  int32    [batch][heads][nq]           number of valid entries of idx
 *   expansions int32 [batch][heads][nq][3]       {nodes of level >= 2 expanded, level-1 nodes
 *                                                 expanded, expanded nodes whose children are
 *                                                 32-bit tree rows (level >= wide_level + 1)}
 *   out    float    [batch][heads][nq][d]
 *
 * Tree layout (one block of alhr_tree_bytes(n, d, value_bound) bytes per (b,h), blocks
 * consecutive): levels 1 .. log2 n in increasing order, level l holding n >> l rows; row j of
 * level l is the exact sum of keys [j*2^l, (j+1)*2^l). At d = 128 a level whose sums are bounded
 * by value_bound * 2^l <= 32767 is stored as int16 rows of 2d bytes ("narrow" levels 1 ..
 * alhr_tree_narrow_levels); every other level (every level at d = 64) as int32 rows of 4d
 * bytes. The byte offset of a
 * level inside a block is alhr_tree_level_offset(). The layout depends on value_bound, so every
 * call that reads a tree must pass the value_bound it was built with. alhr_tree_unpack expands
 * a tree to plain int32 rows.
 *
 * Ownership: every pointer belongs to the caller. The library allocates no device memory and
 * keeps no state between calls; a call only reads its inputs and writes its outputs.
 *
 * Streams: `stream` is a cudaStream_t passed as void* (NULL = legacy default stream). All
 * compute entry points are asynchronous with respect to the host.
 *
 * Errors: arguments are checked on the host before anything is launched; on any non-OK
 * status nothing has been launched and no output has been written. A launch failure returns
 * ALHR_ERR_CUDA. Conditions that only the device can see never trap; the kernel handles them
 * as listed and ORs the matching bit into *dev_err when dev_err is non-NULL:
 *   ALHR_DEVERR_BUDGET_LOW   a budget below 1 was read: it is treated as 1;
 *   ALHR_DEVERR_VALUE_RANGE  a Q or K value outside [-value_bound, value_bound]: it is used as
 *                            is (results stay defined, but narrow tree levels and int32 scores
 *                            may no longer be exact);
 *   ALHR_DEVERR_INDEX        alhr_attend: an idx entry outside [0, i] is skipped (weight 0);
 *   ALHR_DEVERR_TIMEOUT      alhr_topk_labels: a bounded wait on the tensor core ran out; the
 *                            rows of that CTA's query tile (128 queries) are NOT written, so
 *                            labels and scores there keep whatever the buffers held before.
 * Kernels contain no unbounded loop; the only waits (alhr_topk_labels, on its own MMAs) are
 * bounded.
 */
#ifndef ALHR_H
#define ALHR_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ALHR_API __attribute__((visibility("default")))
#else
#define ALHR_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ALHR_OK = 0,
  ALHR_ERR_INVALID_ARG = 1,  /* a NULL required pointer, a misaligned pointer, a bad size   */
  ALHR_ERR_UNSUPPORTED = 2,  /* sizes the kernels do not handle (d, window, max_keys, n)    */
  ALHR_ERR_OVERFLOW = 3,     /* score_bits = 32 requested where int32 scores could overflow */
  ALHR_ERR_CUDA = 4          /* a CUDA launch or runtime call failed                        */
} alhr_status;

/* Bits OR-ed into the optional device word *dev_err. */
#define ALHR_DEVERR_BUDGET_LOW  0x1u /* a budget < 1 was read; it was treated as 1          */
#define ALHR_DEVERR_VALUE_RANGE 0x2u /* a Q or K value had |value| > value_bound            */
#define ALHR_DEVERR_INDEX       0x4u /* alhr_attend: an idx entry outside [0, i] was skipped */
#define ALHR_DEVERR_TIMEOUT     0x8u /* alhr_topk_labels: a bounded wait on the tensor core ran
                                        out; that CTA's rows were not written                */

/* Problem sizes, shared by every entry point. */
typedef struct {
  int32_t batch;       /* >= 1; batch * heads < 2^31 (else ALHR_ERR_UNSUPPORTED)          */
  int32_t heads;       /* >= 1                                                            */
  int32_t n;           /* keys per (b,h): a power of two, 2 <= n <= 2^20                  */
  int32_t d;           /* head dimension: 64 or 128                                       */
  int32_t q_start;     /* first query position; prefill 0, decode n-1                     */
  int32_t nq;          /* queries per (b,h); 0 <= nq, q_start + nq <= n                   */
  int32_t window;      /* neighbour window w, 1 <= w <= 32                                */
  int32_t max_keys;    /* cap on keys per query, 1 <= max_keys <= 96                      */
  int32_t score_bits;  /* 0 = choose, 32 = int32 scores (checked), 64 = int64 scores      */
  int32_t value_bound; /* bound on |Q|, |K|; 0 means 16; at most 127                      */
  int32_t score_norm;  /* descent variant: 0 rank by q . node_sum (the method), 1 by mean    */
  int32_t bucket_log;  /* descent variant: 0 descend to keys (the method), b in 1..15: stop  */
                       /* at buckets of 2^b keys                                          */
} alhr_dims;

/*
 * Descent variants (alhr_route and alhr_forward; both 0 is the method as described):
 *   score_norm = 1: candidates are ranked by their mean score q . node_sum / 2^level instead of
 *     the sum, compared exactly (the kernel ranks by q . node_sum * 2^(log2 n - level)); equal
 *     means go to the lower start. Block-sparse methods rank blocks by such means [page
 *     "ALHR把注意力变成树搜索", §"它和块稀疏、线性注意力有什么区别"].
 *   bucket_log = b > 0: leaf buckets of 2^b keys [same page, §"次二次复杂度成立，需要满足三个前提":
 *     the leaf bucket must not grow with the sequence]. A node of level <= b is not expanded;
 *     the beam keeps r >> b nodes, r being the routed key budget (so at most r keys); the
 *     descent ends when the frontier holds only buckets (the roots are pruned too when they all
 *     are buckets) and every key of every kept bucket is selected and scored.
 * With score_norm = 1 the int32 score width needs d * value_bound^2 * n < 2^31 (the ranking
 * value of a key is q . k * n).
 */

/* Number of tree rows per (b,h): n - 1. Returns 0 when n is not a power of two in [2, 2^20]. */
ALHR_API size_t alhr_tree_rows(int32_t n);

/* Number of narrow (int16) levels: at d = 128 the largest l with value_bound * 2^l <= 32767
 * (value_bound 0 means 16), capped at log2 n; at d = 64 none (every level is int32: there the
 * descent is bound by instruction issue, not by row bytes). -1 for invalid arguments. */
ALHR_API int32_t alhr_tree_narrow_levels(int32_t n, int32_t d, int32_t value_bound);

/* Bytes of one (b,h) block of the tree (a multiple of 128), or 0 for invalid arguments
 * (n a power of two in [2, 2^20], d in {64, 128}, 0 <= value_bound <= 127). */
ALHR_API size_t alhr_tree_bytes(int32_t n, int32_t d, int32_t value_bound);

/* Byte offset of tree level `level` (1 <= level <= log2 n) inside one (b,h) block. Level 0 (the
 * keys themselves) is K and is not stored. Returns (size_t)-1 for invalid arguments. */
ALHR_API size_t alhr_tree_level_offset(int32_t n, int32_t d, int32_t value_bound, int32_t level);

/* Score width the kernels will use for these sizes (32 or 64), or a negative alhr_status
 * (-ALHR_ERR_...) when the sizes are invalid or score_bits = 32 cannot be exact. */
ALHR_API int32_t alhr_score_bits(const alhr_dims* dims);

/* Human-readable name of a status code (static storage, never NULL). */
ALHR_API const char* alhr_status_string(int32_t status);

/* Build identification (static storage): target architecture and library version. */
ALHR_API const char* alhr_build_info(void);

/*
 * Launch shape of the per-query kernels (alhr_forward, alhr_route, alhr_predict_budget), a
 * process-wide setting. Trees, budgets, index sets, counts and expansions are identical in every
 * mode; outputs may differ in the last bits of fp32 (another summation order of the value rows).
 *   ALHR_LAUNCH_AUTO (default): the latency shape when every query of the launch is resident at
 *     once in it (four warps per query while the four-warp CTAs all fit, about 4 per SM; else
 *     two warps per query while those fit, about 7-8 per SM): decode and other small launches;
 *     the throughput shape above.
 *   ALHR_LAUNCH_THROUGHPUT: one warp per query, two CTAs of 14 warps per SM, each warp taking
 *     the next query of its CTA's share from a counter in shared memory.
 *   ALHR_LAUNCH_LATENCY: one CTA of four warps per query, in several waves when the launch has
 *     more queries than resident CTAs.
 * alhr_set_launch_mode returns ALHR_ERR_INVALID_ARG (and changes nothing) for any other value.
 */
typedef enum {
  ALHR_LAUNCH_AUTO = 0,
  ALHR_LAUNCH_THROUGHPUT = 1,
  ALHR_LAUNCH_LATENCY = 2
} alhr_launch_mode;
ALHR_API alhr_status alhr_set_launch_mode(int32_t mode);
ALHR_API int32_t alhr_get_launch_mode(void);

/*
 * alhr_build_tree -- the static key tree [README §Inference stage, first paragraph: the tree
 * is built on the key matrix and stored, once per layer; README opening paragraph: every
 * branch is indexed by the sum of all key vectors beneath it].
 *
 * For every (b,h) writes node(l, j) = sum_{t in [j*2^l, (j+1)*2^l)} K[t] for l = 1..log2 n,
 * exact, in the tree layout above. Only dims->batch, heads, n, d and value_bound are read.
 *   K       device, int8 [batch][heads][n][d], read only
 *   tree    device, 32-byte aligned, batch*heads*alhr_tree_bytes(n, d, value_bound) bytes,
 *           fully overwritten
 *   dev_err device uint32 or NULL; ALHR_DEVERR_VALUE_RANGE if some |K| > value_bound (the
 *           narrow levels are then not exact)
 */
ALHR_API alhr_status alhr_build_tree(const alhr_dims* dims, const int8_t* K, void* tree,
                                     uint32_t* dev_err, void* stream);

/*
 * alhr_topk_labels -- phase-2 labels [README §Training stage, Phase 2: the top-k keys of every
 * query are read off the dense model's attention matrix; §Results and Variables: k = 16].
 *
 * For every (b,h) and query row r (position i = q_start + r) writes the k keys t <= i with the
 * largest exact q . K[t] (the order softmax keeps), best first, equal scores to the lower t;
 * rows with fewer than k causal keys are padded with -1 (and score 0). Scores are computed on
 * the tensor cores (int8 x int8 -> int32, exact) tile by tile; nothing of size n x n is stored.
 * Reads dims->batch, heads, n, d, q_start, nq.
 *   Q       device, int8 [batch][heads][nq][d]; K device, int8 [batch][heads][n][d]
 *   k       1 <= k <= 16
 *   labels  device int32 [batch][heads][nq][k], written
 *   scores  device int32 [batch][heads][nq][k] or NULL, written
 *   dev_err device uint32 or NULL; ALHR_DEVERR_TIMEOUT if a bounded wait on the tensor core
 *           ran out (not expected): the 128-query tile of that CTA is then left unwritten in
 *           labels and scores, and the caller should treat the whole call's outputs as invalid
 * ALHR_ERR_INVALID_ARG for bad sizes or pointers (Q, K 16-byte aligned).
 */
ALHR_API alhr_status alhr_topk_labels(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                                      int32_t k, int32_t* labels, int32_t* scores,
                                      uint32_t* dev_err, void* stream);

/*
 * alhr_update_tree -- the tree after rows [lo, hi) of K changed, e.g. the keys of new tokens
 * appended during decoding [README §Inference stage, first paragraph: the tree is built on the
 * key matrix; page "ALHR把注意力变成树搜索", §"ALHR是什么：让每个Query沿树寻找Key": a new
 * token's attention during decoding; §"接下来最该验证的不是更高压缩比": per-token decode latency
 * is one of the figures to report].
 *
 * Precondition: for every (b,h), `tree` equals what alhr_build_tree wrote (or this call left)
 * for a key matrix that differs from K at most in rows [lo, hi). Postcondition: `tree` equals
 * alhr_build_tree(K), byte for byte. Only the rows over [lo, hi) are read and written: for
 * hi - lo <= 64 one kernel moves every ancestor by the exact change of the level-1 sums beneath
 * it (the old pair sum is the stored level-1 row, so no old key is needed; O(log2 n) rows per
 * (b,h) for one key); larger ranges rebuild the 128-row chunks that cover them, level group by
 * level group. Reads dims->batch, heads, n, d and value_bound.
 *   K       device, int8 [batch][heads][n][d], read only (rows outside [lo, hi) too: the pair
 *           and chunk neighbours)
 *   tree    device, as for alhr_build_tree, updated in place
 *   lo, hi  0 <= lo <= hi <= n, the same for every (b,h); lo == hi does nothing
 *   dev_err device uint32 or NULL; ALHR_DEVERR_VALUE_RANGE if some |K| > value_bound in the rows
 *           read
 * ALHR_ERR_INVALID_ARG for a bad range or pointer. Not thread-safe against kernels reading the
 * same tree on another stream (order them with the caller's stream or events).
 */
ALHR_API alhr_status alhr_update_tree(const alhr_dims* dims, const int8_t* K, void* tree,
                                      int32_t lo, int32_t hi, uint32_t* dev_err, void* stream);

/*
 * alhr_tree_unpack -- the tree as plain int32 rows: nodes[b][h][r][:] for r in [0, n-1), level l
 * at rows [n - (n >> (l-1)), n - (n >> l)) (level-major, level 1 first). Reads dims->batch,
 * heads, n, d and value_bound.
 *   tree   device, as written by alhr_build_tree with the same dims
 *   nodes  device, int32 [batch][heads][n-1][d], fully overwritten
 */
ALHR_API alhr_status alhr_tree_unpack(const alhr_dims* dims, const void* tree, int32_t* nodes,
                                      void* stream);

/*
 * alhr_tree_pack -- the inverse of alhr_tree_unpack: plain level-major int32 node rows (the
 * nodes[b][h][r][:] layout above; node(l, j) = sum of keys [j*2^l, (j+1)*2^l)) written into the
 * tree layout that alhr_predict_budget, alhr_route and alhr_forward read, for callers that
 * build or keep the key tree as int32 rows themselves [README opening paragraph: every branch
 * is indexed by the sum of the key vectors beneath it]. Reads dims->batch, heads, n, d and
 * value_bound.
 *   nodes   device, int32 [batch][heads][n-1][d], 16-byte aligned, read only
 *   tree    device, 32-byte aligned, batch*heads*alhr_tree_bytes(n, d, value_bound) bytes,
 *           fully overwritten
 *   dev_err device uint32 or NULL; ALHR_DEVERR_VALUE_RANGE if a value of a narrow (int16)
 *           level l lies outside [-value_bound * 2^l, value_bound * 2^l] (it cannot then be a
 *           sum of keys within the bound; it is stored saturated to int16)
 * alhr_tree_pack(alhr_tree_unpack(tree)) == tree for every tree alhr_build_tree wrote.
 */
ALHR_API alhr_status alhr_tree_pack(const alhr_dims* dims, const int32_t* nodes, void* tree,
                                    uint32_t* dev_err, void* stream);

/*
 * alhr_predict_budget -- the budget predictor [README §Inference stage, second paragraph: a
 * trainable function of the current query and the global key sum that outputs a leaf group,
 * i.e. the number of keys the query asks for; §Results and Variables: 32 classes, <= 96 keys].
 *
 * For the query at position i: G_i = sum_{t <= i} K[t] (the key sum read causally),
 * logit_c = sum_t W[c][t] q_t + sum_t W[c][d+t] G_i[t] for c = 0..31 in int64,
 * c* = the smallest c with the largest logit, budget = 3*(c*+1).
 * G_i is formed from the tree: the roots of the past-only forest of [0, i-w] plus the window
 * keys (i-w, i].
 *   Q, K, tree   device inputs (layouts above); W device int8 [32][2d]
 *   budget       device int32 [batch][heads][nq], overwritten
 *   dev_err      as above (ALHR_DEVERR_VALUE_RANGE for |q| > value_bound)
 */
ALHR_API alhr_status alhr_predict_budget(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                                         const void* tree, const int8_t* W, int32_t* budget,
                                         uint32_t* dev_err, void* stream);

/*
 * alhr_route -- neighbour search plus budget-limited tree descent [README §Inference stage,
 * third and fourth paragraphs; §Training stage, last paragraph: causality by descending only
 * the subtrees that hold past keys].
 *
 * For the query at position i with budget B (read from `budget`):
 *   B_eff = min(max(B,1), i+1, max_keys);
 *   window: keys i, i-1, ..., max(0, i-w+1), nearest first, cut to B_eff;
 *   r = B_eff - |window|; if r > 0 and i >= w, descend the forest of aligned power-of-two
 *   roots of [0, i-w] (the maximal past-only subtrees, largest first): repeatedly replace every
 *   non-leaf frontier node by its two children and keep the r nodes with the largest exact
 *   integer q . node_sum (ties: lower start position), until every frontier node is a key.
 *   The routed keys are the final frontier; the selection is window + routed.
 *   idx        device int32 [..][max_keys]: selection ascending, -1 padded (required)
 *   count      device int32: |selection| = min(B_eff, i+1) (required)
 *   expansions device int32 [..][3] or NULL: the three expansion counters of the layout table
 *   dev_err    as above (ALHR_DEVERR_BUDGET_LOW, ALHR_DEVERR_VALUE_RANGE)
 */
ALHR_API alhr_status alhr_route(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                                const void* tree, const int32_t* budget, int32_t* idx,
                                int32_t* count, int32_t* expansions, uint32_t* dev_err,
                                void* stream);

/*
 * alhr_attend -- exact attention over the selected keys [README §Inference stage, fifth
 * paragraph: once each query has its keys, standard dot-product attention and sum run].
 *
 * out_i = sum_j softmax_j(s) V[j] over j in idx[0..count), s_j = (q_i . K[j]) / sqrt(d), with the
 * integer dot product exact and the softmax and sum in fp32. A query with count <= 0 gets a
 * zero row. Entries of idx outside [0, i] are skipped (not read) and flag ALHR_DEVERR_INDEX.
 *   Q, K, V, idx, count  device inputs (layouts above)
 *   out                  device float [batch][heads][nq][d], overwritten
 */
ALHR_API alhr_status alhr_attend(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                        const uint16_t* V, const int32_t* idx, const int32_t* count, float* out,
                        uint32_t* dev_err, void* stream);

/*
 * alhr_forward -- the whole inference path in one kernel per query: causal key sum, budget
 * predictor (or budget_override), window, descent and exact attention [README §Inference
 * stage, all five paragraphs]. The tree must have been built by alhr_build_tree.
 *   W                device int8 [32][2d]; may be NULL only when budget_override is given
 *   budget_override  device int32 [batch][heads][nq] or NULL (NULL = use the predictor)
 *   out              device float [batch][heads][nq][d] (required)
 *   idx, count, expansions, budget_out  optional outputs (NULL = not written); budget_out
 *                    receives the budget each query used (predicted or overridden, after the
 *                    clamp to >= 1)
 * Results equal alhr_predict_budget + alhr_route + alhr_attend on the same inputs.
 */
ALHR_API alhr_status alhr_forward(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                         const uint16_t* V, const void* tree, const int8_t* W,
                         const int32_t* budget_override, float* out, int32_t* idx,
                         int32_t* count, int32_t* expansions, int32_t* budget_out,
                         uint32_t* dev_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ALHR_H */
