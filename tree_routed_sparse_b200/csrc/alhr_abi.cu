// alhr_abi.cu -- the C ABI of libalhr.so: argument checks, score-width choice, launches.
//
// Every entry point checks its arguments on the host before anything is launched and returns
// a status; nothing is allocated and no state is kept between calls.
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/alhr.h"
#include "alhr_device.cuh"
#include "internal.h"

namespace {

bool pow2_in_range(int32_t n) { return n >= 2 && n <= (1 << 20) && (n & (n - 1)) == 0; }

int log2_exact(int32_t n) {
  int l = 0;
  while ((int64_t(1) << l) < n) ++l;
  return l;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
// the tree is read with 32-byte loads
bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

int value_bound_of(const alhr_dims* d) { return d->value_bound == 0 ? 16 : d->value_bound; }

// Sizes shared by every entry point.
alhr_status check_common(const alhr_dims* d) {
  if (!d) return ALHR_ERR_INVALID_ARG;
  if (d->batch < 1 || d->heads < 1) return ALHR_ERR_INVALID_ARG;
  if (int64_t(d->batch) * d->heads > int64_t(INT32_MAX)) return ALHR_ERR_UNSUPPORTED;
  if (!pow2_in_range(d->n)) return ALHR_ERR_INVALID_ARG;
  if (d->d != 64 && d->d != 128) return ALHR_ERR_UNSUPPORTED;
  if (d->value_bound < 0 || d->value_bound > 127) return ALHR_ERR_INVALID_ARG;
  return ALHR_OK;
}

alhr_status check_queries(const alhr_dims* d) {
  const alhr_status s = check_common(d);
  if (s != ALHR_OK) return s;
  if (d->q_start < 0 || d->nq < 0 || int64_t(d->q_start) + d->nq > d->n) return ALHR_ERR_INVALID_ARG;
  if (d->window < 1) return ALHR_ERR_INVALID_ARG;
  if (d->window > 32) return ALHR_ERR_UNSUPPORTED;
  if (d->max_keys < 1) return ALHR_ERR_INVALID_ARG;
  if (d->max_keys > alhr::kMaxKeys) return ALHR_ERR_UNSUPPORTED;
  if (d->score_bits != 0 && d->score_bits != 32 && d->score_bits != 64) return ALHR_ERR_INVALID_ARG;
  if (d->score_norm != 0 && d->score_norm != 1) return ALHR_ERR_INVALID_ARG;
  if (d->bucket_log < 0 || d->bucket_log > 15) return ALHR_ERR_INVALID_ARG;
  return ALHR_OK;
}

// Largest |ranking value| over every node a query can score: the biggest root of [0, i - w]
// has level <= log2 n - 1, so |q . node| <= d * vb^2 * n/2 (and d * vb^2 for a key); ranked by
// means, a node's value is q . node << (log2 n - level), at most d * vb^2 * n.
int64_t score_bound(const alhr_dims* d) {
  const int64_t vb = value_bound_of(d);
  const int64_t per = int64_t(d->d) * vb * vb;
  return d->score_norm ? per * int64_t(d->n) : per * (int64_t(d->n) / 2);
}

int resolve_bits(const alhr_dims* d, alhr_status* st) {
  const bool fits32 = score_bound(d) <= int64_t(INT32_MAX);
  *st = ALHR_OK;
  if (d->score_bits == 32) {
    if (!fits32) *st = ALHR_ERR_OVERFLOW;
    return 32;
  }
  if (d->score_bits == 64) return 64;
  return fits32 ? 32 : 64;
}

alhr::QueryArgs base_args(const alhr_dims* d) {
  alhr::QueryArgs a{};
  a.n = d->n;
  a.L = log2_exact(d->n);
  a.q_start = d->q_start;
  a.nq = d->nq;
  a.window = d->window;
  a.max_keys = d->max_keys;
  a.value_bound = value_bound_of(d);
  a.num_queries = int64_t(d->batch) * d->heads * d->nq;
  a.scale = float(1.0 / std::sqrt(double(d->d)));
  a.tl = alhr::make_tree_layout(d->n, d->d, d->value_bound);
  a.norm_l = d->score_norm ? a.L : 0;
  a.bucket = d->bucket_log;
  return a;
}

alhr_status from_cuda(cudaError_t e) { return e == cudaSuccess ? ALHR_OK : ALHR_ERR_CUDA; }

}  // namespace

extern "C" {

size_t alhr_tree_rows(int32_t n) { return pow2_in_range(n) ? size_t(n) - 1 : 0; }

int32_t alhr_tree_narrow_levels(int32_t n, int32_t d, int32_t value_bound) {
  if (!pow2_in_range(n) || (d != 64 && d != 128) || value_bound < 0 || value_bound > 127) return -1;
  return alhr::make_tree_layout(n, d, value_bound).narrow;
}

size_t alhr_tree_bytes(int32_t n, int32_t d, int32_t value_bound) {
  if (!pow2_in_range(n) || (d != 64 && d != 128) || value_bound < 0 || value_bound > 127) return 0;
  return size_t(alhr::make_tree_layout(n, d, value_bound).block_bytes);
}

size_t alhr_tree_level_offset(int32_t n, int32_t d, int32_t value_bound, int32_t level) {
  if (!pow2_in_range(n) || (d != 64 && d != 128) || value_bound < 0 || value_bound > 127 ||
      level < 1 || level > log2_exact(n))
    return size_t(-1);
  return size_t(alhr::make_tree_layout(n, d, value_bound).level_off[level]);
}

int32_t alhr_score_bits(const alhr_dims* d) {
  alhr_status s = check_queries(d);
  if (s != ALHR_OK) return -int32_t(s);
  const int bits = resolve_bits(d, &s);
  return s == ALHR_OK ? bits : -int32_t(s);
}

const char* alhr_status_string(int32_t status) {
  switch (status) {
    case ALHR_OK: return "ALHR_OK";
    case ALHR_ERR_INVALID_ARG: return "ALHR_ERR_INVALID_ARG";
    case ALHR_ERR_UNSUPPORTED: return "ALHR_ERR_UNSUPPORTED";
    case ALHR_ERR_OVERFLOW: return "ALHR_ERR_OVERFLOW";
    case ALHR_ERR_CUDA: return "ALHR_ERR_CUDA";
    default: return "ALHR_ERR_UNKNOWN";
  }
}

const char* alhr_build_info(void) { return "libalhr 0.1 sm_100a"; }

alhr_status alhr_set_launch_mode(int32_t mode) {
  if (mode != ALHR_LAUNCH_AUTO && mode != ALHR_LAUNCH_THROUGHPUT && mode != ALHR_LAUNCH_LATENCY)
    return ALHR_ERR_INVALID_ARG;
  alhr::set_query_launch_mode(mode);
  return ALHR_OK;
}

int32_t alhr_get_launch_mode(void) { return alhr::query_launch_mode(); }

alhr_status alhr_build_tree(const alhr_dims* dims, const int8_t* K, void* tree,
                            uint32_t* dev_err, void* stream) {
  const alhr_status s = check_common(dims);
  if (s != ALHR_OK) return s;
  if (!K || !tree || !aligned16(K) || !aligned32(tree)) return ALHR_ERR_INVALID_ARG;
  const long long bh = (long long)dims->batch * dims->heads;
  const alhr::TreeLayout tl = alhr::make_tree_layout(dims->n, dims->d, dims->value_bound);
  return from_cuda(alhr::launch_build_tree(K, static_cast<char*>(tree), tl, bh,
                                           value_bound_of(dims), dev_err,
                                           static_cast<cudaStream_t>(stream)));
}

alhr_status alhr_topk_labels(const alhr_dims* dims, const int8_t* Q, const int8_t* K, int32_t k,
                             int32_t* labels, int32_t* scores, uint32_t* dev_err, void* stream) {
  const alhr_status s = check_common(dims);
  if (s != ALHR_OK) return s;
  if (dims->q_start < 0 || dims->nq < 0 || int64_t(dims->q_start) + dims->nq > dims->n)
    return ALHR_ERR_INVALID_ARG;
  if (k < 1 || k > 16) return ALHR_ERR_INVALID_ARG;
  if (dims->nq == 0) return ALHR_OK;
  if (!Q || !K || !labels || !aligned16(Q) || !aligned16(K)) return ALHR_ERR_INVALID_ARG;
  const long long bh = (long long)dims->batch * dims->heads;
  return from_cuda(alhr::launch_topk_labels(Q, K, labels, scores, dims->n, dims->d,
                                            dims->q_start, dims->nq, k, bh, dev_err,
                                            static_cast<cudaStream_t>(stream)));
}

alhr_status alhr_update_tree(const alhr_dims* dims, const int8_t* K, void* tree, int32_t lo,
                             int32_t hi, uint32_t* dev_err, void* stream) {
  const alhr_status s = check_common(dims);
  if (s != ALHR_OK) return s;
  if (lo < 0 || hi < lo || hi > dims->n) return ALHR_ERR_INVALID_ARG;
  if (lo == hi) return ALHR_OK;
  if (!K || !tree || !aligned16(K) || !aligned32(tree)) return ALHR_ERR_INVALID_ARG;
  const long long bh = (long long)dims->batch * dims->heads;
  const alhr::TreeLayout tl = alhr::make_tree_layout(dims->n, dims->d, dims->value_bound);
  return from_cuda(alhr::launch_update_tree(K, static_cast<char*>(tree), tl, bh, lo, hi,
                                            value_bound_of(dims), dev_err,
                                            static_cast<cudaStream_t>(stream)));
}

alhr_status alhr_tree_unpack(const alhr_dims* dims, const void* tree, int32_t* nodes,
                             void* stream) {
  const alhr_status s = check_common(dims);
  if (s != ALHR_OK) return s;
  if (!tree || !nodes || !aligned32(tree) || !aligned16(nodes)) return ALHR_ERR_INVALID_ARG;
  const long long bh = (long long)dims->batch * dims->heads;
  const alhr::TreeLayout tl = alhr::make_tree_layout(dims->n, dims->d, dims->value_bound);
  return from_cuda(alhr::launch_tree_unpack(static_cast<const char*>(tree), tl, bh, nodes,
                                            static_cast<cudaStream_t>(stream)));
}

alhr_status alhr_tree_pack(const alhr_dims* dims, const int32_t* nodes, void* tree,
                           uint32_t* dev_err, void* stream) {
  const alhr_status s = check_common(dims);
  if (s != ALHR_OK) return s;
  if (!tree || !nodes || !aligned32(tree) || !aligned16(nodes)) return ALHR_ERR_INVALID_ARG;
  const long long bh = (long long)dims->batch * dims->heads;
  const alhr::TreeLayout tl = alhr::make_tree_layout(dims->n, dims->d, dims->value_bound);
  return from_cuda(alhr::launch_tree_pack(nodes, tl, bh, value_bound_of(dims),
                                          static_cast<char*>(tree), dev_err,
                                          static_cast<cudaStream_t>(stream)));
}

alhr_status alhr_predict_budget(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                                const void* tree, const int8_t* W, int32_t* budget,
                                uint32_t* dev_err, void* stream) {
  alhr_status s = check_queries(dims);
  if (s != ALHR_OK) return s;
  const int bits = resolve_bits(dims, &s);
  if (s != ALHR_OK) return s;
  if (dims->nq == 0) return ALHR_OK;  // nothing to read or write
  if (!Q || !K || !tree || !W || !budget) return ALHR_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned32(tree) || !aligned16(W)) return ALHR_ERR_INVALID_ARG;
  alhr::QueryArgs a = base_args(dims);
  a.Q = Q; a.K = K; a.tree = static_cast<const char*>(tree); a.W = W; a.budget_out = budget; a.dev_err = dev_err;
  return from_cuda(alhr::launch_predict(a, dims->d, bits, static_cast<cudaStream_t>(stream)));
}

alhr_status alhr_route(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                       const void* tree, const int32_t* budget, int32_t* idx, int32_t* count,
                       int32_t* expansions, uint32_t* dev_err, void* stream) {
  alhr_status s = check_queries(dims);
  if (s != ALHR_OK) return s;
  const int bits = resolve_bits(dims, &s);
  if (s != ALHR_OK) return s;
  if (dims->nq == 0) return ALHR_OK;  // nothing to read or write
  if (!Q || !K || !tree || !budget || !idx || !count) return ALHR_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned32(tree)) return ALHR_ERR_INVALID_ARG;
  alhr::QueryArgs a = base_args(dims);
  a.Q = Q; a.K = K; a.tree = static_cast<const char*>(tree); a.budget_in = budget;
  a.idx_out = idx; a.count_out = count; a.exp_out = expansions; a.dev_err = dev_err;
  return from_cuda(alhr::launch_route(a, dims->d, bits, static_cast<cudaStream_t>(stream)));
}

alhr_status alhr_attend(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                        const uint16_t* V, const int32_t* idx, const int32_t* count, float* out,
                        uint32_t* dev_err, void* stream) {
  const alhr_status s = check_queries(dims);
  if (s != ALHR_OK) return s;
  if (dims->nq == 0) return ALHR_OK;  // nothing to read or write
  if (!Q || !K || !V || !idx || !count || !out) return ALHR_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(out)) return ALHR_ERR_INVALID_ARG;
  alhr::QueryArgs a = base_args(dims);
  a.Q = Q; a.K = K; a.V = V; a.idx_in = idx; a.count_in = count; a.out = out; a.dev_err = dev_err;
  return from_cuda(alhr::launch_attend(a, dims->d, static_cast<cudaStream_t>(stream)));
}

alhr_status alhr_forward(const alhr_dims* dims, const int8_t* Q, const int8_t* K,
                         const uint16_t* V, const void* tree, const int8_t* W,
                         const int32_t* budget_override, float* out, int32_t* idx,
                         int32_t* count, int32_t* expansions, int32_t* budget_out,
                         uint32_t* dev_err, void* stream) {
  alhr_status s = check_queries(dims);
  if (s != ALHR_OK) return s;
  const int bits = resolve_bits(dims, &s);
  if (s != ALHR_OK) return s;
  if (dims->nq == 0) return ALHR_OK;  // nothing to read or write
  if (!Q || !K || !V || !tree || !out) return ALHR_ERR_INVALID_ARG;
  if (!W && !budget_override) return ALHR_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned32(tree) || !aligned16(out))
    return ALHR_ERR_INVALID_ARG;
  if (!budget_override && !aligned16(W)) return ALHR_ERR_INVALID_ARG;
  alhr::QueryArgs a = base_args(dims);
  a.Q = Q; a.K = K; a.V = V; a.tree = static_cast<const char*>(tree); a.W = W;
  a.budget_in = budget_override;
  a.out = out; a.idx_out = idx; a.count_out = count; a.exp_out = expansions;
  a.budget_out = budget_out; a.dev_err = dev_err;
  return from_cuda(alhr::launch_forward(a, dims->d, bits, budget_override == nullptr,
                                        static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
