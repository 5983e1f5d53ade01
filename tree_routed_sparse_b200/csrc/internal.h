// internal.h -- launchers shared between the C ABI layer and the kernel files.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "tree_layout.h"

namespace alhr {

struct QueryArgs;

// Tree build: levels 1..log2 n of every (b,h) block (see tree_build.cu).
cudaError_t launch_build_tree(const int8_t* K, char* tree, const TreeLayout& tl, long long bh,
                              int value_bound, uint32_t* dev_err, cudaStream_t st);
// After rows [lo, hi) of K changed: every tree row over them, made equal to a full build's
// (see tree_build.cu).
cudaError_t launch_update_tree(const int8_t* K, char* tree, const TreeLayout& tl, long long bh,
                               int lo, int hi, int value_bound, uint32_t* dev_err,
                               cudaStream_t st);
// The tree as plain int32 rows, level-major (see tree_build.cu).
cudaError_t launch_tree_unpack(const char* tree, const TreeLayout& tl, long long bh,
                               int32_t* nodes, cudaStream_t st);
// Plain int32 rows into the tree layout (see tree_build.cu).
cudaError_t launch_tree_pack(const int32_t* nodes, const TreeLayout& tl, long long bh, int vb,
                             char* tree, uint32_t* dev_err, cudaStream_t st);

// Warp-per-query kernels (see query_kernels.cu).
cudaError_t launch_forward(const QueryArgs& a, int d, int score_bits, bool predict,
                           cudaStream_t st);
cudaError_t launch_route(const QueryArgs& a, int d, int score_bits, cudaStream_t st);
cudaError_t launch_predict(const QueryArgs& a, int d, int score_bits, cudaStream_t st);
cudaError_t launch_attend(const QueryArgs& a, int d, cudaStream_t st);
// The latency shape: one query per CTA (see cta_query_kernels.cu); mode is a Mode of
// query_common.cuh. Unless `forced`, it launches only when every query is resident at once
// (*launched tells whether it launched; if not, the caller takes the throughput shape).
cudaError_t launch_query_cta(const QueryArgs& a, int d, int score_bits, int mode, bool forced,
                             bool* launched, cudaStream_t st);

// Phase-2 labels: top-k keys of every query's causal q . K row (see label_kernels.cu).
cudaError_t launch_topk_labels(const int8_t* Q, const int8_t* K, int32_t* labels,
                               int32_t* scores, int n, int d, int q_start, int nq, int k,
                               long long bh, uint32_t* dev_err, cudaStream_t st);

// Process-wide launch shape of the per-query kernels: 0 auto, 1 throughput, 2 latency.
void set_query_launch_mode(int mode);
int query_launch_mode();

}  // namespace alhr
