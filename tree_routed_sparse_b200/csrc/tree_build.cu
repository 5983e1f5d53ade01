// tree_build.cu -- the static key tree of ALHR on sm_100a.
//
// README of ALHR ("Adaptive learnable Hierarchical routing"), opening paragraph: every branch
// of the static binary tree is indexed by the sum of the key vectors beneath it; section
// "Inference stage", first paragraph: the tree is built on the key matrix once per layer and
// stored.
//
// One CTA owns a chunk of 2^m consecutive rows of level `lin` (lin = 0: the int8 keys) of one
// (b,h) and produces levels lin+1 .. lin+m of that chunk entirely in shared memory, so the keys
// are read once and every tree row is written once (algorithmic bytes = K + tree). Rows are
// moved with 16-byte vector accesses; a row of a level is contiguous with its neighbours, so
// every warp store covers whole 32-byte sectors. Levels above the chunk height are produced by
// further launches over the (much smaller) level-m rows.
#include <cuda_runtime.h>

#include "alhr_device.cuh"
#include "internal.h"

namespace alhr {

namespace {

constexpr int kTreeThreads = 256;
constexpr int kChunkLog = 7;  // 128 input rows per CTA

template <int D, bool kFromKeys>
__global__ void __launch_bounds__(kTreeThreads)
    tree_chunk_kernel(const int8_t* __restrict__ K, int32_t* __restrict__ nodes, int n, int lin,
                      int m, int chunks_per_head, int value_bound, uint32_t* dev_err) {
  extern __shared__ int4 smem4[];  // [2^m][D] int32
  constexpr int Q4 = D / 4;                 // int4 per row
  const long long bh = blockIdx.x / chunks_per_head;
  const int chunk = blockIdx.x - int(bh * chunks_per_head);
  const int rows = 1 << m;
  int32_t* Nh = nodes + bh * (long long)(n - 1) * D;

  if constexpr (kFromKeys) {
    const int4* src = reinterpret_cast<const int4*>(K + (bh * n + (long long)chunk * rows) * D);
    bool bad = false;
    for (int k = threadIdx.x; k < rows * D / 16; k += kTreeThreads) {
      const int4 t = __ldg(src + k);
      const int wv[4] = {t.x, t.y, t.z, t.w};
      int4* dst = smem4 + 4 * k;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int x = wv[u];
        const int4 o = make_int4((x << 24) >> 24, (x << 16) >> 24, (x << 8) >> 24, x >> 24);
        bad |= o.x > value_bound | o.x < -value_bound | o.y > value_bound | o.y < -value_bound |
               o.z > value_bound | o.z < -value_bound | o.w > value_bound | o.w < -value_bound;
        dst[u] = o;
      }
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0 && dev_err)
      atomicOr(dev_err, ALHR_DEVERR_VALUE_RANGE);
  } else {
    const int4* src = reinterpret_cast<const int4*>(Nh + (level_row(n, lin) + (long long)chunk * rows) * D);
    for (int k = threadIdx.x; k < rows * Q4; k += kTreeThreads) smem4[k] = __ldg(src + k);
    __syncthreads();
  }

  // at most (rows/2) * Q4 outputs per level; per thread: rows*Q4/2/256
  constexpr int kMaxPer = ((1 << kChunkLog) / 2) * Q4 / kTreeThreads;
  for (int s = 1; s <= m; ++s) {
    const int orows = rows >> s;
    const int total = orows * Q4;
    int4* dst = reinterpret_cast<int4*>(Nh + (level_row(n, lin + s) + (long long)chunk * orows) * D);
    int4 res[kMaxPer > 0 ? kMaxPer : 1];
#pragma unroll
    for (int u = 0; u < kMaxPer; ++u) {
      const int k = threadIdx.x + u * kTreeThreads;
      if (k < total) {
        const int row = k / Q4, col = k - row * Q4;
        const int4 a = smem4[(2 * row) * Q4 + col];
        const int4 b = smem4[(2 * row + 1) * Q4 + col];
        res[u] = make_int4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
        dst[k] = res[u];
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kMaxPer; ++u) {
      const int k = threadIdx.x + u * kTreeThreads;
      if (k < total) smem4[k] = res[u];
    }
    __syncthreads();
  }
}

template <int D>
cudaError_t build_tree_d(const int8_t* K, int32_t* nodes, long long bh, int n, int value_bound,
                         uint32_t* dev_err, cudaStream_t st) {
  int L = 0;
  while ((1 << L) < n) ++L;
  const size_t smem_max = size_t(1 << kChunkLog) * D * sizeof(int);
  // the opt-in above 48 KB of dynamic shared memory is a per-device function attribute
  static bool configured[128] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128 || !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(tree_chunk_kernel<D, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tree_chunk_kernel<D, false>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 128) configured[dev] = true;
  }
  int lin = 0;
  while (lin < L) {
    const int m = (L - lin) < kChunkLog ? (L - lin) : kChunkLog;
    const int chunks = (n >> lin) >> m;
    const long long grid = bh * chunks;
    const size_t smem = size_t(1 << m) * D * sizeof(int);
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (lin == 0) {
      tree_chunk_kernel<D, true><<<unsigned(grid), kTreeThreads, smem, st>>>(
          K, nodes, n, lin, m, chunks, value_bound, dev_err);
    } else {
      tree_chunk_kernel<D, false><<<unsigned(grid), kTreeThreads, smem, st>>>(
          K, nodes, n, lin, m, chunks, value_bound, dev_err);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    lin += m;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_build_tree(const int8_t* K, int32_t* nodes, long long bh, int n, int d,
                              int value_bound, uint32_t* dev_err, cudaStream_t st) {
  return d == 64 ? build_tree_d<64>(K, nodes, bh, n, value_bound, dev_err, st)
                 : build_tree_d<128>(K, nodes, bh, n, value_bound, dev_err, st);
}

}  // namespace alhr
