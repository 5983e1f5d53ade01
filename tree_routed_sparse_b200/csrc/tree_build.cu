// tree_build.cu -- the static key tree of ALHR on sm_100a.
//
// README of ALHR ("Adaptive learnable Hierarchical routing"), opening paragraph: every branch
// of the static binary tree is indexed by the sum of the key vectors beneath it; section
// "Inference stage", first paragraph: the tree is built on the key matrix once per layer and
// stored.
//
// One CTA owns a chunk of 2^m consecutive rows of level `lin` (lin = 0: the int8 keys) of one
// (b,h) and produces levels lin+1 .. lin+m of that chunk entirely in shared memory (int32), so
// the keys are read once and every tree row is written once (algorithmic bytes = K + tree).
// Rows are written in the block layout of tree_layout.h: int16 for the narrow levels, int32
// above. A level is contiguous, so the stores of a warp cover whole sectors. Levels above the
// chunk height come from further launches over the (much smaller) level-(lin+m) rows.
#include <cuda_runtime.h>

#include "alhr_device.cuh"
#include "internal.h"

namespace alhr {

namespace {

constexpr int kTreeThreads = 256;
constexpr int kChunkLog = 7;   // 128 input rows per CTA
constexpr int kStreamP = 4;    // keys per batch of the streaming kernel: 2^kStreamP
// Levels from the keys per row group of the streaming kernel: 7 for large builds; 5 when the
// build is small (under 2^24 keys in all), where a shorter chain of batches per row group and
// more row groups in flight matter more than the one extra launch for the levels above.
constexpr int kStreamLog = 7;
constexpr int kStreamLogSmall = 5;
constexpr long long kStreamSmallKeys = 1LL << 24;

enum InKind : int { kFromKeys = 0, kFromNarrow = 1, kFromWide = 2 };

template <int D, int IN>
__global__ void __launch_bounds__(kTreeThreads)
    tree_chunk_kernel(const int8_t* __restrict__ K, char* __restrict__ tree, const TreeLayout tl,
                      int lin, int m, int chunk0, int chunks_per_head, int value_bound,
                      uint32_t* dev_err) {
  extern __shared__ int4 smem4[];  // [2^m][D] int32
  constexpr int Q4 = D / 4;        // int4 per row
  const long long bh = blockIdx.x / chunks_per_head;
  const int chunk = chunk0 + int(blockIdx.x - bh * chunks_per_head);
  const int rows = 1 << m;
  const int n = tl.n;
  char* Th = tree + bh * tl.block_bytes;

  if constexpr (IN == kFromKeys) {
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
  } else if constexpr (IN == kFromNarrow) {
    const int4* src = reinterpret_cast<const int4*>(Th + tl.level_off[lin] +
                                                    (long long)chunk * rows * 2 * D);
    for (int k = threadIdx.x; k < rows * D / 8; k += kTreeThreads) {
      const int4 t = __ldg(src + k);  // 8 int16
      const int wv[4] = {t.x, t.y, t.z, t.w};
      int* dst = reinterpret_cast<int*>(smem4) + 8 * k;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        dst[2 * u] = (wv[u] << 16) >> 16;
        dst[2 * u + 1] = wv[u] >> 16;
      }
    }
    __syncthreads();
  } else {
    const int4* src = reinterpret_cast<const int4*>(Th + tl.level_off[lin] +
                                                    (long long)chunk * rows * 4 * D);
    for (int k = threadIdx.x; k < rows * Q4; k += kTreeThreads) smem4[k] = __ldg(src + k);
    __syncthreads();
  }

  // at most (rows/2) * Q4 outputs per level; per thread: rows*Q4/2/256
  constexpr int kMaxPer = ((1 << kChunkLog) / 2) * Q4 / kTreeThreads;
  for (int s = 1; s <= m; ++s) {
    const int lv = lin + s;
    const int orows = rows >> s;
    const int total = orows * Q4;
    const bool narrow = lv <= tl.narrow;
    char* dst = Th + tl.level_off[lv] + (long long)chunk * orows * tl.row_bytes(lv);
    int4 res[kMaxPer > 0 ? kMaxPer : 1];
#pragma unroll
    for (int u = 0; u < kMaxPer; ++u) {
      const int k = threadIdx.x + u * kTreeThreads;
      if (k < total) {
        const int row = k / Q4, col = k - row * Q4;
        const int4 a = smem4[(2 * row) * Q4 + col];
        const int4 b = smem4[(2 * row + 1) * Q4 + col];
        res[u] = make_int4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
        if (narrow) {
          // exact: |sum| <= value_bound * 2^lv <= 32767 on a narrow level
          const uint2 packed = make_uint2((unsigned(res[u].x) & 0xffffu) | (unsigned(res[u].y) << 16),
                                          (unsigned(res[u].z) & 0xffffu) | (unsigned(res[u].w) << 16));
          reinterpret_cast<uint2*>(dst)[k] = packed;
        } else {
          reinterpret_cast<int4*>(dst)[k] = res[u];
        }
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

// Levels 1 .. m straight from the keys, streamed: a row group of D/4 lanes owns one chunk of
// 2^m consecutive keys of one (b,h), lane c holding columns [4c, 4c+4) of every key (one 4-byte
// load per key). The chunk is read in batches of 2^P keys, all loads of a batch issued before
// any sum and one batch ahead; levels 1 .. P above a batch are summed in registers, and levels
// P+1 .. m are carried from batch to batch in a per-lane stack that works like a binary counter
// on the batch index. Every node is written once, as soon as the last key beneath it has been
// read, and no shared memory or barrier is involved, so many batches of many warps are in flight
// at once.
template <int D, int P>
__global__ void __launch_bounds__(kTreeThreads)
    tree_stream_kernel(const int8_t* __restrict__ K, char* __restrict__ tree, const TreeLayout tl,
                       int m, int chunk0, int chunks_per_head, long long units, int value_bound,
                       uint32_t* dev_err) {
  constexpr int G = D / 4;          // lanes per row group
  constexpr int R = 1 << P;         // keys per batch
  constexpr int kMaxUp = kStreamLog - P;  // levels carried across batches (m <= kStreamLog)
  const long long gt = blockIdx.x * (long long)kTreeThreads + threadIdx.x;
  const long long unit = gt / G;
  if (unit >= units) return;        // no warp-wide operation below: a partial warp may leave
  const int c = int(gt - unit * G);
  const long long bh = unit / chunks_per_head;
  const int chunk = chunk0 + int(unit - bh * chunks_per_head);
  const int n = tl.n;
  char* Th = tree + bh * tl.block_bytes;
  const int* src = reinterpret_cast<const int*>(K + (bh * n + ((long long)chunk << m)) * D) + c;
  const int narrow = tl.narrow;

  auto emit = [&](int l, long long j, const int4& v) {
    char* row = Th + tl.level_off[l] + j * (long long)(l <= narrow ? 2 * D : 4 * D);
    if (l <= narrow) {
      // exact: |sum| <= value_bound * 2^l <= 32767 on a narrow level
      *(reinterpret_cast<uint2*>(row) + c) =
          make_uint2(__byte_perm(v.x, v.y, 0x5410), __byte_perm(v.z, v.w, 0x5410));
    } else {
      *(reinterpret_cast<int4*>(row) + c) = v;
    }
  };
  auto sum4 = [](const int4& a, const int4& b) {
    return make_int4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
  };

  int4 stack[kMaxUp > 0 ? kMaxUp : 1];
  bool bad = false;
  const int batches = 1 << (m - P);
  const long long key0 = (long long)chunk << m;  // first key of the chunk
  // the next batch's loads are issued before the current batch is summed (two batches in
  // flight per row group)
  int wn[R];
#pragma unroll
  for (int t = 0; t < R; ++t) wn[t] = __ldg(src + t * (D / 4));
  for (int bi = 0; bi < batches; ++bi) {
    int w[R];
#pragma unroll
    for (int t = 0; t < R; ++t) w[t] = wn[t];
    if (bi + 1 < batches) {
#pragma unroll
      for (int t = 0; t < R; ++t) wn[t] = __ldg(src + ((bi + 1) * R + t) * (D / 4));
    }
    int4 lv[R / 2];
#pragma unroll
    for (int t = 0; t < R / 2; ++t) {
      const int a = w[2 * t], b = w[2 * t + 1];
      const int4 x = make_int4((a << 24) >> 24, (a << 16) >> 24, (a << 8) >> 24, a >> 24);
      const int4 y = make_int4((b << 24) >> 24, (b << 16) >> 24, (b << 8) >> 24, b >> 24);
      bad |= x.x > value_bound | x.x < -value_bound | x.y > value_bound | x.y < -value_bound |
             x.z > value_bound | x.z < -value_bound | x.w > value_bound | x.w < -value_bound |
             y.x > value_bound | y.x < -value_bound | y.y > value_bound | y.y < -value_bound |
             y.z > value_bound | y.z < -value_bound | y.w > value_bound | y.w < -value_bound;
      lv[t] = sum4(x, y);
    }
    const long long b0 = key0 + (long long)bi * R;  // first key of the batch
#pragma unroll
    for (int l = 1; l <= P; ++l) {
      const int cnt = R >> l;
#pragma unroll
      for (int t = 0; t < cnt; ++t) {
        if (l > 1) lv[t] = sum4(lv[2 * t], lv[2 * t + 1]);
        emit(l, (b0 >> l) + t, lv[t]);
      }
    }
    // levels above the batch: carry like a binary counter on bi
    int4 v = lv[0];
    bool carry = true;
#pragma unroll
    for (int s = 1; s <= kMaxUp; ++s) {
      if (s <= m - P && carry) {
        if (((bi >> (s - 1)) & 1) == 0) {
          stack[s - 1] = v;
          carry = false;
        } else {
          v = sum4(stack[s - 1], v);
          emit(P + s, b0 >> (P + s), v);
        }
      }
    }
  }
  if (bad && dev_err) atomicOr(dev_err, ALHR_DEVERR_VALUE_RANGE);
}

// The tree as plain int32 rows: one thread per 4 values of an output row.
template <int D>
__global__ void __launch_bounds__(256)
    tree_unpack_kernel(const char* __restrict__ tree, const TreeLayout tl, long long bh,
                       int4* __restrict__ nodes) {
  constexpr int Q4 = D / 4;
  const int n = tl.n;
  const long long per_block = (long long)(n - 1) * Q4;
  const long long total = bh * per_block;
  for (long long k = blockIdx.x * (long long)blockDim.x + threadIdx.x; k < total;
       k += (long long)gridDim.x * blockDim.x) {
    const long long b = k / per_block;
    const long long rem = k - b * per_block;
    const int r = int(rem / Q4), c = int(rem - (long long)r * Q4);
    int l = 1;
    while (l < tl.L && r >= n - (n >> l)) ++l;  // level l holds rows [n - (n>>(l-1)), n - (n>>l))
    const int j = r - (n - (n >> (l - 1)));
    const char* row = tree + b * tl.block_bytes + tl.level_off[l] + (long long)j * tl.row_bytes(l);
    int4 v;
    if (l <= tl.narrow) {
      const uint2 p = __ldg(reinterpret_cast<const uint2*>(row) + c);
      v = make_int4(int(p.x << 16) >> 16, int(p.x) >> 16, int(p.y << 16) >> 16, int(p.y) >> 16);
    } else {
      v = __ldg(reinterpret_cast<const int4*>(row) + c);
    }
    nodes[k] = v;
  }
}

// ---- incremental update of a few keys (decode appends)
//
// Rows [lo, hi) of K changed. Every level-1 row over them moves by delta(k) = K[2k] + K[2k+1]
// - stored row (the stored row is the old pair sum, so no old key is needed), and every
// ancestor at level l moves by the sum of the deltas of the level-1 rows beneath it. One CTA
// per (b,h): the deltas go to shared memory first (reading the old level-1 rows), then every
// affected row of every level is read, moved and written once, with the (level, row, column)
// items of all levels in one flat index space so that their loads are independent.
constexpr int kDeltaMaxKeys = 64;  // larger ranges are rebuilt chunk by chunk
constexpr int kDeltaThreads = 256;

template <int D>
__device__ __forceinline__ int4 ld_row4(const char* Th, const TreeLayout& tl, int l, int j, int c) {
  const char* row = Th + tl.offset_of(l) + (long long)j * tl.row_bytes(l);
  if (l <= tl.narrow) {
    const uint2 p = *(reinterpret_cast<const uint2*>(row) + c);
    return make_int4(int(p.x << 16) >> 16, int(p.x) >> 16, int(p.y << 16) >> 16, int(p.y) >> 16);
  }
  return *(reinterpret_cast<const int4*>(row) + c);
}

template <int D>
__device__ __forceinline__ void st_row4(char* Th, const TreeLayout& tl, int l, int j, int c,
                                        int4 v) {
  char* row = Th + tl.offset_of(l) + (long long)j * tl.row_bytes(l);
  if (l <= tl.narrow) {
    *(reinterpret_cast<uint2*>(row) + c) =
        make_uint2((unsigned(v.x) & 0xffffu) | (unsigned(v.y) << 16),
                   (unsigned(v.z) & 0xffffu) | (unsigned(v.w) << 16));
  } else {
    *(reinterpret_cast<int4*>(row) + c) = v;
  }
}

template <int D>
__global__ void __launch_bounds__(kDeltaThreads)
    tree_delta_kernel(const int8_t* __restrict__ K, char* __restrict__ tree, const TreeLayout tl,
                      int lo, int hi, int value_bound, uint32_t* dev_err) {
  constexpr int Q4 = D / 4;
  __shared__ int4 delta[(kDeltaMaxKeys / 2 + 1) * Q4];
  const long long bh = blockIdx.x;
  const int n = tl.n;
  char* Th = tree + bh * tl.block_bytes;
  const int8_t* Kh = K + bh * (long long)n * D;
  const int k0 = lo >> 1, k1 = (hi - 1) >> 1;  // level-1 rows over [lo, hi)
  const int span = k1 - k0 + 1;

  bool bad = false;
  for (int t = threadIdx.x; t < span * Q4; t += kDeltaThreads) {
    const int kk = t / Q4, c = t - kk * Q4;
    const int k = k0 + kk;
    const int a = __ldg(reinterpret_cast<const int*>(Kh + (long long)(2 * k) * D) + c);
    const int b = __ldg(reinterpret_cast<const int*>(Kh + (long long)(2 * k + 1) * D) + c);
    const int4 va = make_int4((a << 24) >> 24, (a << 16) >> 24, (a << 8) >> 24, a >> 24);
    const int4 vb = make_int4((b << 24) >> 24, (b << 16) >> 24, (b << 8) >> 24, b >> 24);
    const bool in_a = 2 * k >= lo && 2 * k < hi, in_b = 2 * k + 1 >= lo && 2 * k + 1 < hi;
    if (in_a) bad |= va.x > value_bound | va.x < -value_bound | va.y > value_bound |
                     va.y < -value_bound | va.z > value_bound | va.z < -value_bound |
                     va.w > value_bound | va.w < -value_bound;
    if (in_b) bad |= vb.x > value_bound | vb.x < -value_bound | vb.y > value_bound |
                     vb.y < -value_bound | vb.z > value_bound | vb.z < -value_bound |
                     vb.w > value_bound | vb.w < -value_bound;
    const int4 old = ld_row4<D>(Th, tl, 1, k, c);
    delta[t] = make_int4(va.x + vb.x - old.x, va.y + vb.y - old.y, va.z + vb.z - old.z,
                         va.w + vb.w - old.w);
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0 && dev_err)
    atomicOr(dev_err, ALHR_DEVERR_VALUE_RANGE);

  int total = 0;
  for (int l = 1; l <= tl.L; ++l) total += (((hi - 1) >> l) - (lo >> l) + 1) * Q4;
  // kPer items per thread per round: all their rows are loaded before any is written back
  // (items are disjoint rows/columns), so one round costs one memory round trip
  constexpr int kPer = 4;
  for (int f0 = 0; f0 < total; f0 += kPer * kDeltaThreads) {
    int lv[kPer], jv[kPer], cv[kPer];
    int4 acc[kPer];
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      const int f = f0 + u * kDeltaThreads + threadIdx.x;
      lv[u] = 0;
      if (f < total) {
        int l = 1, g = f;
        for (;;) {  // level of flat item f
          const int items = (((hi - 1) >> l) - (lo >> l) + 1) * Q4;
          if (g < items) break;
          g -= items;
          ++l;
        }
        const int jj = g / Q4;
        lv[u] = l;
        jv[u] = (lo >> l) + jj;
        cv[u] = g - jj * Q4;
        acc[u] = ld_row4<D>(Th, tl, l, jv[u], cv[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < kPer; ++u) {
      if (lv[u] == 0) continue;
      const int l = lv[u], j = jv[u], c = cv[u];
      // level-1 rows beneath node (l, j), clipped to the updated span
      const int s0 = max(j << (l - 1), k0) - k0;
      const int s1 = min(((j + 1) << (l - 1)) - 1, k1) - k0;
      for (int s = s0; s <= s1; ++s) {
        const int4 dv = delta[s * Q4 + c];
        acc[u].x += dv.x;
        acc[u].y += dv.y;
        acc[u].z += dv.z;
        acc[u].w += dv.w;
      }
      st_row4<D>(Th, tl, l, j, c, acc[u]);
    }
  }
}

// Levels lin+1 .. of the chunks covering keys [lo, hi) (all of them for [0, n)).
template <int D>
cudaError_t build_tree_d(const int8_t* K, char* tree, const TreeLayout& tl, long long bh,
                         int lo, int hi, int value_bound, uint32_t* dev_err, cudaStream_t st) {
  const int L = tl.L;
  const size_t smem_max = size_t(1 << kChunkLog) * D * sizeof(int);
  // the opt-in above 48 KB of dynamic shared memory is a per-device function attribute
  static thread_local bool configured[128] = {};  // per host thread: no shared state
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128 || !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(tree_chunk_kernel<D, kFromKeys>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tree_chunk_kernel<D, kFromNarrow>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(tree_chunk_kernel<D, kFromWide>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem_max));
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 128) configured[dev] = true;
  }
  const int stream_log =
      bh * (long long)(hi - lo) < kStreamSmallKeys ? kStreamLogSmall : kStreamLog;
  int lin = 0;
  while (lin < L) {
    const bool stream = lin == 0 && L >= kStreamP;
    const int mmax = stream ? stream_log : kChunkLog;
    const int m = (L - lin) < mmax ? (L - lin) : mmax;
    const int c0 = (lo >> lin) >> m, c1 = ((hi - 1) >> lin) >> m;
    const int chunks = c1 - c0 + 1;
    const long long grid = bh * chunks;
    const size_t smem = size_t(1 << m) * D * sizeof(int);
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (stream) {
      const long long threads = grid * (D / 4);
      const long long blocks = (threads + kTreeThreads - 1) / kTreeThreads;
      if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
      tree_stream_kernel<D, kStreamP><<<unsigned(blocks), kTreeThreads, 0, st>>>(
          K, tree, tl, m, c0, chunks, grid, value_bound, dev_err);
    } else if (lin == 0) {
      tree_chunk_kernel<D, kFromKeys><<<unsigned(grid), kTreeThreads, smem, st>>>(
          K, tree, tl, lin, m, c0, chunks, value_bound, dev_err);
    } else if (lin <= tl.narrow) {
      tree_chunk_kernel<D, kFromNarrow><<<unsigned(grid), kTreeThreads, smem, st>>>(
          K, tree, tl, lin, m, c0, chunks, value_bound, dev_err);
    } else {
      tree_chunk_kernel<D, kFromWide><<<unsigned(grid), kTreeThreads, smem, st>>>(
          K, tree, tl, lin, m, c0, chunks, value_bound, dev_err);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    lin += m;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_build_tree(const int8_t* K, char* tree, const TreeLayout& tl, long long bh,
                              int value_bound, uint32_t* dev_err, cudaStream_t st) {
  return tl.d == 64 ? build_tree_d<64>(K, tree, tl, bh, 0, tl.n, value_bound, dev_err, st)
                    : build_tree_d<128>(K, tree, tl, bh, 0, tl.n, value_bound, dev_err, st);
}

cudaError_t launch_update_tree(const int8_t* K, char* tree, const TreeLayout& tl, long long bh,
                               int lo, int hi, int value_bound, uint32_t* dev_err,
                               cudaStream_t st) {
  if (hi <= lo) return cudaSuccess;
  if (hi - lo > kDeltaMaxKeys)
    return tl.d == 64 ? build_tree_d<64>(K, tree, tl, bh, lo, hi, value_bound, dev_err, st)
                      : build_tree_d<128>(K, tree, tl, bh, lo, hi, value_bound, dev_err, st);
  if (bh > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  if (tl.d == 64)
    tree_delta_kernel<64><<<unsigned(bh), kDeltaThreads, 0, st>>>(K, tree, tl, lo, hi,
                                                                  value_bound, dev_err);
  else
    tree_delta_kernel<128><<<unsigned(bh), kDeltaThreads, 0, st>>>(K, tree, tl, lo, hi,
                                                                   value_bound, dev_err);
  return cudaGetLastError();
}

// The inverse of tree_unpack_kernel: plain level-major int32 rows [bh][n-1][d] into the tree
// layout (int16 rows for the narrow levels). A value of a narrow level outside
// [-vb * 2^l, vb * 2^l] cannot be the sum of 2^l keys within the value bound: it is saturated to
// int16 and flags ALHR_DEVERR_VALUE_RANGE.
template <int D>
__global__ void __launch_bounds__(256)
    tree_pack_kernel(const int4* __restrict__ nodes, const TreeLayout tl, long long bh, int vb,
                     char* __restrict__ tree, uint32_t* dev_err) {
  constexpr int Q4 = D / 4;
  const int n = tl.n;
  const long long per_block = (long long)(n - 1) * Q4;
  const long long total = bh * per_block;
  bool bad = false;
  for (long long k = blockIdx.x * (long long)blockDim.x + threadIdx.x; k < total;
       k += (long long)gridDim.x * blockDim.x) {
    const long long b = k / per_block;
    const long long rem = k - b * per_block;
    const int r = int(rem / Q4), c = int(rem - (long long)r * Q4);
    int l = 1;
    while (l < tl.L && r >= n - (n >> l)) ++l;  // level l holds rows [n - (n>>(l-1)), n - (n>>l))
    const int j = r - (n - (n >> (l - 1)));
    char* row = tree + b * tl.block_bytes + tl.level_off[l] + (long long)j * tl.row_bytes(l);
    const int4 v = __ldg(nodes + k);
    if (l <= tl.narrow) {
      const int lim = vb << l;  // <= 32767 on a narrow level
      const int e[4] = {v.x, v.y, v.z, v.w};
      unsigned h[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        bad |= e[t] > lim || e[t] < -lim;
        h[t] = unsigned(min(max(e[t], -32768), 32767)) & 0xffffu;
      }
      reinterpret_cast<uint2*>(row)[c] = make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
    } else {
      reinterpret_cast<int4*>(row)[c] = v;
    }
  }
  if (bad && dev_err) atomicOr(dev_err, ALHR_DEVERR_VALUE_RANGE);
}

cudaError_t launch_tree_pack(const int32_t* nodes, const TreeLayout& tl, long long bh, int vb,
                             char* tree, uint32_t* dev_err, cudaStream_t st) {
  const long long total = bh * (long long)(tl.n - 1) * (tl.d / 4);
  long long blocks = (total + 255) / 256;
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  if (blocks < 1) return cudaSuccess;
  const int4* src = reinterpret_cast<const int4*>(nodes);
  if (tl.d == 64)
    tree_pack_kernel<64><<<unsigned(blocks), 256, 0, st>>>(src, tl, bh, vb, tree, dev_err);
  else
    tree_pack_kernel<128><<<unsigned(blocks), 256, 0, st>>>(src, tl, bh, vb, tree, dev_err);
  return cudaGetLastError();
}

cudaError_t launch_tree_unpack(const char* tree, const TreeLayout& tl, long long bh,
                               int32_t* nodes, cudaStream_t st) {
  const long long total = bh * (long long)(tl.n - 1) * (tl.d / 4);
  long long blocks = (total + 255) / 256;
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  if (blocks < 1) return cudaSuccess;
  if (tl.d == 64)
    tree_unpack_kernel<64><<<unsigned(blocks), 256, 0, st>>>(tree, tl, bh,
                                                             reinterpret_cast<int4*>(nodes));
  else
    tree_unpack_kernel<128><<<unsigned(blocks), 256, 0, st>>>(tree, tl, bh,
                                                              reinterpret_cast<int4*>(nodes));
  return cudaGetLastError();
}

}  // namespace alhr
