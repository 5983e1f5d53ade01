// tree_layout.h -- byte layout of one (b,h) block of the key tree (host and device).
//
// Levels 1 .. log2 n follow each other in increasing order; level l holds n >> l rows, row j
// being the exact sum of keys [j*2^l, (j+1)*2^l). A level whose sums are bounded by
// value_bound * 2^l <= 32767 ("narrow") is stored, at d = 128, as int16 rows of 2d bytes, every
// level above (and every level at d = 64) as int32 rows of 4d bytes. Narrow levels are the
// lowest ones, which hold almost every row and take almost every read of the descent, so at
// d = 128 the tree and its reads shrink by nearly half while every stored sum stays exact.
#pragma once

#include <cstdint>

namespace alhr {

constexpr int kMaxLevels = 20;  // n <= 2^20

struct TreeLayout {
  int n, d, L;
  int narrow;                           // levels 1 .. narrow are int16
  long long block_bytes;                // bytes of one (b,h) block
  long long level_off[kMaxLevels + 2];  // byte offset of level l inside a block (index l >= 1)

  __host__ __device__ __forceinline__ int row_bytes(int level) const {
    return level <= narrow ? 2 * d : 4 * d;
  }
  // Byte offset of level l (>= 1), in closed form (no table lookup: lanes of a warp ask for
  // different levels at once): levels 1 .. l-1 hold n - (n >> (l-1)) rows, the first
  // n - (n >> narrow) of them narrow.
  __host__ __device__ __forceinline__ long long offset_of(int level) const {
    const long long before = (long long)n - (long long)(n >> (level - 1));
    const long long nar = (long long)n - (long long)(n >> narrow);
    return level - 1 <= narrow ? before * 2 * d : nar * 2 * d + (before - nar) * 4 * d;
  }
  // Byte offset of row j of level l inside a block, in 32-bit arithmetic (a block is < 2^30
  // bytes: at most (2^20 - 1) rows of 512 bytes).
  __host__ __device__ __forceinline__ int row_offset(int level, int j) const {
    const int before = n - (n >> (level - 1));
    const int nar = n - (n >> narrow);
    const int off = level - 1 <= narrow ? before * 2 * d : nar * 2 * d + (before - nar) * 4 * d;
    return off + j * row_bytes(level);
  }
};

// value_bound 0 means 16. n must be a power of two in [2, 2^20]; checked by the callers.
__host__ __device__ inline TreeLayout make_tree_layout(int n, int d, int value_bound) {
  TreeLayout t{};
  const long long vb = value_bound == 0 ? 16 : value_bound;
  t.n = n;
  t.d = d;
  int L = 0;
  while ((1 << L) < n) ++L;
  t.L = L;
  // int16 levels are used at d = 128, where the bytes of a row dominate a descent step; at
  // d = 64 the step is bound by instruction issue and latency, and int32 rows measured faster
  int narrow = 0;
  if (d == 128)
    while (narrow < L && (vb << (narrow + 1)) <= 32767) ++narrow;
  t.narrow = narrow;
  long long off = 0;
  t.level_off[0] = 0;
  for (int l = 1; l <= L; ++l) {
    t.level_off[l] = off;
    off += (long long)(n >> l) * t.row_bytes(l);
  }
  for (int l = L + 1; l < kMaxLevels + 2; ++l) t.level_off[l] = off;
  t.block_bytes = off;
  return t;
}

}  // namespace alhr
