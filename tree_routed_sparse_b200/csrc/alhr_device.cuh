// alhr_device.cuh -- device building blocks of the warp-per-query ALHR path (sm_100a).
//
// One warp owns one query. Lane l owns dims [l*DPL, (l+1)*DPL) of every d-wide row (DPL = d/32),
// so every row the warp reads is one coalesced access of d (keys), 2d (values) or 4d (tree
// sums) bytes. Scores of up to R rows are finished together by a transposed butterfly (one
// shuffle per row instead of five). The frontier and the candidates of the descent live in a
// per-warp shared-memory buffer.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/alhr.h"

namespace alhr {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxKeys = 96;        // 32 budget classes x 3 keys
constexpr int kMaxFrontier = 96;    // r <= max_keys - 1 nodes survive a step
constexpr int kMaxCand = 192;       // a step offers at most 2 r candidates
constexpr int kCandSlots = kMaxCand / 32;
constexpr int kFrontSlots = kMaxFrontier / 32;
constexpr int kWarps = 8;           // queries in flight per CTA

// Node descriptor: (start << 5) | level; the node covers keys [start, start + 2^level).
__device__ __forceinline__ int desc_level(int desc) { return desc & 31; }
__device__ __forceinline__ int desc_start(int desc) { return desc >> 5; }
__device__ __forceinline__ int make_desc(int start, int level) { return (start << 5) | level; }

// First row of tree level `level` (>= 1) in the level-major layout of one (b,h).
__device__ __forceinline__ long long level_row(int n, int level) {
  return (long long)n - (long long)(n >> (level - 1));
}

struct QueryArgs {
  int n, L, q_start, nq, window, max_keys, value_bound;
  long long num_queries;  // batch * heads * nq
  float scale;            // fl32(1/sqrt(d))
  const int8_t* Q;
  const int8_t* K;
  const uint16_t* V;
  const int32_t* nodes;
  const int8_t* W;
  const int32_t* budget_in;  // budget override / route input (nullable)
  const int32_t* idx_in;     // attend input
  const int32_t* count_in;   // attend input
  float* out;
  int32_t* idx_out;
  int32_t* count_out;
  int32_t* exp_out;
  int32_t* budget_out;
  uint32_t* dev_err;
};

// ------------------------------------------------------------------ per-lane row loads

// DPL int8 values of a key row (or a query row) at lane `lane`, sign-extended.
template <int DPL>
__device__ __forceinline__ void load_i8(const int8_t* row, int lane, int (&v)[DPL]) {
  if constexpr (DPL == 2) {
    const int t = __ldg(reinterpret_cast<const short*>(row) + lane);
    v[0] = (t << 24) >> 24;
    v[1] = (t << 16) >> 24;
  } else {
    const int t = __ldg(reinterpret_cast<const int*>(row) + lane);
    v[0] = (t << 24) >> 24;
    v[1] = (t << 16) >> 24;
    v[2] = (t << 8) >> 24;
    v[3] = t >> 24;
  }
}

// DPL int32 values of a tree row at lane `lane`.
template <int DPL>
__device__ __forceinline__ void load_i32(const int32_t* row, int lane, int (&v)[DPL]) {
  if constexpr (DPL == 2) {
    const int2 t = __ldg(reinterpret_cast<const int2*>(row) + lane);
    v[0] = t.x;
    v[1] = t.y;
  } else {
    const int4 t = __ldg(reinterpret_cast<const int4*>(row) + lane);
    v[0] = t.x;
    v[1] = t.y;
    v[2] = t.z;
    v[3] = t.w;
  }
}

// DPL bf16 values of a value row at lane `lane`, as floats (bf16 -> f32 is exact).
template <int DPL>
__device__ __forceinline__ void load_bf16(const uint16_t* row, int lane, float (&v)[DPL]) {
  if constexpr (DPL == 2) {
    const unsigned t = __ldg(reinterpret_cast<const unsigned*>(row) + lane);
    v[0] = __uint_as_float(t << 16);
    v[1] = __uint_as_float(t & 0xffff0000u);
  } else {
    const uint2 t = __ldg(reinterpret_cast<const uint2*>(row) + lane);
    v[0] = __uint_as_float(t.x << 16);
    v[1] = __uint_as_float(t.x & 0xffff0000u);
    v[2] = __uint_as_float(t.y << 16);
    v[3] = __uint_as_float(t.y & 0xffff0000u);
  }
}

// Row (level, j) of one head: a key row (level 0) or a stored tree sum (level >= 1).
template <int DPL>
__device__ __forceinline__ void load_node(const int8_t* Kh, const int32_t* Nh, int n, int level,
                                          int j, int lane, int (&v)[DPL]) {
  constexpr int D = 32 * DPL;
  if (level == 0) {
    load_i8<DPL>(Kh + (long long)j * D, lane, v);
  } else {
    load_i32<DPL>(Nh + (level_row(n, level) + j) * D, lane, v);
  }
}

template <typename S, int DPL>
__device__ __forceinline__ S lane_dot(const int (&q)[DPL], const int (&v)[DPL]) {
  S s = 0;
#pragma unroll
  for (int e = 0; e < DPL; ++e) s += S(q[e]) * S(v[e]);
  return s;
}

// Transposed butterfly: lane x returns the warp-wide sum of v[x % R].
template <typename S, int R>
__device__ __forceinline__ S transpose_reduce(S (&v)[R], int lane) {
#pragma unroll
  for (int h = R / 2; h >= 1; h /= 2) {
    const bool up = (lane & h) != 0;
#pragma unroll
    for (int j = 0; j < h; ++j) {
      const S keep = up ? v[j + h] : v[j];
      const S send = up ? v[j] : v[j + h];
      v[j] = keep + __shfl_xor_sync(kFull, send, h);
    }
  }
#pragma unroll
  for (int off = R; off < 32; off *= 2) v[0] += __shfl_xor_sync(kFull, v[0], off);
  return v[0];
}

template <typename S>
__device__ __forceinline__ S warp_min(S x) {
#pragma unroll
  for (int off = 16; off >= 1; off /= 2) {
    const S y = __shfl_xor_sync(kFull, x, off);
    x = y < x ? y : x;
  }
  return x;
}

template <typename S>
__device__ __forceinline__ S warp_max(S x) {
#pragma unroll
  for (int off = 16; off >= 1; off /= 2) {
    const S y = __shfl_xor_sync(kFull, x, off);
    x = y > x ? y : x;
  }
  return x;
}

__device__ __forceinline__ float warp_maxf(float x) {
#pragma unroll
  for (int off = 16; off >= 1; off /= 2) x = fmaxf(x, __shfl_xor_sync(kFull, x, off));
  return x;
}

__device__ __forceinline__ float warp_sumf(float x) {
#pragma unroll
  for (int off = 16; off >= 1; off /= 2) x += __shfl_xor_sync(kFull, x, off);
  return x;
}

__device__ __forceinline__ int warp_count(bool p) { return __popc(__ballot_sync(kFull, p)); }

__device__ __forceinline__ unsigned lanemask_lt(int lane) { return (1u << lane) - 1u; }

__device__ __forceinline__ void flag(uint32_t* dev_err, unsigned bit) {
  if (dev_err) atomicOr(dev_err, bit);
}

template <typename S>
struct ScoreLimits;
template <>
struct ScoreLimits<int> {
  static constexpr int lowest = -2147483647 - 1;
  static constexpr int highest = 2147483647;
};
template <>
struct ScoreLimits<long long> {
  static constexpr long long lowest = -9223372036854775807LL - 1;
  static constexpr long long highest = 9223372036854775807LL;
};

// Per-warp scratch of the descent (shared memory).
template <typename S>
struct WarpBuf {
  int cdesc[kMaxCand];
  S cscore[kMaxCand];
  int xdesc[kMaxFrontier];
  S xscore[kMaxFrontier];
};

// ------------------------------------------------------------------ top-r selection
//
// Keeps, among the C candidates in buf (C > r), the r with the largest score, ties to the lower
// start, and packs them into buf[0, r). Exact: the r-th largest score T is found by bisection on
// the integer score, then the candidates tied at T are cut by bisection on their start.
template <typename S>
__device__ __forceinline__ void select_top_r(WarpBuf<S>& B, int C, int r, int lane) {
  constexpr S kLow = ScoreLimits<S>::lowest;
  S sc[kCandSlots];
  int ds[kCandSlots];
  __syncwarp();
#pragma unroll
  for (int s = 0; s < kCandSlots; ++s) {
    const int e = lane + 32 * s;
    const bool ok = e < C;
    sc[s] = ok ? B.cscore[e] : kLow;
    ds[s] = ok ? B.cdesc[e] : 0;
  }
  S lo, hi;
  {
    S mn = ScoreLimits<S>::highest, mx = kLow;
#pragma unroll
    for (int s = 0; s < kCandSlots; ++s) {
      if (sc[s] != kLow) {
        mn = sc[s] < mn ? sc[s] : mn;
        mx = sc[s] > mx ? sc[s] : mx;
      }
    }
    lo = warp_min<S>(mn);
    hi = warp_max<S>(mx);
  }
  // largest T with #{score >= T} >= r
  for (int guard = 0; guard < 70 && lo < hi; ++guard) {
    const S mid = S((long long)lo + (((long long)hi - (long long)lo + 1) >> 1));
    int c = 0;
#pragma unroll
    for (int s = 0; s < kCandSlots; ++s) c += sc[s] >= mid ? 1 : 0;
    c = __reduce_add_sync(kFull, c);
    if (c >= r) lo = mid; else hi = mid - 1;
  }
  const S T = lo;
  int gt = 0, eq = 0;
#pragma unroll
  for (int s = 0; s < kCandSlots; ++s) {
    gt += sc[s] > T ? 1 : 0;
    eq += sc[s] == T ? 1 : 0;
  }
  gt = __reduce_add_sync(kFull, gt);
  eq = __reduce_add_sync(kFull, eq);
  const int need = r - gt;
  int U = 0x7fffffff;
  if (need < eq) {
    // smallest U with #{score == T and start <= U} >= need
    int lo2 = 0, hi2 = 0x7fffffff;
    for (int guard = 0; guard < 34 && lo2 < hi2; ++guard) {
      const int mid = lo2 + ((hi2 - lo2) >> 1);
      int c = 0;
#pragma unroll
      for (int s = 0; s < kCandSlots; ++s) c += (sc[s] == T && desc_start(ds[s]) <= mid) ? 1 : 0;
      c = __reduce_add_sync(kFull, c);
      if (c >= need) hi2 = mid; else lo2 = mid + 1;
    }
    U = lo2;
  }
  __syncwarp();
  int base = 0;
#pragma unroll
  for (int s = 0; s < kCandSlots; ++s) {
    const bool keep = sc[s] != kLow && (sc[s] > T || (sc[s] == T && desc_start(ds[s]) <= U));
    const unsigned bal = __ballot_sync(kFull, keep);
    if (keep) {
      const int pos = base + __popc(bal & lanemask_lt(lane));
      B.cdesc[pos] = ds[s];
      B.cscore[pos] = sc[s];
    }
    base += __popc(bal);
  }
  __syncwarp();
}

}  // namespace alhr
