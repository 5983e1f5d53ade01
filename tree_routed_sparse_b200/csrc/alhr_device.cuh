// alhr_device.cuh -- device building blocks of the warp-per-query ALHR path (sm_100a).
//
// One warp owns one query. Rows are scored in "row groups": TPR = d/16 consecutive lanes share a
// row and each lane holds 16 of its dims (see the row-group layout below), so one warp pass
// scores RPI = 32/TPR rows (8 at d=64, 4 at d=128): an int32 tree row is two 32-byte loads and
// 16 multiply-adds per lane, an int16 tree row 8 dp2a, a key row four dp4a, and a row score
// costs log2(TPR) shuffles. The value rows of the final weighted sum use value groups instead:
// d/8 lanes share a value row, one 16-byte load of 8 bf16 each. The frontier and the
// candidates of the descent live in a per-warp shared-memory buffer.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/alhr.h"
#include "tree_layout.h"

namespace alhr {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kMaxKeys = 96;        // 32 budget classes x 3 keys
constexpr int kMaxFrontier = 96;    // r <= max_keys - 1 nodes survive a step
constexpr int kMaxCand = 192;       // a step offers at most 2 r candidates
constexpr int kMaxWindow = 32;      // the largest neighbour window the kernels accept
constexpr int kFrontSlots = kMaxFrontier / 32;
constexpr int kWarps = 8;           // warps (queries) per CTA of the unfused attention kernel

template <int D>
struct Lay {
  static constexpr int TPR = D / 16;    // lanes per row in the row-group layout
  static constexpr int RPI = 32 / TPR;  // rows per warp pass
  static constexpr int DPL = D / 32;    // dims per lane in the value layout
};

// Node descriptor: (start << 5) | level; the node covers keys [start, start + 2^level).
__device__ __forceinline__ int desc_level(int desc) { return desc & 31; }
__device__ __forceinline__ int desc_start(int desc) { return (desc >> 5) & 0xFFFFF; }
__device__ __forceinline__ int make_desc(int start, int level) { return (start << 5) | level; }

// First row of tree level `level` (>= 1) in the level-major layout of one (b,h).
__device__ __forceinline__ long long level_row(int n, int level) {
  return (long long)n - (long long)(n >> (level - 1));
}

struct QueryArgs {
  int n, L, q_start, nq, window, max_keys, value_bound;
  int norm_l;  // 0: rank candidates by q . node_sum; L: by q . node_sum << (L - level) (means)
  int bucket;  // leaf bucket level: nodes of level <= bucket are not expanded (0: keys)
  long long num_queries;  // batch * heads * nq
  float scale;            // fl32(1/sqrt(d))
  const int8_t* Q;
  const int8_t* K;
  const uint16_t* V;
  const char* tree;          // key tree, one block of tl.block_bytes per (b,h)
  TreeLayout tl;
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

__device__ __forceinline__ int sx8(int w, int byte) { return (w << (24 - 8 * byte)) >> 24; }

// A warp's walk over the flat query index qi = bh * nq + r in steps of `stride`, keeping
// (bh, r) up to date with one division at the start instead of one per query.
struct QueryCursor {
  long long qi, bh, step_bh;
  int r, step_r;
  __device__ __forceinline__ QueryCursor(long long first, int nq, long long stride) {
    qi = first;
    bh = first / nq;
    r = int(first - bh * nq);
    step_bh = stride / nq;
    step_r = int(stride - step_bh * nq);
  }
  __device__ __forceinline__ void advance(long long stride, int nq) {
    qi += stride;
    bh += step_bh;
    r += step_r;  // r, step_r < nq, so one carry at most
    if (r >= nq) {
      r -= nq;
      ++bh;
    }
  }
};

// Byte offset of row j of tree level l (>= 1) inside a block of the layout of tree_layout.h,
// from scalars only (levels 1 .. l-1 hold n - (n >> (l-1)) rows, the first n - (n >> narrow) of
// them int16 rows of 2d bytes, the rest int32 rows of 4d bytes).
template <int D>
__device__ __forceinline__ int tree_row_offset(int n, int narrow, int level, int j) {
  const int before = n - (n >> (level - 1));
  if (narrow == 0) return (before + j) * 4 * D;
  const int nar = n - (n >> narrow);
  const bool is_narrow = level <= narrow;
  const int off = is_narrow ? before * 2 * D : nar * 2 * D + (before - nar) * 4 * D;
  return off + j * (is_narrow ? 2 * D : 4 * D);
}

// The row-group layout, shared by every row kind (TPR = d/16 lanes per row, sub = lane % TPR):
// at d = 128 lane `sub` holds the 16 consecutive dims 16*sub .. 16*sub+15 of a row; at d = 64
// it holds the two 8-dim chunks 8c .. 8c+7, c = sub and sub + TPR. Either way the lane's dims
// come as four 4-dim words j = 0..3 (dims 4j .. 4j+3 of the lane's 16). Consecutive dims mean
// fewer, wider loads (one 32-byte load for an int16 row, one 16-byte load for a key row);
// chunks measured faster at d = 64, where they keep the fused kernel within its registers.
template <int D>
constexpr bool kBlockLayout = (D == 128);

// The query in the row-group layout (qp: the lane's four packed words, for dp4a against key
// rows and dp2a against int16 rows; qn: the same 16 values sign-extended, qn[4j + e] = dim e of
// word j, for int32 rows).
struct RowQ {
  int qp[4];
  int qn[16];
};

// 32 bytes from global memory in one load (sm_100; p 32-byte aligned).
__device__ __forceinline__ void ldg32B(const void* p, int (&w)[8]) {
  asm volatile("ld.global.nc.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]),
                 "=r"(w[6]), "=r"(w[7])
               : "l"(p));
}

// The lane's four words of an int8 row (a query or a key): one 16-byte load (d = 128) or two
// 8-byte loads (d = 64).
template <int D>
__device__ __forceinline__ void ld_bytes16(const int8_t* row, int sub, int (&w)[4]) {
  constexpr int TPR = Lay<D>::TPR;
  if constexpr (kBlockLayout<D>) {
    const int4 t = __ldg(reinterpret_cast<const int4*>(row) + sub);
    w[0] = t.x;
    w[1] = t.y;
    w[2] = t.z;
    w[3] = t.w;
  } else {
    const int2* p = reinterpret_cast<const int2*>(row) + sub;
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int2 t = __ldg(p + TPR * v);
      w[2 * v] = t.x;
      w[2 * v + 1] = t.y;
    }
  }
}

template <int D>
__device__ __forceinline__ void load_rowq(const int8_t* qrow, int sub, RowQ& q) {
  ld_bytes16<D>(qrow, sub, q.qp);
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) q.qn[4 * j + e] = sx8(q.qp[j], e);
}

// An int16 tree row (2d bytes) in its row-group layout: 8 words of two int16 each, word k
// holding dims 2k, 2k+1 of the lane's 16 (one 32-byte load at d = 128, two 16-byte loads at
// d = 64; rows are 32-byte aligned: the tree buffer is, and every row is a multiple of 256 bytes).
template <int D>
__device__ __forceinline__ void ld_tree16(const char* row, int sub, int (&w)[8]) {
  constexpr int TPR = Lay<D>::TPR;
  if constexpr (kBlockLayout<D>) {
    ldg32B(row + 32 * sub, w);
  } else {
    const int4* p = reinterpret_cast<const int4*>(row) + sub;
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const int4 t = __ldg(p + TPR * v);
      w[4 * v + 0] = t.x;
      w[4 * v + 1] = t.y;
      w[4 * v + 2] = t.z;
      w[4 * v + 3] = t.w;
    }
  }
}

// q . row over the lane's 16 dims of an int16 row: 8 two-way int16 x int8 dot products.
__device__ __forceinline__ int dot_tree16(const RowQ& q, const int (&w)[8]) {
  int s = 0;
  // two independent accumulator chains (the intrinsic is not reassociated by the compiler)
  int t = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    s = __dp2a_lo(w[2 * j], q.qp[j], s);
    t = __dp2a_hi(w[2 * j + 1], q.qp[j], t);
  }
  s += t;
  return s;
}

// An int16 tree row widened to the lane's 16 int32 values; used where rows of different widths
// are summed (the causal key sum).
template <int D>
__device__ __forceinline__ void ld_tree16_as32(const char* row, int sub, int (&x)[16]) {
  int w[8];
  ld_tree16<D>(row, sub, w);
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x[2 * k] = (w[k] << 16) >> 16;
    x[2 * k + 1] = w[k] >> 16;
  }
}

// A tree row (int32) in the row-group layout: two 32-byte loads per lane.
template <int D>
__device__ __forceinline__ void ld_tree(const char* row, int sub, int (&x)[16]) {
  constexpr int TPR = Lay<D>::TPR;
  int w0[8], w1[8];
  if constexpr (kBlockLayout<D>) {
    ldg32B(row + 64 * sub, w0);
    ldg32B(row + 64 * sub + 32, w1);
  } else {
    ldg32B(row + 32 * sub, w0);
    ldg32B(row + 32 * (sub + TPR), w1);
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x[k] = w0[k];
    x[8 + k] = w1[k];
  }
}

// A key row (int8) in the row-group layout, as the lane's four packed words.
template <int D>
__device__ __forceinline__ void ld_key(const int8_t* row, int sub, int (&xp)[4]) {
  ld_bytes16<D>(row, sub, xp);
}

// Slot of word m (dims 4m .. 4m+3) of a predictor weight row in shared memory, and the slot of
// word j of the lane `sub`: words are grouped by their position in the lane's 16 dims, so the
// lanes of a row group read consecutive slots.
template <int D>
__device__ __forceinline__ int w_slot(int m) {
  return kBlockLayout<D> ? (m & 3) * (D / 16) + (m >> 2) : (m & 1) * (D / 8) + (m >> 1);
}
template <int D>
__device__ __forceinline__ int w_lane_slot(int sub, int j) {
  constexpr int TPR = Lay<D>::TPR;
  return kBlockLayout<D> ? j * (D / 16) + sub : (j & 1) * (D / 8) + sub + TPR * (j >> 1);
}

template <typename S>
__device__ __forceinline__ S dot_tree(const RowQ& q, const int (&x)[16]) {
  S s = 0;
#pragma unroll
  for (int j = 0; j < 16; ++j) s += S(q.qn[j]) * S(x[j]);
  return s;
}

__device__ __forceinline__ int dot_key(const RowQ& q, const int (&xp)[4]) {
  int s = 0;
#pragma unroll
  for (int v = 0; v < 4; ++v) s = __dp4a(xp[v], q.qp[v], s);
  return s;
}

// Sum over the TPR lanes of a row group (every lane of the group gets the sum).
template <typename S, int TPR>
__device__ __forceinline__ S group_sum(S s) {
#pragma unroll
  for (int off = 1; off < TPR; off *= 2) s += __shfl_xor_sync(kFull, s, off);
  return s;
}

// DPL bf16 values of a value row in the value layout, as floats (bf16 -> f32 is exact).
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

// The softmax-weighted sum of the selected value rows, in value groups: VPR = d/8 lanes share
// a row (one 16-byte load of 8 bf16 per lane) and a warp pass covers KPP = 32/VPR rows, UV
// passes in flight. Keys and weights come from shared memory (selk/selp). The groups' partial
// sums are added by log2(KPP) shuffle stages and the first group writes the fp32 row, scaled
// by inv (the reciprocal of the softmax denominator).
template <int D, int UV>
__device__ __forceinline__ void gather_values(const int* selk, const float* selp, int count,
                                              float inv, const uint16_t* Vh, int lane,
                                              float* out_row) {
  constexpr int VPR = D / 8;
  constexpr int KPP = 32 / VPR;
  const int kg = lane / VPR;
  const int vs = lane % VPR;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int base = 0; base < count; base += UV * KPP) {
    uint4 raw[UV];
    float p[UV];
#pragma unroll
    for (int u = 0; u < UV; ++u) {
      // a value group past the end loads the last selected row again with weight 0
      const int k = base + u * KPP + kg;
      raw[u] = __ldg(reinterpret_cast<const uint4*>(Vh + (long long)selk[min(k, count - 1)] * D) + vs);
      p[u] = k < count ? selp[k] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < UV; ++u) {
      const unsigned w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[2 * j] = fmaf(p[u], __uint_as_float(w[j] << 16), acc[2 * j]);
        acc[2 * j + 1] = fmaf(p[u], __uint_as_float(w[j] & 0xffff0000u), acc[2 * j + 1]);
      }
    }
  }
#pragma unroll
  for (int off = VPR; off < 32; off *= 2)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(kFull, acc[j], off);
  if (lane < VPR) {
    float4* o = reinterpret_cast<float4*>(out_row + 8 * vs);
    o[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    o[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
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
template <>
__device__ __forceinline__ int warp_min<int>(int x) { return __reduce_min_sync(kFull, x); }

template <typename S>
__device__ __forceinline__ S warp_max(S x) {
#pragma unroll
  for (int off = 16; off >= 1; off /= 2) {
    const S y = __shfl_xor_sync(kFull, x, off);
    x = y > x ? y : x;
  }
  return x;
}
template <>
__device__ __forceinline__ int warp_max<int>(int x) { return __reduce_max_sync(kFull, x); }

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

// A node of the frontier or a candidate: its descriptor and its score.
template <typename S>
struct Cand {
  int desc;
  S score;
};

// N nodes in shared memory. With int32 scores each node is one 8-byte record, so one access
// moves both fields; with int64 scores descriptors and scores are kept apart (a 16-byte padded
// record measured slower).
template <typename S, int N>
struct CandArray {
  int d[N];
  S s[N];
  __device__ __forceinline__ Cand<S> get(int e) const { return Cand<S>{d[e], s[e]}; }
  __device__ __forceinline__ void put(int e, int desc, S score) {
    d[e] = desc;
    s[e] = score;
  }
  __device__ __forceinline__ int desc(int e) const { return d[e]; }
  __device__ __forceinline__ S score(int e) const { return s[e]; }
  __device__ __forceinline__ void set_desc(int e, int v) { d[e] = v; }
  __device__ __forceinline__ void set_score(int e, S v) { s[e] = v; }
};
template <int N>
struct CandArray<int, N> {
  int2 c[N];  // (desc, score)
  __device__ __forceinline__ Cand<int> get(int e) const {
    const int2 v = c[e];
    return Cand<int>{v.x, v.y};
  }
  __device__ __forceinline__ void put(int e, int desc, int score) { c[e] = make_int2(desc, score); }
  __device__ __forceinline__ int desc(int e) const { return c[e].x; }
  __device__ __forceinline__ int score(int e) const { return c[e].y; }
  __device__ __forceinline__ void set_desc(int e, int v) { c[e].x = v; }
  __device__ __forceinline__ void set_score(int e, int v) { c[e].y = v; }
};

// Per-warp scratch of one query (shared memory).
template <typename S>
struct WarpBuf {
  CandArray<S, kMaxCand> cand;       // frontier / candidates
  CandArray<S, kMaxFrontier> xnode;  // nodes expanded this step
  // The descent's per-step lists and the attention's staged selection are never live at the
  // same time (the selection is staged after the last step, and a barrier separates it from the
  // next query's descent), so they share storage: a smaller buffer leaves more of the SM's
  // unified shared memory / L1 to the cache.
  union {
    struct {
      int xrow[kMaxFrontier];  // byte offset of each expanded node's left child row (tree
                               // block or key rows of the head)
      S xleft[kMaxFrontier];   // score of that left child
    };
    struct {
      int selk[kMaxKeys];      // the selected keys and their softmax weights
      float selp[kMaxKeys];
    };
  };
  int plist[32];             // the roots of the descent forest, largest first
  int winsc[kMaxWindow + 4]; // scores of the window keys (+ a spare slot for idle row groups;
                             // padded so that the buffer stays a multiple of 16 bytes)
};
static_assert(sizeof(WarpBuf<int>) % 16 == 0 && sizeof(WarpBuf<long long>) % 16 == 0,
              "per-warp buffers keep 16-byte alignment");

// ------------------------------------------------------------------ top-r selection

template <int NS>
struct TieStarts {
  int v[NS];  // start of each tied candidate of this lane, INT_MAX for the others
};

// Smallest U with #{tied candidates with start <= U} >= need (starts are distinct). Ties at the
// threshold are rare, so this runs out of line and keeps the hot selection code small.
template <int NS>
__device__ __noinline__ int tie_cut(TieStarts<NS> ts, int need) {
  int lo2 = 0, hi2 = 1 << 20;
  for (int guard = 0; guard < 24 && lo2 < hi2; ++guard) {
    const int mid = lo2 + ((hi2 - lo2) >> 1);
    int c = 0;
#pragma unroll
    for (int s = 0; s < NS; ++s) c += ts.v[s] <= mid ? 1 : 0;
    c = __reduce_add_sync(kFull, c);
    if (c >= need) hi2 = mid; else lo2 = mid + 1;
  }
  return lo2;
}
// Upper midpoint of [lo, hi] (lo < hi), exact.
template <typename T>
__device__ __forceinline__ T upper_mid(T lo, T hi) {
  return T((long long)lo + (((long long)hi - (long long)lo + 1) >> 1));
}
// 32-bit scores: valid scores are above INT_MIN (the empty-slot mark), so hi - lo + 1 < 2^32
// and the unsigned difference is exact.
template <>
__device__ __forceinline__ int upper_mid<int>(int lo, int hi) {
  return lo + int((unsigned(hi) - unsigned(lo) + 1u) >> 1);
}

// The threshold of the top r among the lane's NS candidate scores (kLow marks an empty slot):
// the r-th largest score thr, and the cut on start positions among the candidates tied at thr
// (candidates with score thr and start <= cut are kept; cut = INT_MAX when no tie straddles).
// Exact: thr is found by bisection on the integer score; candidates tied at thr are then cut by
// bisection on their start position (starts are distinct).
template <typename T, int NS>
__device__ __forceinline__ void top_r_threshold(const T (&sc)[NS], const int (&ds)[NS], int r,
                                                T& thr, int& cut) {
  constexpr T kLow = ScoreLimits<T>::lowest;
  T mn = ScoreLimits<T>::highest, mx = kLow;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    if (sc[s] != kLow) {
      mn = sc[s] < mn ? sc[s] : mn;
      mx = sc[s] > mx ? sc[s] : mx;
    }
  }
  T lo = warp_min<T>(mn);
  T hi = warp_max<T>(mx);
  // Bisection for the largest T with #{score >= T} >= r. It stops as soon as a midpoint has
  // exactly r candidates at or above it: that set is the top r (nothing at or above the
  // midpoint is left out, so no tie can straddle the cut), which takes about log2(C) probes
  // instead of log2(score range).
  bool exact = false;
  for (int guard = 0; guard < 70 && lo < hi; ++guard) {
    const T mid = upper_mid<T>(lo, hi);
    int c = 0;
#pragma unroll
    for (int s = 0; s < NS; ++s) c += sc[s] >= mid ? 1 : 0;
    c = __reduce_add_sync(kFull, c);
    if (c == r) {
      lo = mid;
      exact = true;
      break;
    }
    if (c > r) lo = mid; else hi = mid - 1;
  }
  thr = lo;
  int need = 0, eq = 0;
  if (!exact) {
    int gt = 0;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      gt += sc[s] > lo ? 1 : 0;
      eq += sc[s] == lo ? 1 : 0;
    }
    gt = __reduce_add_sync(kFull, gt);
    eq = __reduce_add_sync(kFull, eq);
    need = r - gt;
  }
  cut = 0x7fffffff;
  if (!exact && need < eq) {
    TieStarts<NS> ts;
#pragma unroll
    for (int s = 0; s < NS; ++s) ts.v[s] = sc[s] == lo ? desc_start(ds[s]) : 0x7fffffff;
    cut = tie_cut<NS>(ts, need);
  }
}

// Which of the lane's NS candidates (score, descriptor; kLow marks an empty slot) are among the
// r with the largest score, ties to the lower start (r < the number of candidates). With 64-bit
// scores the threshold search runs on 32-bit copies whenever every candidate's score fits in 32
// bits (one vote per call; the same set either way).
template <typename S, int NS>
__device__ __forceinline__ void top_r_keep(const S (&sc)[NS], const int (&ds)[NS], int r,
                                           bool (&keep)[NS]) {
  constexpr S kLow = ScoreLimits<S>::lowest;
  bool narrow = false;
  if constexpr (sizeof(S) == 8) {
    bool fits = true;
#pragma unroll
    for (int s = 0; s < NS; ++s)
      fits &= sc[s] == kLow || (sc[s] > S(ScoreLimits<int>::lowest) &&
                                sc[s] <= S(ScoreLimits<int>::highest));
    narrow = __all_sync(kFull, fits);
  }
  if (narrow) {
    int s32[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) s32[s] = sc[s] == kLow ? ScoreLimits<int>::lowest : int(sc[s]);
    int thr, cut;
    top_r_threshold<int, NS>(s32, ds, r, thr, cut);
#pragma unroll
    for (int s = 0; s < NS; ++s)
      keep[s] = s32[s] != ScoreLimits<int>::lowest &&
                (s32[s] > thr || (s32[s] == thr && desc_start(ds[s]) <= cut));
  } else {
    S thr;
    int cut;
    top_r_threshold<S, NS>(sc, ds, r, thr, cut);
#pragma unroll
    for (int s = 0; s < NS; ++s)
      keep[s] = sc[s] != kLow && (sc[s] > thr || (sc[s] == thr && desc_start(ds[s]) <= cut));
  }
}

// Keeps, among the C candidates (r < C <= 32*NS), the r with the largest score, ties to the
// lower start, and packs them into the front of the buffer. With 64-bit scores the threshold
// search runs on 32-bit copies whenever every candidate's score fits in 32 bits (one vote per
// call; the same set either way).
template <typename S, int NS, bool NORM>
__device__ __forceinline__ void select_top_r_ns(WarpBuf<S>& B, int C, int r, int lane,
                                                int norm_l) {
  constexpr S kLow = ScoreLimits<S>::lowest;
  S sc[NS];
  int ds[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const int e = lane + 32 * s;
    const bool ok = e < C;
    Cand<S> cd{0, kLow};
    if (ok) cd = B.cand.get(e);
    sc[s] = cd.score;
    ds[s] = cd.desc;
    // ranking by means: q . sum / 2^level, scaled by 2^L to stay an exact integer
    if (NORM && norm_l && ok) sc[s] = sc[s] * (S(1) << (norm_l - desc_level(ds[s])));
  }
  bool keep[NS];
  top_r_keep<S, NS>(sc, ds, r, keep);
  __syncwarp();
  int base = 0;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const unsigned bal = __ballot_sync(kFull, keep[s]);
    if (keep[s]) {
      const int pos = base + __popc(bal & lanemask_lt(lane));
      B.cand.put(pos, ds[s],
                 (NORM && norm_l) ? S(sc[s] >> (norm_l - desc_level(ds[s]))) : sc[s]);
    }
    base += __popc(bal);
  }
  __syncwarp();
}

// NORM compiles in the ranking by means (norm_l != 0: scores scaled by 2^(norm_l - level)).
template <typename S, bool NORM>
__device__ __forceinline__ void select_top_r(WarpBuf<S>& B, int C, int r, int lane,
                                             int norm_l) {
  __syncwarp();
  // two instantiations only: the fused kernel is large enough that instruction-cache misses
  // cost more than the spare slot comparisons (measured)
  if (C <= 96) select_top_r_ns<S, 3, NORM>(B, C, r, lane, norm_l);
  else select_top_r_ns<S, 6, NORM>(B, C, r, lane, norm_l);
}

}  // namespace alhr
