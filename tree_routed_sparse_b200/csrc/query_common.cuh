// query_common.cuh -- pieces shared by the two shapes of the per-query kernels (sm_100a): the
// warp-per-query kernels of query_kernels.cu and the CTA-per-query kernels of
// cta_query_kernels.cu. Both follow the README of ALHR, section "Inference stage".
#pragma once

#include "alhr_device.cuh"

namespace alhr {

enum Mode : int { kForwardPredict = 0, kForwardOverride = 1, kRouteOnly = 2, kPredictOnly = 3 };

// Writes the two children of expanded node x (the node p; its left child's score `left`).
template <typename S>
__device__ __forceinline__ void put_children(WarpBuf<S>& B, int nl, int x, Cand<S> p, S left) {
  const int cl = desc_level(p.desc) - 1;
  const int st = desc_start(p.desc);
  const S ps = p.score;
  B.cand.put(nl + 2 * x, make_desc(st, cl), left);
  B.cand.put(nl + 2 * x + 1, make_desc(st + (1 << cl), cl), ps - left);
}

// Dynamic shared memory of a query kernel: the predictor weights (the G half widened to
// int32, then the q half as packed int8 words; within a class row the 4-dim words are stored
// grouped by their position in a lane's 16 dims, and rows are padded, so that the row groups,
// which read different classes at once, hit different banks) followed by one WarpBuf per
// warp.
template <int D>
struct WLayout {
  static constexpr int g_stride = D + 16;     // ints per class row of the G half
  static constexpr int q_stride = D / 4 + 4;  // words per class row of the q half
};
template <typename S, int D, int MODE>
struct QuerySmem {
  static constexpr bool kUsesW = (MODE == kForwardPredict || MODE == kPredictOnly);
  static constexpr size_t w_bytes =
      kUsesW ? size_t(32 * WLayout<D>::g_stride + 32 * WLayout<D>::q_stride) * 4 : 0;
  static constexpr size_t bytes_for(int warps) { return w_bytes + warps * sizeof(WarpBuf<S>); }
};

// Predictor weights into shared memory, in the layout of WLayout (all threads of the CTA take
// part; the caller synchronises before reading them). W is read as 16-byte pieces, every piece
// of a thread loaded before any is stored (one round trip to memory instead of one per word:
// this runs at the start of every CTA, so at decode it sits on the critical path).
template <int D>
__device__ __forceinline__ void stage_weights(const int8_t* W, int* sWg, int* sWq) {
  constexpr int GS = WLayout<D>::g_stride;
  constexpr int QS = WLayout<D>::q_stride;
  constexpr int kPieces = 32 * 2 * D / 16;  // 16-byte pieces of W [32][2d]
  constexpr int kPerThread = 8;             // pieces per thread per round (blockDim >= 128)
  const int4* W4 = reinterpret_cast<const int4*>(W);
  for (int base = 0; base < kPieces; base += kPerThread * blockDim.x) {
    int4 v[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int k = base + u * blockDim.x + threadIdx.x;
      if (k < kPieces) v[u] = __ldg(W4 + k);
    }
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int k = base + u * blockDim.x + threadIdx.x;
      if (k < kPieces) {
        const int c = k / (2 * D / 16);               // class row
        const int m0 = (k - c * (2 * D / 16)) * 4;    // first 4-byte word of the piece in the row
        const int wv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int m = m0 + j;  // words 0 .. D/4-1: the q half; D/4 .. D/2-1: the G half
          if (m < D / 4) {
            // word m (dims 4m .. 4m+3) goes to slot w_slot<D>(m), so that the lanes of a row
            // group read consecutive slots
            sWq[c * QS + w_slot<D>(m)] = wv[j];
          } else {
            // the G half, widened to int32: dims t = 4(m - D/4) .. +3
            const int t = 4 * (m - D / 4);
            int* g = sWg + c * GS + 4 * w_slot<D>(t >> 2);
#pragma unroll
            for (int e = 0; e < 4; ++e) g[e] = sx8(wv[j], e);
          }
        }
      }
    }
  }
}

// Logit of class c for the lane's 16 dims of q and G (the caller sums over the row group):
// W[c] . [q; G], int64.
template <int D>
__device__ __forceinline__ long long class_logit_part(const int* sWg, const int* sWq, int c, int sub,
                                                      const RowQ& q, const int (&G)[16]) {
  constexpr int GS = WLayout<D>::g_stride;
  constexpr int QS = WLayout<D>::q_stride;
  int sq = 0;
  long long sg = 0;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int m = w_lane_slot<D>(sub, v);  // slot of the lane's word v
    sq = __dp4a(sWq[c * QS + m], q.qp[v], sq);
    const int4 wg = *reinterpret_cast<const int4*>(sWg + c * GS + 4 * m);
    sg += (long long)wg.x * G[4 * v] + (long long)wg.y * G[4 * v + 1] +
          (long long)wg.z * G[4 * v + 2] + (long long)wg.w * G[4 * v + 3];
  }
  return sg + sq;
}

// Leaf buckets (descent variant): the kept nodes, all of level <= bucket, become the list of
// their keys, each scored q . k, in place of the frontier; returns the number of keys. At most
// r >> bucket nodes (< 64) and r keys (< 96). Out of line: only the bucket variant reaches it.
template <typename S, int D>
__device__ __noinline__ int expand_buckets(WarpBuf<S>& B, int nf, const int8_t* Kh, const RowQ q,
                                           int lane) {
  constexpr int TPR = Lay<D>::TPR;
  constexpr int RPI = Lay<D>::RPI;
  const int grp = lane / TPR, sub = lane % TPR;
  int total = 0;
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int e = lane + 32 * s;
    int sz = 0, st = 0;
    if (e < nf) {
      const int ds = B.cand.desc(e);
      sz = 1 << desc_level(ds);
      st = desc_start(ds);
    }
    int incl = sz;  // inclusive scan of the bucket sizes over the lanes
#pragma unroll
    for (int off = 1; off < 32; off *= 2) {
      const int y = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += y;
    }
    const int pos = total + incl - sz;
    for (int t = 0; t < sz; ++t) B.xrow[pos + t] = st + t;
    total += __shfl_sync(kFull, incl, 31);
  }
  __syncwarp();
  for (int base = 0; base < total; base += RPI) {
    const int k = base + grp;
    int xp[4] = {0, 0, 0, 0};
    if (k < total) ld_key<D>(Kh + (long long)B.xrow[k] * D, sub, xp);
    const int sc = group_sum<int, TPR>(dot_key(q, xp));
    if (k < total && sub == 0) {
      B.cand.put(k, make_desc(B.xrow[k], 0), S(sc));
    }
  }
  __syncwarp();
  return total;
}

// The selection in ascending order, -1 padded: the routed keys (all below the window) sorted by
// rank counting, then the window keys. Out of line: only the route outputs ask for it.
template <typename S>
__device__ __noinline__ void write_selection(const WarpBuf<S>& B, int nf, int nsel_win, int i,
                                             int32_t* io, int max_keys, int lane) {
#pragma unroll
  for (int s = 0; s < kFrontSlots; ++s) {
    const int e = lane + 32 * s;
    if (e < nf) {
      const int st = desc_start(B.cand.desc(e));
      int rank = 0;
      for (int f = 0; f < nf; ++f) rank += desc_start(B.cand.desc(f)) < st ? 1 : 0;
      io[rank] = st;
    }
  }
  if (lane < nsel_win) io[nf + nsel_win - 1 - lane] = i - lane;
  for (int pp = nf + nsel_win + lane; pp < max_keys; pp += 32) io[pp] = -1;
}

// Any node of the forest (a key at level 0, an int16 or int32 tree row above) as this lane's 16
// per-dimension integers; used by the latency mode's batched passes over causal-sum rows and roots.
template <int D, bool kNarrow>
__device__ __forceinline__ void ld_node32(const char* Th, const int8_t* Kh, int n, int narrow,
                                          int pd, int sub, int (&x)[16]) {
  const int lvl = desc_level(pd);
  const int st = desc_start(pd);
  if (lvl == 0) {
    int xp[4];
    ld_key<D>(Kh + (long long)st * D, sub, xp);
#pragma unroll
    for (int v = 0; v < 4; ++v)
#pragma unroll
      for (int e = 0; e < 4; ++e) x[4 * v + e] = sx8(xp[v], e);
  } else if (kNarrow && lvl <= narrow) {
    ld_tree16_as32<D>(Th + tree_row_offset<D>(n, narrow, lvl, st >> lvl), sub, x);
  } else {
    ld_tree<D>(Th + tree_row_offset<D>(n, narrow, lvl, st >> lvl), sub, x);
  }
}

// Counts of the classified lists of a step: keys (and buckets) in cand[0, nl); nodes to expand in
// the x lists, [0, nw) with int32 left-child rows, [nw, nw + nn) with int16 ones, then nk with
// keys as left children.
struct StepLists {
  int nl, nw, nn, nk;
};

// Warp 0's serial part of a descent step, in one pass over registers: the step's candidates
// (the frontier's keys cand[0, nl) and both children of every expanded node, the right child
// scored as parent - left), the best `limit` of them when there are more (exact top r, ties to
// the lower start; rank by means with NORM), and the kept ones written straight into the next
// step's classified lists. Returns the new counts.
template <typename S, int D, int NS, bool NORM>
__device__ __forceinline__ StepLists step_select_classify(WarpBuf<S>& B, int nl, int nx, int limit,
                                                          int lane, int norm_l, int bucket, int n,
                                                          int narrow) {
  constexpr S kLow = ScoreLimits<S>::lowest;
  constexpr bool kNarrow = (D == 128);
  const int C = nl + 2 * nx;
  S sc[NS];   // scores (stored back as they are)
  S rk[NS];   // ranking values (scores, or scaled to means)
  int ds[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const int e = lane + 32 * s;
    sc[s] = kLow;
    ds[s] = 0;
    if (e < nl) {
      const Cand<S> cd = B.cand.get(e);
      sc[s] = cd.score;
      ds[s] = cd.desc;
    } else if (e < C) {
      const int c = e - nl;
      const Cand<S> p = B.xnode.get(c >> 1);
      const S left = B.xleft[c >> 1];
      const int cl = desc_level(p.desc) - 1;
      const int st = desc_start(p.desc);
      ds[s] = make_desc((c & 1) ? st + (1 << cl) : st, cl);
      sc[s] = (c & 1) ? p.score - left : left;
    }
    rk[s] = (NORM && norm_l && e < C) ? sc[s] * (S(1) << (norm_l - desc_level(ds[s]))) : sc[s];
  }
  bool keep[NS];
  if (C > limit) {
    top_r_keep<S, NS>(rk, ds, limit, keep);
  } else {
#pragma unroll
    for (int s = 0; s < NS; ++s) keep[s] = lane + 32 * s < C;
  }
  __syncwarp();  // every read of cand / xnode / xleft above is done before the lists are rewritten
  // classify the kept: 1 key or bucket (stays), 2 int32 left-child row, 3 int16 one, 4 key child
  int cat[NS];
  unsigned b1[NS], b2[NS], b3[NS], b4[NS];
  StepLists o{0, 0, 0, 0};
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const int lv = desc_level(ds[s]);
    cat[s] = !keep[s] ? 0 : (lv <= bucket ? 1 : (lv == 1 ? 4 : ((!kNarrow || lv - 1 > narrow) ? 2 : 3)));
    b1[s] = __ballot_sync(kFull, cat[s] == 1);
    b2[s] = __ballot_sync(kFull, cat[s] == 2);
    b3[s] = kNarrow ? __ballot_sync(kFull, cat[s] == 3) : 0u;
    b4[s] = __ballot_sync(kFull, cat[s] == 4);
    o.nl += __popc(b1[s]);
    o.nw += __popc(b2[s]);
    o.nn += __popc(b3[s]);
    o.nk += __popc(b4[s]);
  }
  const unsigned below = lanemask_lt(lane);
  int p1 = 0, p2 = 0, p3 = o.nw, p4 = o.nw + o.nn;
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    if (cat[s] == 1) {
      B.cand.put(p1 + __popc(b1[s] & below), ds[s], sc[s]);
    } else if (cat[s] >= 2) {
      const int pos = cat[s] == 2 ? p2 + __popc(b2[s] & below)
                                  : (cat[s] == 3 ? p3 + __popc(b3[s] & below)
                                                 : p4 + __popc(b4[s] & below));
      const int cl = desc_level(ds[s]) - 1;
      const int st = desc_start(ds[s]);
      B.xnode.put(pos, ds[s], sc[s]);
      B.xrow[pos] = cat[s] == 4 ? st * D : tree_row_offset<D>(n, narrow, cl, st >> cl);
    }
    p1 += __popc(b1[s]);
    p2 += __popc(b2[s]);
    p3 += __popc(b3[s]);
    p4 += __popc(b4[s]);
  }
  __syncwarp();
  return o;
}

template <typename S, int D, bool NORM>
__device__ __forceinline__ StepLists step_select_classify_any(WarpBuf<S>& B, int nl, int nx,
                                                              int limit, int lane, int norm_l,
                                                              int bucket, int n, int narrow) {
  if (nl + 2 * nx <= 96)
    return step_select_classify<S, D, 3, NORM>(B, nl, nx, limit, lane, norm_l, bucket, n, narrow);
  return step_select_classify<S, D, 6, NORM>(B, nl, nx, limit, lane, norm_l, bucket, n, narrow);
}

}  // namespace alhr
