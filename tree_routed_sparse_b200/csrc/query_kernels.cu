// query_kernels.cu -- warp-per-query kernels of the ALHR inference path (sm_100a).
//
// Follows the README of ALHR ("Adaptive learnable Hierarchical routing"), section "Inference
// stage": budget predictor on the query and the causal key sum, the own key and its neighbour
// window first, then a budget-limited descent of the past-only forest, then exact attention
// over the selected keys.
//
// Per query (one warp, rows scored in row groups, see alhr_device.cuh):
//   1. causal sum: G_i = sum of keys [0, i] = (sum of the roots of the past-only forest, the
//      aligned power-of-two blocks of [0, i-w]) + (sum of the window keys (i-w, i]). Both kinds
//      of rows are read in one pass and scored there too: the roots for the descent, the window
//      keys for the attention, so G_i costs no extra row;
//   2. budget: logits over 32 classes from W in shared memory (int64, ties -> lower class), or
//      the given budget (the roots and window keys are then read only where they are used);
//   3. the descent: each step reads only the LEFT child of every expanded node (the right
//      child's score is parent - left, exact in integers) and keeps the best r by an exact
//      integer bisection (select_top_r);
//   4. attention: routed keys keep the scores of the descent (their key rows are not read
//      again), the window keys theirs from phase 1, and the value rows are gathered.
// Descent variants (runtime, both off by default): ranking by means (the selection scales each
// candidate's sum by 2^(L - level)), and leaf buckets (nodes of level <= b are not expanded, the
// beam keeps r >> b of them, and their keys are listed and scored after the descent).
#include <atomic>
#include <cuda_runtime.h>

#include "internal.h"
#include "query_common.cuh"

namespace alhr {

// Bit 29 of a node descriptor is free (start < 2^20): it marks, in the list of causal-sum
// blocks, a block that is also a root of the descent forest.
constexpr int kFlagRoot = 1 << 29;

// The next query ticket of a CTA's shared counter, for the whole warp.
__device__ __forceinline__ int take_ticket(int* counter, int lane) {
  int t = 0;
  if (lane == 0) t = atomicAdd(counter, 1);
  return __shfl_sync(kFull, t, 0);
}

// Shape of the throughput launch: CTAs of 14 warps (one query each), two per SM, i.e. 28
// queries in flight per SM at 72 registers per thread, for both score widths. Measured against
// 8-warp CTAs (three per SM at 80 registers with int32 scores, two at 126 with int64): the extra
// warps hide more of each query's dependent latency (L2 round trips of the child rows, the
// selection's reductions), and two large CTAs hold fewer per-CTA copies of the predictor weights
// in shared memory than seven 4-warp CTAs would, which leaves more of the SM's unified shared
// memory / L1 to the cache.
constexpr int kQueryWarps = 14;
constexpr int kQueryBlocksPerSm = 2;
// At d = 128 this is the number of int16 rows (two 16-byte loads each) in flight; int32 rows at
// d = 128 go one per pass.
template <typename S, int D>
constexpr int tree_rows_in_flight() {
  return D == 128 ? (sizeof(S) == 4 ? 3 : 2) : (sizeof(S) == 4 ? 2 : 1);
}

// One pass over expanded nodes whose left child is an int32 tree row: each row group loads US
// rows (US in flight per lane) and leaves their scores in xleft.
template <int US, typename S, int D>
__device__ __forceinline__ void tree_child_pass(WarpBuf<S>& B, const char* Th, const RowQ& q,
                                                int base, int end, int grp, int sub) {
  constexpr int RPI = Lay<D>::RPI;
  constexpr int TPR = Lay<D>::TPR;
  int x[US][16];
#pragma unroll
  for (int u = 0; u < US; ++u) {
    // a row group past the end loads the pass's last row again (in bounds; its score is not
    // stored), so that no lane spends instructions clearing registers
    const int xi = base + u * RPI + grp;
    ld_tree<D>(Th + B.xrow[min(xi, end - 1)], sub, x[u]);
  }
  if constexpr (US > 2) __syncwarp();  // latency shape: reconverge before the group sums
#pragma unroll
  for (int u = 0; u < US; ++u) {
    const int xi = base + u * RPI + grp;
    const S left = group_sum<S, TPR>(dot_tree<S>(q, x[u]));
    if (xi < end && sub == 0) B.xleft[xi] = left;
  }
}

// One pass over expanded nodes whose left child is an int16 tree row (positions [base, end) of
// the x lists, all narrow): US rows per group, every load issued before any is scored.
template <int US, typename S, int D>
__device__ __forceinline__ void narrow_child_pass(WarpBuf<S>& B, const char* Th, const RowQ& q,
                                                  int base, int end, int grp, int sub) {
  constexpr int RPI = Lay<D>::RPI;
  constexpr int TPR = Lay<D>::TPR;
  int w[US][8];
#pragma unroll
  for (int u = 0; u < US; ++u) {
    const int xi = base + u * RPI + grp;  // past the end: the last row again, not stored
    ld_tree16<D>(Th + B.xrow[min(xi, end - 1)], sub, w[u]);
  }
  __syncwarp();  // reconverge before the group sums
#pragma unroll
  for (int u = 0; u < US; ++u) {
    const int xi = base + u * RPI + grp;
    // the whole row's score fits in int32 (|q| <= 127, |x| <= 32767, d = 128), so the group
    // sum runs in int32 and is widened once
    const S left = S(group_sum<int, TPR>(dot_tree16(q, w[u])));
    if (xi < end && sub == 0) B.xleft[xi] = left;
  }
}

// The warp-per-query kernel (the throughput shape: two CTAs of 14 warps per SM, for
// launches that fill the GPU; smaller launches take the CTA-per-query kernel of
// cta_query_kernels.cu). VAR compiles in the descent variants (ranking by means, leaf buckets;
// chosen at run time from the arguments); without it the method's descent carries none of their
// code.
template <typename S, int D, int MODE, bool VAR>
__global__ void __launch_bounds__(kQueryWarps * 32, kQueryBlocksPerSm)
    query_kernel(const QueryArgs a) {
  constexpr int NW = kQueryWarps;
  constexpr int TPR = Lay<D>::TPR;
  constexpr int RPI = Lay<D>::RPI;
  // tree rows per group per pass (at d = 128: int16 rows; int32 rows go one per pass)
  constexpr int U = tree_rows_in_flight<S, D>();
  constexpr int UV = 2;  // value-row passes in flight
  constexpr bool kUsesW = (MODE == kForwardPredict || MODE == kPredictOnly);
  constexpr bool kDescend = (MODE != kPredictOnly);
  constexpr bool kAttend = (MODE == kForwardPredict || MODE == kForwardOverride);
  constexpr bool kNarrow = (D == 128);  // int16 tree levels exist (see tree_layout.h)
  // How G_i is formed with the predictor. At d = 128: from the forest roots of [0, i-w] and the
  // window keys, which the query reads anyway (no extra row). At d = 64: from the blocks of the
  // binary decomposition of [0, i+1), whose largest blocks are also the largest roots (read
  // once for both) -- about 2.6 more rows per query, but measured 3 % faster there than summing
  // the window keys into G_i, which costs 16 more instructions per key row and spills
  // registers in this register-bound kernel.
  constexpr bool kGBlocks = kUsesW && D == 64;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  constexpr int GS = WLayout<D>::g_stride;
  int* sWg = reinterpret_cast<int*>(smem_raw);
  int* sWq = sWg + 32 * GS;
  WarpBuf<S>* wbuf = reinterpret_cast<WarpBuf<S>*>(smem_raw + QuerySmem<S, D, MODE>::w_bytes);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int grp = lane / TPR;
  const int sub = lane % TPR;
  // Queries are handed out as tickets: ticket t of this CTA is query (blockIdx.x + (t / NW) *
  // gridDim.x) * NW + t % NW, so the CTA's warps work on neighbouring queries (rows they share
  // stay in L1), and a warp that finishes early takes the next ticket instead of leaving its
  // slot idle in the launch's tail (a static split left 7 % of the warp slots idle; the tickets
  // measured 2-7 % faster). Which warp runs a query changes nothing in its results.
  __shared__ int s_ticket;
  if (threadIdx.x == 0) s_ticket = NW;  // tickets 0 .. NW-1 are the warps' first
  if constexpr (kUsesW) stage_weights<D>(a.W, sWg, sWq);
  __syncthreads();
  WarpBuf<S>& B = wbuf[warp];
  const int n = a.n;
  const int w = a.window;
  const long long tree_block = a.tl.block_bytes;
  const int narrow = kNarrow ? a.tl.narrow : 0;  // int16 levels 1 .. narrow (d = 128 only)
  const int bucket = VAR ? a.bucket : 0;          // descent variants: leaf bucket level,
  const int norm_l = VAR ? a.norm_l : 0;          // ranking by means (0: by sums)
  const bool small = a.num_queries <= 0xffffffffLL;  // a 32-bit division suffices

  // tickets only grow, and so do their queries: the first ticket past the end ends the warp
  // (a CTA hands out fewer than num_queries / gridDim.x + 2 * NW < 2^31 of them)
  for (int t = warp;; t = take_ticket(&s_ticket, lane)) {
    const int chunk = t / NW;
    const long long qi =
        ((long long)blockIdx.x + (long long)chunk * gridDim.x) * NW + (t - chunk * NW);
    if (qi >= a.num_queries) break;
    long long bh;
    int pos;
    if (small) {
      const unsigned b32 = unsigned(qi) / unsigned(a.nq);
      bh = b32;
      pos = int(unsigned(qi) - b32 * unsigned(a.nq));
    } else {
      bh = qi / a.nq;
      pos = int(qi - bh * a.nq);
    }
    const int i = a.q_start + pos;
    const int8_t* Kh = a.K + bh * (long long)n * D;
    const char* Th = a.tree + bh * tree_block;

    RowQ q;
    load_rowq<D>(a.Q + qi * D, sub, q);
    {
      bool bad = false;
#pragma unroll
      for (int j = 0; j < 16; ++j) bad |= (q.qn[j] > a.value_bound) | (q.qn[j] < -a.value_bound);
      if (__any_sync(kFull, bad) && lane == 0) flag(a.dev_err, ALHR_DEVERR_VALUE_RANGE);
    }

    const int nwin = min(w, i + 1);  // keys of the window
    const int M = i - w + 1;         // keys before the window: [0, M)
    const unsigned Mu = M > 0 ? unsigned(M) : 0u;
    const int nR = __popc(Mu);       // roots of the descent forest: the blocks of [0, M)
    // kGBlocks: the blocks of [0, i+1) above the highest bit where i+1 and i-w+1 differ are also
    // the largest roots; the rest of the roots (below that bit) are read only for the descent
    const unsigned A = unsigned(i + 1);
    const int p = kGBlocks ? (M > 0 ? 31 - __clz(A ^ Mu) : 31) : 31;
    const unsigned low_mask = p >= 31 ? 0xffffffffu : ((2u << p) - 1u);
    const int n_common = kGBlocks ? __popc(Mu & ~low_mask) : 0;

    int budget = 0, b_eff = 0, nsel_win = 0, r = 0;
    auto settle = [&](int bud) {
      if (bud < 1) {
        if (lane == 0) flag(a.dev_err, ALHR_DEVERR_BUDGET_LOW);
        bud = 1;
      }
      budget = bud;
      b_eff = min(min(bud, i + 1), a.max_keys);
      nsel_win = min(b_eff, nwin);
      r = b_eff - nsel_win;
    };
    if constexpr (!kUsesW) settle(__ldg(a.budget_in + qi));

    // ---- 1. causal sum G_i and budget
    if constexpr (kUsesW) {
      int G[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) G[j] = 0;
      if constexpr (kGBlocks) {
        // the blocks of [0, i+1), largest first; the shared roots' scores go to the front of
        // the candidate list
        const int nA = __popc(A);
        __syncwarp();
        if ((A >> lane) & 1u) {
          const int b = lane;
          const int rank = __popc(A >> b) - 1;
          const int start = int((A >> b) << b) - (1 << b);
          B.plist[rank] = make_desc(start, b) | ((M > 0 && b > p) ? kFlagRoot : 0);
        }
        __syncwarp();
        for (int base = 0; base < nA; base += RPI) {
          const int k = base + grp;
          const bool active = k < nA;
          const int pd = active ? B.plist[k] : 0;
          const int lvl = desc_level(pd);
          const int st = desc_start(pd);
          S sc = 0;
          if (active) {
            if (lvl > 0) {
              int x[16];
              const char* row = Th + tree_row_offset<D>(n, narrow, lvl, st >> lvl);
              if (kNarrow && lvl <= narrow) ld_tree16_as32<D>(row, sub, x);
              else ld_tree<D>(row, sub, x);
#pragma unroll
              for (int j = 0; j < 16; ++j) G[j] += x[j];
              sc = dot_tree<S>(q, x);
            } else {
              int xp[4];
              ld_key<D>(Kh + (long long)st * D, sub, xp);
#pragma unroll
              for (int v = 0; v < 4; ++v)
#pragma unroll
                for (int e = 0; e < 4; ++e) G[4 * v + e] += sx8(xp[v], e);
              sc = S(dot_key(q, xp));
            }
          }
          sc = group_sum<S, TPR>(sc);
          // the shared roots are the first ones; every lane stores (the same value per row
          // group; rows that are no roots into a spare slot), so no divergent store precedes the
          // cross-group sum of G_i below
          B.cand.put((active && (pd & kFlagRoot)) ? k : kMaxCand - 1, pd & ~kFlagRoot, sc);
        }
      } else {
        // the forest roots, largest first
        __syncwarp();
        if ((Mu >> lane) & 1u) {
          const int b = lane;
          B.plist[__popc(Mu >> b) - 1] = make_desc(int((Mu >> b) << b) - (1 << b), b);
        }
        __syncwarp();
        // roots: one row per group per pass. Every lane of a row group stores the score (the
        // same value; rows past the end into a spare slot), so the pass has no divergent store
        // before the cross-group sum of G_i below.
        for (int base = 0; base < nR; base += RPI) {
          const int k = base + grp;
          const bool active = k < nR;
          const int pd = active ? B.plist[k] : 0;
          const int lvl = desc_level(pd);
          const int st = desc_start(pd);
          S sc = 0;
          if (active) {
            if (lvl > 0) {
              int x[16];
              const char* row = Th + tree_row_offset<D>(n, narrow, lvl, st >> lvl);
              if (kNarrow && lvl <= narrow) ld_tree16_as32<D>(row, sub, x);
              else ld_tree<D>(row, sub, x);
#pragma unroll
              for (int j = 0; j < 16; ++j) G[j] += x[j];
              sc = dot_tree<S>(q, x);
            } else {
              int xp[4];
              ld_key<D>(Kh + (long long)st * D, sub, xp);
#pragma unroll
              for (int v = 0; v < 4; ++v)
#pragma unroll
                for (int e = 0; e < 4; ++e) G[4 * v + e] = __dp4a(xp[v], 1 << (8 * e), G[4 * v + e]);
              sc = S(dot_key(q, xp));
            }
          }
          sc = group_sum<S, TPR>(sc);
          B.cand.put(active ? k : kMaxCand - 1, pd, sc);
        }
        // window keys i, i-1, ..., one per group per pass: scores for the attention, values
        // into G_i (dp4a with a one-hot byte picks one sign-extended dimension)
        for (int base = 0; base < nwin; base += RPI) {
          const int x = base + grp;
          int xp[4] = {0, 0, 0, 0};
          if (x < nwin) ld_key<D>(Kh + (long long)(i - x) * D, sub, xp);
#pragma unroll
          for (int v = 0; v < 4; ++v)
#pragma unroll
            for (int e = 0; e < 4; ++e) G[4 * v + e] = __dp4a(xp[v], 1 << (8 * e), G[4 * v + e]);
          const int sw = group_sum<int, TPR>(dot_key(q, xp));
          B.winsc[x < nwin ? x : kMaxWindow] = sw;
        }
      }
      __syncwarp();
#pragma unroll
      for (int off = TPR; off < 32; off *= 2)
#pragma unroll
        for (int j = 0; j < 16; ++j) G[j] += __shfl_xor_sync(kFull, G[j], off);

      // ---- 2. budget predictor: group grp scores classes grp, grp+RPI, ...
      long long best = ScoreLimits<long long>::lowest;
#pragma unroll
      for (int k = 0; k < 32 / RPI; ++k) {
        const int c = grp + RPI * k;
        const long long logit = group_sum<long long, TPR>(class_logit_part<D>(sWg, sWq, c, sub, q, G));
        // largest logit, then lowest class: pack (logit, 31 - class)
        const long long key = logit * 32 + (31 - c);
        best = key > best ? key : best;
      }
#pragma unroll
      for (int off = TPR; off < 32; off *= 2) {
        const long long o = __shfl_xor_sync(kFull, best, off);
        best = o > best ? o : best;
      }
      settle(3 * (31 - int(best & 31) + 1));
    }

    if constexpr (MODE == kPredictOnly) {
      if (lane == 0) a.budget_out[qi] = budget;
      continue;
    }

    // ---- 3. descent of the past-only forest
    int nf = 0, exp_hi = 0, exp_l1 = 0, exp_wide = 0;
    const int keep = r >> bucket;  // beam width in buckets (keys when bucket = 0)
    if (kDescend && keep > 0) {    // r > 0 implies i >= w, i.e. M > 0
      // roots not scored yet: all of them without the predictor, those below the shared
      // blocks with kGBlocks
      if constexpr (!kUsesW || kGBlocks) {
        const unsigned rest = Mu & low_mask;
        const int nB = __popc(rest);
        __syncwarp();
        if ((rest >> lane) & 1u) {
          const int b = lane;
          B.plist[__popc(rest >> b) - 1] = make_desc(int((Mu >> b) << b) - (1 << b), b);
        }
        __syncwarp();
        for (int base = 0; base < nB; base += RPI) {
          const int k = base + grp;
          const bool active = k < nB;
          const int pd = active ? B.plist[k] : 0;
          const int lvl = desc_level(pd);
          const int st = desc_start(pd);
          S sc = 0;
          if (active) {
            if (lvl == 0) {
              int xp[4];
              ld_key<D>(Kh + (long long)st * D, sub, xp);
              sc = S(dot_key(q, xp));
            } else if (!kNarrow || lvl > narrow) {
              int x[16];
              ld_tree<D>(Th + tree_row_offset<D>(n, narrow, lvl, st >> lvl), sub, x);
              sc = dot_tree<S>(q, x);
            } else {
              int w[8];
              ld_tree16<D>(Th + tree_row_offset<D>(n, narrow, lvl, st >> lvl), sub, w);
              sc = S(dot_tree16(q, w));
            }
          }
          sc = group_sum<S, TPR>(sc);
          if (active && sub == 0) B.cand.put(n_common + k, pd, sc);
        }
      }
      nf = nR;

      for (int step = 0; step < 32; ++step) {
        __syncwarp();
        // classify the frontier: keys stay; nodes to expand by the width of their left child's
        // row: int32 tree row (level - 1 > narrow), int16 tree row, or key (level 1)
        int fd[kFrontSlots];
        S fs[kFrontSlots];
        int cat[kFrontSlots];  // 0 none, 1 key, 2 wide child, 3 narrow child, 4 key child
        unsigned bl_[kFrontSlots], bw_[kFrontSlots], bn_[kFrontSlots], bk_[kFrontSlots];
        int nl = 0, nw = 0, nn = 0, nk = 0;
#pragma unroll
        for (int s = 0; s < kFrontSlots; ++s) {
          cat[s] = 0;
          bl_[s] = bw_[s] = bn_[s] = bk_[s] = 0u;
          fd[s] = 0;
          fs[s] = S(0);
          if (32 * s < nf) {  // warp-uniform: only the slots the frontier occupies
            const int e = lane + 32 * s;
            if (e < nf) {
              const Cand<S> cd = B.cand.get(e);
              fd[s] = cd.desc;
              fs[s] = cd.score;
              const int lv = desc_level(fd[s]);
              cat[s] = lv <= bucket ? 1 : (lv == 1 ? 4 : ((!kNarrow || lv - 1 > narrow) ? 2 : 3));
            }
            bl_[s] = __ballot_sync(kFull, cat[s] == 1);
            bw_[s] = __ballot_sync(kFull, cat[s] == 2);
            if constexpr (kNarrow) bn_[s] = __ballot_sync(kFull, cat[s] == 3);
            bk_[s] = __ballot_sync(kFull, cat[s] == 4);
            nl += __popc(bl_[s]);
            nw += __popc(bw_[s]);
            nn += __popc(bn_[s]);
            nk += __popc(bk_[s]);
          }
        }
        const int nhi = nw + nn;  // tree-row children
        const int nx = nhi + nk;
        if (nx == 0) {
          // nothing to expand; more nodes than the beam only when the roots are all buckets
          if constexpr (VAR) {
            if (nf > keep) {
              select_top_r<S, true>(B, nf, keep, lane, norm_l);
              nf = keep;
            }
          }
          break;
        }
        exp_hi += nhi;
        exp_l1 += nk;
        exp_wide += nw;
        __syncwarp();
        {
          // keys stay candidates; expanded nodes go to the x lists ([wide | narrow | key]) with
          // the byte offset of their left child's row, computed once per node here
          const unsigned below = lanemask_lt(lane);
          int ow = 0, on = nw, ok = nhi, ol = 0;
#pragma unroll
          for (int s = 0; s < kFrontSlots; ++s) {
            if (cat[s] >= 2) {
              const int pos = cat[s] == 2 ? ow + __popc(bw_[s] & below)
                                          : (cat[s] == 3 ? on + __popc(bn_[s] & below)
                                                         : ok + __popc(bk_[s] & below));
              const int cl = desc_level(fd[s]) - 1;
              const int st = desc_start(fd[s]);
              B.xnode.put(pos, fd[s], fs[s]);
              B.xrow[pos] = cat[s] == 4 ? st * D : tree_row_offset<D>(n, narrow, cl, st >> cl);
            } else if (cat[s] == 1) {
              const int pos = ol + __popc(bl_[s] & below);
              B.cand.put(pos, fd[s], fs[s]);
            }
            ow += __popc(bw_[s]);
            on += __popc(bn_[s]);
            ok += __popc(bk_[s]);
            ol += __popc(bl_[s]);
          }
        }
        __syncwarp();
        // left children that are tree rows: U rows per group in flight (a single pass body:
        // a separate short tail pass measured slower through instruction-cache misses)
        if constexpr (kNarrow) {
          // int32 and int16 rows in passes of their own, so that every pass issues all of its
          // loads before it scores any (one memory round trip per pass)
          for (int base = 0; base < nw; base += RPI)
            tree_child_pass<1, S, D>(B, Th, q, base, nw, grp, sub);
          for (int base = nw; base < nhi; base += U * RPI)
            narrow_child_pass<U, S, D>(B, Th, q, base, nhi, grp, sub);
        } else {
          for (int base = 0; base < nhi; base += U * RPI)
            tree_child_pass<U, S, D>(B, Th, q, base, nhi, grp, sub);
        }
        // left children that are keys: one per group per pass
        for (int base = nhi; base < nx; base += RPI) {
          const int xi = base + grp;
          int xp[4];
          ld_key<D>(Kh + B.xrow[min(xi, nx - 1)], sub, xp);  // past the end: not stored
          const int left = group_sum<int, TPR>(dot_key(q, xp));
          if (xi < nx && sub == 0) B.xleft[xi] = S(left);
        }
        __syncwarp();
        // both children of every expanded node, one node per lane
        for (int x0 = lane; x0 < nx; x0 += 32)
          put_children<S>(B, nl, x0, B.xnode.get(x0), B.xleft[x0]);
        const int C = nl + 2 * nx;
        if (C > keep) {
          select_top_r<S, VAR>(B, C, keep, lane, norm_l);
          nf = keep;
        } else {
          nf = C;
        }
      }
      if constexpr (VAR)
        if (bucket > 0) nf = expand_buckets<S, D>(B, nf, Kh, q, lane);
    }

    // ---- window key scores (attention only needs the selected ones; with the predictor at
    //      d = 128 they were taken in phase 1)
    if constexpr (kAttend && !(kUsesW && !kGBlocks)) {
      for (int base = 0; base < nsel_win; base += RPI) {
        const int x = base + grp;
        int xp[4];
        ld_key<D>(Kh + (long long)(i - min(x, nsel_win - 1)) * D, sub, xp);  // past: not stored
        const int s = group_sum<int, TPR>(dot_key(q, xp));
        if (x < nsel_win && sub == 0) B.winsc[x] = s;
      }
    }
    __syncwarp();

    // ---- optional outputs of the route
    const int count = nsel_win + nf;
    if (a.count_out && lane == 0) a.count_out[qi] = count;
    if (a.exp_out && lane == 0) {
      a.exp_out[3 * qi] = exp_hi;
      a.exp_out[3 * qi + 1] = exp_l1;
      a.exp_out[3 * qi + 2] = exp_wide;
    }
    if (a.budget_out && lane == 0) a.budget_out[qi] = budget;
    if (a.idx_out) write_selection<S>(B, nf, nsel_win, i, a.idx_out + qi * a.max_keys, a.max_keys, lane);

    // ---- 4. exact attention over window + routed keys
    if constexpr (kAttend) {
      const float scale = a.scale;
      const float sw = lane < nsel_win ? float(B.winsc[lane]) * scale : -INFINITY;
      float sr[kFrontSlots];
      int kr[kFrontSlots];
#pragma unroll
      for (int s = 0; s < kFrontSlots; ++s) {
        const int e = lane + 32 * s;
        Cand<S> cd{0, S(0)};
        if (e < nf) cd = B.cand.get(e);
        sr[s] = e < nf ? float(cd.score) * scale : -INFINITY;
        kr[s] = desc_start(cd.desc);
      }
      float m = sw;
#pragma unroll
      for (int s = 0; s < kFrontSlots; ++s) m = fmaxf(m, sr[s]);
      m = warp_maxf(m);
      const float pw = lane < nsel_win ? __expf(sw - m) : 0.f;
      float pr[kFrontSlots];
      float psum = pw;
#pragma unroll
      for (int s = 0; s < kFrontSlots; ++s) {
        pr[s] = (lane + 32 * s) < nf ? __expf(sr[s] - m) : 0.f;
        psum += pr[s];
      }
      const float den = warp_sumf(psum);
      // stage keys and weights: window keys first, then the routed keys
      if (lane < nsel_win) {
        B.selk[lane] = i - lane;
        B.selp[lane] = pw;
      }
#pragma unroll
      for (int s = 0; s < kFrontSlots; ++s) {
        const int e = lane + 32 * s;
        if (e < nf) {
          B.selk[nsel_win + e] = kr[s];
          B.selp[nsel_win + e] = pr[s];
        }
      }
      __syncwarp();
      gather_values<D, UV>(B.selk, B.selp, nsel_win + nf, 1.f / den, a.V + bh * (long long)n * D,
                          lane, a.out + qi * D);
    }
  }
}

// Exact attention over a given selection (idx, count): key rows for the scores (row groups),
// value rows for the sum. Entries outside [0, i] are skipped and flagged.
template <int D>
__global__ void __launch_bounds__(kWarps * 32) attend_kernel(const QueryArgs a) {
  constexpr int TPR = Lay<D>::TPR;
  constexpr int RPI = Lay<D>::RPI;
  __shared__ WarpBuf<int> wbuf[kWarps];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int grp = lane / TPR;
  const int sub = lane % TPR;
  WarpBuf<int>& B = wbuf[warp];
  const int n = a.n;
  const long long stride = (long long)gridDim.x * kWarps;
  for (QueryCursor cur((long long)blockIdx.x * kWarps + warp, a.nq, stride);
       cur.qi < a.num_queries; cur.advance(stride, a.nq)) {
    const long long qi = cur.qi;
    const long long bh = cur.bh;
    const int i = a.q_start + cur.r;
    const int8_t* Kh = a.K + bh * (long long)n * D;
    const uint16_t* Vh = a.V + bh * (long long)n * D;
    RowQ q;
    load_rowq<D>(a.Q + qi * D, sub, q);
    const int cnt = max(0, min(__ldg(a.count_in + qi), a.max_keys));
    int key[kFrontSlots];
    bool ok[kFrontSlots];
    bool bad = false;
    __syncwarp();
#pragma unroll
    for (int s = 0; s < kFrontSlots; ++s) {
      const int e = lane + 32 * s;
      key[s] = e < cnt ? __ldg(a.idx_in + qi * a.max_keys + e) : -1;
      ok[s] = e < cnt && key[s] >= 0 && key[s] <= i;
      bad |= e < cnt && !ok[s];
      if (e < cnt) B.cand.set_desc(e, ok[s] ? key[s] : -1);
    }
    if (__any_sync(kFull, bad) && lane == 0) flag(a.dev_err, ALHR_DEVERR_INDEX);
    __syncwarp();
    for (int base = 0; base < cnt; base += RPI) {
      const int x = base + grp;
      const int kk = x < cnt ? B.cand.desc(x) : -1;
      int xp[4] = {0, 0, 0, 0};
      if (kk >= 0) ld_key<D>(Kh + (long long)kk * D, sub, xp);
      const int s = group_sum<int, TPR>(dot_key(q, xp));
      if (x < cnt && sub == 0) B.cand.set_score(x, s);
    }
    __syncwarp();
    float sc[kFrontSlots];
#pragma unroll
    for (int s = 0; s < kFrontSlots; ++s)
      sc[s] = ok[s] ? float(B.cand.score(lane + 32 * s)) * a.scale : -INFINITY;
    float m = -INFINITY;
#pragma unroll
    for (int s = 0; s < kFrontSlots; ++s) m = fmaxf(m, sc[s]);
    m = warp_maxf(m);
    float pr[kFrontSlots];
    float psum = 0.f;
#pragma unroll
    for (int s = 0; s < kFrontSlots; ++s) {
      pr[s] = ok[s] ? __expf(sc[s] - m) : 0.f;
      psum += pr[s];
    }
    const float den = warp_sumf(psum);
    // skipped entries keep weight 0 and read row 0 of the head (always in bounds)
#pragma unroll
    for (int s = 0; s < kFrontSlots; ++s) {
      const int e = lane + 32 * s;
      if (e < cnt) {
        B.selk[e] = ok[s] ? key[s] : 0;
        B.selp[e] = pr[s];
      }
    }
    __syncwarp();
    gather_values<D, 2>(B.selk, B.selp, cnt, den > 0.f ? 1.f / den : 0.f, Vh, lane,
                        a.out + qi * D);
  }
}

// ------------------------------------------------------------------ launchers

namespace {

constexpr int kOccSlots = 66;

// Grid size of a persistent launch: the resident CTAs of every SM, capped by the work. The
// per-device occupancy (and the opt-in to more than 48 KB of dynamic shared memory) is
// computed once per device and kernel.
template <typename KernelT>
int blocks_for(KernelT kernel, int slot, size_t smem, long long queries, cudaError_t* err,
               int warps = kWarps) {
  static thread_local int cached_dev = -1;
  static thread_local int sms = 0;
  static thread_local int per_sm[kOccSlots] = {0};
  *err = cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != cached_dev) {
    for (int k = 0; k < kOccSlots; ++k) per_sm[k] = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cached_dev = dev;
  }
  if (per_sm[slot] == 0) {
    if (smem > 48 * 1024) {
      *err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      if (*err != cudaSuccess) return 0;
    }
    int b = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, warps * 32, smem);
    per_sm[slot] = b > 0 ? b : 1;
  }
  const long long need = (queries + warps - 1) / warps;
  const long long cap = (long long)sms * per_sm[slot];
  return int(need < cap ? need : cap);
}

template <typename S, int D, int MODE, bool VAR>
cudaError_t launch_query_mode(const QueryArgs& a, cudaStream_t st) {
  constexpr int slot = ((MODE * 2 + (D == 128 ? 1 : 0)) * 2 + (sizeof(S) == 8 ? 1 : 0)) * 2 +
                       (VAR ? 1 : 0);
  static_assert(slot < 64, "occupancy cache slot");
  constexpr int nw = kQueryWarps;
  constexpr size_t smem = QuerySmem<S, D, MODE>::bytes_for(nw);
  auto kern = query_kernel<S, D, MODE, VAR>;
  cudaError_t err;
  const int blocks = blocks_for(kern, slot, smem, a.num_queries, &err, nw);
  if (err != cudaSuccess) return err;
  if (blocks <= 0) return cudaSuccess;
  kern<<<blocks, nw * 32, smem, st>>>(a);
  return cudaGetLastError();
}

std::atomic<int> g_launch_mode{0};

// Auto: a launch whose queries are all resident at once as one CTA each (latency shape: four
// warps per query up to four CTAs per SM, two warps per query beyond that) takes that shape;
// larger launches take one warp per query. The latency mode forces the CTA shape.
template <typename S, int D, int MODE>
cudaError_t launch_query(const QueryArgs& a, cudaStream_t st) {
  const int mode = g_launch_mode.load(std::memory_order_relaxed);
  if (mode != 1) {
    bool launched = false;
    const cudaError_t e =
        launch_query_cta(a, D, sizeof(S) == 4 ? 32 : 64, MODE, mode == 2, &launched, st);
    if (e != cudaSuccess || launched) return e;
  }
  // the predictor alone never descends: it needs no variant instantiation
  if (MODE != kPredictOnly && (a.norm_l != 0 || a.bucket != 0))
    return launch_query_mode<S, D, MODE, MODE != kPredictOnly>(a, st);
  return launch_query_mode<S, D, MODE, false>(a, st);
}

template <int MODE>
cudaError_t dispatch_query(const QueryArgs& a, int d, int score_bits, cudaStream_t st) {
  if (d == 64) {
    return score_bits == 32 ? launch_query<int, 64, MODE>(a, st)
                            : launch_query<long long, 64, MODE>(a, st);
  }
  return score_bits == 32 ? launch_query<int, 128, MODE>(a, st)
                          : launch_query<long long, 128, MODE>(a, st);
}

}  // namespace

cudaError_t launch_forward(const QueryArgs& a, int d, int score_bits, bool predict,
                           cudaStream_t st) {
  return predict ? dispatch_query<kForwardPredict>(a, d, score_bits, st)
                 : dispatch_query<kForwardOverride>(a, d, score_bits, st);
}

cudaError_t launch_route(const QueryArgs& a, int d, int score_bits, cudaStream_t st) {
  return dispatch_query<kRouteOnly>(a, d, score_bits, st);
}

cudaError_t launch_predict(const QueryArgs& a, int d, int score_bits, cudaStream_t st) {
  return dispatch_query<kPredictOnly>(a, d, score_bits, st);
}

void set_query_launch_mode(int mode) { g_launch_mode.store(mode, std::memory_order_relaxed); }
int query_launch_mode() { return g_launch_mode.load(std::memory_order_relaxed); }

cudaError_t launch_attend(const QueryArgs& a, int d, cudaStream_t st) {
  cudaError_t err;
  if (d == 64) {
    const int blocks = blocks_for(attend_kernel<64>, 64, 0, a.num_queries, &err);
    if (err != cudaSuccess) return err;
    attend_kernel<64><<<blocks, kWarps * 32, 0, st>>>(a);
  } else {
    const int blocks = blocks_for(attend_kernel<128>, 65, 0, a.num_queries, &err);
    if (err != cudaSuccess) return err;
    attend_kernel<128><<<blocks, kWarps * 32, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace alhr
