// cta_query_kernels.cu -- CTA-per-query kernels of the ALHR inference path (sm_100a): the
// latency shape, for launches too small to fill the GPU with one warp per query (decode).
//
// Same computation as the warp-per-query kernels of query_kernels.cu (README of ALHR, section
// "Inference stage": causal key sum and budget predictor, own key and neighbour window, descent
// of the past-only forest, exact attention), with one query per CTA of kCtaWarps warps. A query
// at decode time is a chain of about log2 n dependent descent steps, so its latency is what
// counts: the row work of every phase is spread over the CTA's kCtaWarps * RPI row groups (the
// roots and window keys of the causal sum, a step's left-child rows, the value rows), so that a
// step's rows take one round trip to memory and are scored in parallel, while warp 0 alone runs
// the short serial parts on the shared buffers (classifying the frontier, writing the children,
// the top-r selection). Two CTA barriers per descent step order the two.
#include <cstddef>
#include <cuda_runtime.h>

#include "internal.h"
#include "query_common.cuh"

namespace alhr {

// Warps per query: four for launches whose queries all fit the GPU at once as CTAs of four
// warps (at most four per SM), two for launches up to about twice that size (so that those
// too are resident at once, at half the row parallelism per query).
constexpr int kCtaWarps = 4;
constexpr int kCtaWarpsWide = 2;

// Shared state of one query: the warp-per-query buffer (used here by the whole CTA) plus the
// cross-warp partial sums and the counts warp 0 hands to the others.
template <typename S, int D, int NWC>
struct CtaBuf {
  WarpBuf<S> B;
  long long logit[32];              // class logits of the predictor
  alignas(16) int gpart[NWC][D];    // per-warp partial sums of G_i (lane-slot order:
                                    // sub * 16 + j), read and written as int4
  alignas(16) float opart[NWC][D];  // per-warp partial sums of the output row (float4)
  int ctl[8];                             // counts of a descent step (wide, narrow, key, leaf, nf)
  float inv;                              // 1 / softmax denominator
};
// the 16-byte accesses above need 16-byte offsets
using CtaBufI64 = CtaBuf<int, 64, kCtaWarps>;
using CtaBufL128 = CtaBuf<long long, 128, kCtaWarpsWide>;
static_assert(offsetof(CtaBufI64, gpart) % 16 == 0 && offsetof(CtaBufI64, opart) % 16 == 0,
              "CtaBuf alignment");
static_assert(offsetof(CtaBufL128, gpart) % 16 == 0 && offsetof(CtaBufL128, opart) % 16 == 0,
              "CtaBuf alignment");

template <typename S, int D, int MODE, int NWC>
struct CtaSmem {
  static_assert(QuerySmem<S, D, MODE>::w_bytes % 16 == 0, "CtaBuf placement");
  static constexpr size_t bytes = QuerySmem<S, D, MODE>::w_bytes + sizeof(CtaBuf<S, D, NWC>);
};

// L2 prefetch of the rows the next step may read: the left children of both children of the
// expanded node at position xi (level lv, start st), i.e. two rows of level lv - 2 (keys when
// lv = 2). Issued by every lane for its part of the row, as a load of that row would be.
template <int D>
__device__ __forceinline__ void prefetch_grandchildren(const char* Th, const int8_t* Kh, int n,
                                                       int narrow, int bucket, int desc, int sub) {
  const int lv = desc_level(desc);
  if (lv - 1 <= bucket || lv < 2) return;  // the children are not expanded
  const int gl = lv - 2;
  const int st = desc_start(desc);
#pragma unroll
  for (int side = 0; side < 2; ++side) {
    const int s2 = st + side * (1 << (lv - 1));
    const char* p;
    int bytes;
    if (gl == 0) {
      p = reinterpret_cast<const char*>(Kh) + (long long)s2 * D;
      bytes = D;
    } else {
      p = Th + tree_row_offset<D>(n, narrow, gl, s2 >> gl);
      bytes = (D == 128 && gl <= narrow) ? 2 * D : 4 * D;
    }
    // the row group's TPR lanes cover the row in 32-byte pieces (a 128-byte line each: a row
    // is at most 4 lines)
    for (int off = 128 * sub; off < bytes; off += 128 * Lay<D>::TPR)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p + off));
  }
}

// One pass over CTA-wide positions [base, end) of the expanded-node lists: row group gg takes
// positions base + gg + u * NG (u < US), loads them all, then scores them. KIND 0: int32 tree
// rows, 1: int16 tree rows, 2: key rows. A warp without positions in the pass skips it.
template <int KIND, int US, typename S, int D, int NWC>
__device__ __forceinline__ void cta_child_pass(WarpBuf<S>& B, const char* Th, const int8_t* Kh,
                                               const RowQ& q, int base, int end, int warp,
                                               int gg, int sub, int n, int narrow, int bucket) {
  constexpr int RPI = Lay<D>::RPI;
  constexpr int TPR = Lay<D>::TPR;
  constexpr int NG = NWC * RPI;
  if (base + warp * RPI >= end) return;  // warp-uniform
  constexpr int WORDS = KIND == 0 ? 16 : (KIND == 1 ? 8 : 4);
  int x[US][WORDS];
#pragma unroll
  for (int u = 0; u < US; ++u) {
    // a row group past the end loads the pass's last row again (in bounds; its score is not
    // stored), so that no lane spends instructions clearing registers
    const int xi = base + u * NG + gg;
    const int xr = B.xrow[min(xi, end - 1)];
    if constexpr (KIND == 0) ld_tree<D>(Th + xr, sub, x[u]);
    else if constexpr (KIND == 1) ld_tree16<D>(Th + xr, sub, x[u]);
    else ld_key<D>(Kh + xr, sub, x[u]);
    if (xi < end) prefetch_grandchildren<D>(Th, Kh, n, narrow, bucket, B.xnode.desc(xi), sub);
  }
  __syncwarp();
#pragma unroll
  for (int u = 0; u < US; ++u) {
    const int xi = base + u * NG + gg;
    S left;
    if constexpr (KIND == 0) left = group_sum<S, TPR>(dot_tree<S>(q, x[u]));
    else if constexpr (KIND == 1) left = S(group_sum<int, TPR>(dot_tree16(q, x[u])));
    else left = S(group_sum<int, TPR>(dot_key(q, x[u])));
    if (xi < end && sub == 0) B.xleft[xi] = left;
  }
}

// The value rows of keys [k0, k1) of the staged selection, weighted, summed over the warp's
// value groups; the warp's partial output row goes to part[0 .. D).
template <int D, int UV>
__device__ __forceinline__ void gather_values_part(const int* selk, const float* selp, int k0,
                                                   int k1, const uint16_t* Vh, int lane,
                                                   float* part) {
  constexpr int VPR = D / 8;
  constexpr int KPP = 32 / VPR;
  const int kg = lane / VPR;
  const int vs = lane % VPR;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
  for (int base = k0; base < k1; base += UV * KPP) {
    uint4 raw[UV];
    float p[UV];
#pragma unroll
    for (int u = 0; u < UV; ++u) {
      // a value group past the end loads the last row of the range again with weight 0
      const int k = base + u * KPP + kg;
      raw[u] = __ldg(reinterpret_cast<const uint4*>(Vh + (long long)selk[min(k, k1 - 1)] * D) + vs);
      p[u] = k < k1 ? selp[k] : 0.f;
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
    float4* o = reinterpret_cast<float4*>(part + 8 * vs);
    o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// VAR compiles in the descent variants (ranking by means, leaf buckets), as in query_kernel.
template <typename S, int D, int MODE, bool VAR, int NWC>
__global__ void __launch_bounds__(NWC * 32, 16 / NWC) cta_query_kernel(const QueryArgs a) {
  constexpr int TPR = Lay<D>::TPR;
  constexpr int RPI = Lay<D>::RPI;
  constexpr int NG = NWC * RPI;  // row groups of the CTA
  constexpr bool kUsesW = (MODE == kForwardPredict || MODE == kPredictOnly);
  constexpr bool kDescend = (MODE != kPredictOnly);
  constexpr bool kAttend = (MODE == kForwardPredict || MODE == kForwardOverride);
  constexpr bool kNarrow = (D == 128);
  // rows per group and pass: int32 tree rows, int16 tree rows, key rows (a step expands at most
  // kMaxFrontier - 1 nodes: one pass of each kind covers NG * U of them)
  constexpr int UW = D == 128 ? 3 : 3;
  constexpr int UN = 6;
  constexpr int UK = D == 128 ? 6 : 3;

  extern __shared__ __align__(16) unsigned char smem_raw[];
  int* sWg = reinterpret_cast<int*>(smem_raw);
  int* sWq = sWg + 32 * WLayout<D>::g_stride;
  CtaBuf<S, D, NWC>& C =
      *reinterpret_cast<CtaBuf<S, D, NWC>*>(smem_raw + QuerySmem<S, D, MODE>::w_bytes);
  WarpBuf<S>& B = C.B;

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int grp = lane / TPR;
  const int sub = lane % TPR;
  const int gg = warp * RPI + grp;  // this lane's row group in the CTA
  if constexpr (kUsesW) stage_weights<D>(a.W, sWg, sWq);
  // The serial parts run on one warp, chosen to put the serial warps of the CTAs sharing an SM
  // on different SM sub-partitions (schedulers). A heuristic: if the SM hands a CTA four
  // consecutive warp slots, one per sub-partition, the CTA whose first slot is 4k takes its warp
  // k mod 4. Any choice gives the same results; this one only spreads the serial chains.
  if (threadIdx.x == 0) {
    unsigned wid;
    asm volatile("mov.u32 %0, %%warpid;" : "=r"(wid));
    C.ctl[5] = int((wid / 4) % NWC);
  }
  __syncthreads();
  const int sw = C.ctl[5];
  const int n = a.n;
  const int w = a.window;
  const long long tree_block = a.tl.block_bytes;
  const int narrow = kNarrow ? a.tl.narrow : 0;
  const int bucket = VAR ? a.bucket : 0;
  const int norm_l = VAR ? a.norm_l : 0;

  for (long long qi = blockIdx.x; qi < a.num_queries; qi += gridDim.x) {
    __syncthreads();  // the weights are staged; the previous query is done with the buffers
    const long long bh = qi / a.nq;
    const int i = a.q_start + int(qi - bh * a.nq);
    const int8_t* Kh = a.K + bh * (long long)n * D;
    const char* Th = a.tree + bh * tree_block;

    RowQ q;
    load_rowq<D>(a.Q + qi * D, sub, q);
    if (warp == sw) {
      bool bad = false;
#pragma unroll
      for (int j = 0; j < 16; ++j) bad |= (q.qn[j] > a.value_bound) | (q.qn[j] < -a.value_bound);
      if (__any_sync(kFull, bad) && lane == 0) flag(a.dev_err, ALHR_DEVERR_VALUE_RANGE);
    }

    const int nwin = min(w, i + 1);
    const int M = i - w + 1;
    const unsigned Mu = M > 0 ? unsigned(M) : 0u;
    const int nR = __popc(Mu);

    int budget = 0, b_eff = 0, nsel_win = 0, r = 0;
    auto settle = [&](int bud) {
      if (bud < 1) {
        if (threadIdx.x == 0) flag(a.dev_err, ALHR_DEVERR_BUDGET_LOW);
        bud = 1;
      }
      budget = bud;
      b_eff = min(min(bud, i + 1), a.max_keys);
      nsel_win = min(b_eff, nwin);
      r = b_eff - nsel_win;
    };
    if constexpr (!kUsesW) settle(__ldg(a.budget_in + qi));

    if (warp == sw && ((Mu >> lane) & 1u))
      B.plist[__popc(Mu >> lane) - 1] = make_desc(int((Mu >> lane) << lane) - (1 << lane), lane);
    __syncthreads();

    // ---- 1. causal sum G_i = (roots of [0, i-w]) + (window keys), scored in the same pass
    if constexpr (kUsesW) {
      constexpr int U1 = (kMaxLevels + kMaxWindow + NG - 1) / NG;
      const int nI = nR + nwin;
      int G[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) G[j] = 0;
      S rsc[U1];
      // rounds of up to 4 rows per group in flight (one round with four warps per query)
      constexpr int UG = U1 < 4 ? U1 : 4;
#pragma unroll
      for (int u0 = 0; u0 < U1; u0 += UG) {
        if (u0 * NG < nI) {  // CTA-uniform
          int x[UG][16];
#pragma unroll
          for (int uu = 0; uu < UG; ++uu) {
            const int k = (u0 + uu) * NG + gg;
#pragma unroll
            for (int j = 0; j < 16; ++j) x[uu][j] = 0;
            if (u0 + uu < U1 && k < nI)
              ld_node32<D, kNarrow>(Th, Kh, n, narrow,
                                    k < nR ? B.plist[k] : make_desc(i - (k - nR), 0), sub, x[uu]);
          }
          __syncwarp();
#pragma unroll
          for (int uu = 0; uu < UG; ++uu) {
            if (u0 + uu < U1) {
              rsc[u0 + uu] = S(0);
              if ((u0 + uu) * NG < nI) {  // CTA-uniform
#pragma unroll
                for (int j = 0; j < 16; ++j) G[j] += x[uu][j];
                rsc[u0 + uu] = group_sum<S, TPR>(dot_tree<S>(q, x[uu]));
              }
            }
          }
        } else {
#pragma unroll
          for (int uu = 0; uu < UG; ++uu)
            if (u0 + uu < U1) rsc[u0 + uu] = S(0);
        }
      }
#pragma unroll
      for (int off = TPR; off < 32; off *= 2)
#pragma unroll
        for (int j = 0; j < 16; ++j) G[j] += __shfl_xor_sync(kFull, G[j], off);
      if (grp == 0) {
        int4* gp = reinterpret_cast<int4*>(&C.gpart[warp][sub * 16]);
#pragma unroll
        for (int v = 0; v < 4; ++v) gp[v] = make_int4(G[4 * v], G[4 * v + 1], G[4 * v + 2], G[4 * v + 3]);
      }
#pragma unroll
      for (int u = 0; u < U1; ++u) {
        const int k = u * NG + gg;
        if (k < nI && sub == 0) {
          if (k < nR) B.cand.put(k, B.plist[k], rsc[u]);
          else B.winsc[k - nR] = int(rsc[u]);
        }
      }
      __syncthreads();
#pragma unroll
      for (int j = 0; j < 16; ++j) G[j] = 0;
#pragma unroll
      for (int ww = 0; ww < NWC; ++ww) {
        const int4* gp = reinterpret_cast<const int4*>(&C.gpart[ww][sub * 16]);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const int4 t = gp[v];
          G[4 * v] += t.x;
          G[4 * v + 1] += t.y;
          G[4 * v + 2] += t.z;
          G[4 * v + 3] += t.w;
        }
      }
      // ---- 2. budget predictor: the CTA's row groups take the 32 classes
#pragma unroll
      for (int kk = 0; kk < (32 + NG - 1) / NG; ++kk) {
        const int c = gg + NG * kk;
        if (c < 32) {  // row-group-uniform
          const long long lg = group_sum<long long, TPR>(class_logit_part<D>(sWg, sWq, c, sub, q, G));
          if (sub == 0) C.logit[c] = lg;
        }
      }
      __syncthreads();
      // largest logit, then lowest class (every warp finds the same)
      long long key = C.logit[lane] * 32 + (31 - lane);
      key = warp_max<long long>(key);
      settle(3 * (31 - int(key & 31) + 1));
    }

    if constexpr (MODE == kPredictOnly) {
      if (threadIdx.x == 0) a.budget_out[qi] = budget;
      continue;
    }

    // ---- 3. descent of the past-only forest
    int nf = 0, exp_hi = 0, exp_l1 = 0, exp_wide = 0;  // counters: warp 0's copies
    const int keep = r >> bucket;
    if (kDescend && keep > 0) {
      if constexpr (!kUsesW) {
        constexpr int UR = (kMaxLevels + NG - 1) / NG;
        int x[UR][16];
#pragma unroll
        for (int u = 0; u < UR; ++u) {
          const int k = u * NG + gg;
#pragma unroll
          for (int j = 0; j < 16; ++j) x[u][j] = 0;
          if (k < nR) ld_node32<D, kNarrow>(Th, Kh, n, narrow, B.plist[k], sub, x[u]);
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < UR; ++u) {
          const int k = u * NG + gg;
          const S sc = group_sum<S, TPR>(dot_tree<S>(q, x[u]));
          if (k < nR && sub == 0) B.cand.put(k, B.plist[k], sc);
        }
        __syncthreads();
      }
      // warp 0 classifies the roots (no pruning before the first expansion; with leaf
      // buckets, roots that are all buckets are pruned to the beam)
      if (warp == sw) {
        StepLists o = step_select_classify_any<S, D, VAR>(B, nR, 0, 1 << 30, lane, norm_l, bucket,
                                                          n, narrow);
        if constexpr (VAR) {
          if (o.nw + o.nn + o.nk == 0 && o.nl > keep)
            o = step_select_classify_any<S, D, true>(B, o.nl, 0, keep, lane, norm_l, bucket, n,
                                                     narrow);
        }
        exp_hi += o.nw + o.nn;
        exp_l1 += o.nk;
        exp_wide += o.nw;
        if (lane == 0) {
          C.ctl[0] = o.nw;
          C.ctl[1] = o.nn;
          C.ctl[2] = o.nk;
          C.ctl[3] = o.nl;
        }
      }
      __syncthreads();
      for (int step = 0; step < 32; ++step) {
        const int nw = C.ctl[0], nhi = nw + C.ctl[1], nx = nhi + C.ctl[2], nl = C.ctl[3];
        if (nx == 0) {  // CTA-uniform: every frontier node is a key (or a bucket)
          nf = nl;
          break;
        }
        // left children over the CTA's row groups: int32 rows, int16 rows, key rows (and an L2
        // prefetch of the rows the next step may need)
        for (int base = 0; base < nw; base += NG * UW)
          cta_child_pass<0, UW, S, D, NWC>(B, Th, Kh, q, base, nw, warp, gg, sub, n, narrow, bucket);
        if constexpr (kNarrow)
          for (int base = nw; base < nhi; base += NG * UN)
            cta_child_pass<1, UN, S, D, NWC>(B, Th, Kh, q, base, nhi, warp, gg, sub, n, narrow, bucket);
        for (int base = nhi; base < nx; base += NG * UK)
          cta_child_pass<2, UK, S, D, NWC>(B, Th, Kh, q, base, nx, warp, gg, sub, n, narrow, bucket);
        __syncthreads();
        if (warp == sw) {
          const StepLists o = step_select_classify_any<S, D, VAR>(B, nl, nx, keep, lane, norm_l,
                                                                  bucket, n, narrow);
          exp_hi += o.nw + o.nn;
          exp_l1 += o.nk;
          exp_wide += o.nw;
          if (lane == 0) {
            C.ctl[0] = o.nw;
            C.ctl[1] = o.nn;
            C.ctl[2] = o.nk;
            C.ctl[3] = o.nl;
          }
        }
        __syncthreads();
      }
      if constexpr (VAR) {
        if (bucket > 0) {
          __syncthreads();  // every warp has read ctl before warp 0 rewrites it
          if (warp == sw) {
            nf = expand_buckets<S, D>(B, nf, Kh, q, lane);
            if (lane == 0) C.ctl[4] = nf;
          }
          __syncthreads();
          nf = C.ctl[4];
        }
      }
    }

    // ---- window key scores (with the predictor they were taken in phase 1)
    if constexpr (kAttend && !kUsesW) {
      constexpr int UWIN = (kMaxWindow + NG - 1) / NG;
#pragma unroll
      for (int u = 0; u < UWIN; ++u) {
        const int x = u * NG + gg;
        if (u * NG < nsel_win) {  // CTA-uniform
          int xp[4] = {0, 0, 0, 0};
          if (x < nsel_win) ld_key<D>(Kh + (long long)(i - x) * D, sub, xp);
          const int s = group_sum<int, TPR>(dot_key(q, xp));
          if (x < nsel_win && sub == 0) B.winsc[x] = s;
        }
      }
    }
    __syncthreads();

    // ---- outputs of the route (warp 0)
    const int count = nsel_win + nf;
    if (warp == sw) {
      if (lane == 0) {
        if (a.count_out) a.count_out[qi] = count;
        if (a.exp_out) {
          a.exp_out[3 * qi] = exp_hi;
          a.exp_out[3 * qi + 1] = exp_l1;
          a.exp_out[3 * qi + 2] = exp_wide;
        }
        if (a.budget_out) a.budget_out[qi] = budget;
      }
      if (a.idx_out)
        write_selection<S>(B, nf, nsel_win, i, a.idx_out + qi * a.max_keys, a.max_keys, lane);
    }

    // ---- 4. exact attention over window + routed keys
    if constexpr (kAttend) {
      if (warp == sw) {
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
        if (lane == 0) C.inv = 1.f / den;
      }
      __syncthreads();
      const int per = (count + NWC - 1) / NWC;
      const int k0 = min(count, warp * per);
      gather_values_part<D, 8>(B.selk, B.selp, k0, min(count, k0 + per),
                               a.V + bh * (long long)n * D, lane, C.opart[warp]);
      __syncthreads();
      const float inv = C.inv;
      for (int t = threadIdx.x; t < D; t += NWC * 32) {
        float o = 0.f;
#pragma unroll
        for (int ww = 0; ww < NWC; ++ww) o += C.opart[ww][t];
        a.out[qi * D + t] = o * inv;
      }
    }
  }
}

namespace {

// Resident CTAs per SM of one instantiation (cached per device) and, with `launch`, the launch.
template <typename S, int D, int MODE, bool VAR, int NWC>
cudaError_t cta_mode(const QueryArgs& a, cudaStream_t st, bool launch, long long* per_sm_out) {
  constexpr size_t smem = CtaSmem<S, D, MODE, NWC>::bytes;
  auto kern = cta_query_kernel<S, D, MODE, VAR, NWC>;
  static thread_local int cached_dev = -1;
  static thread_local int per_sm = 0, sms = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != cached_dev) {
    if (smem > 48 * 1024) {
      const cudaError_t e =
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
      if (e != cudaSuccess) return e;
    }
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int b = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kern, NWC * 32, smem);
    per_sm = b > 0 ? b : 1;
    cached_dev = dev;
  }
  const long long cap = (long long)sms * per_sm;
  if (per_sm_out) *per_sm_out = cap;
  if (!launch) return cudaSuccess;
  const int blocks = int(a.num_queries < cap ? a.num_queries : cap);
  if (blocks <= 0) return cudaSuccess;
  kern<<<blocks, NWC * 32, smem, st>>>(a);
  return cudaGetLastError();
}

// Four warps per query while every query fits at once that way; else two while they fit; else,
// when `forced` is false, nothing is launched (*launched = false: the caller takes the
// throughput shape); when forced, four warps per query in several waves.
template <typename S, int D, int MODE>
cudaError_t cta_dispatch(const QueryArgs& a, cudaStream_t st, bool forced, bool* launched) {
  const bool var = MODE != kPredictOnly && (a.norm_l != 0 || a.bucket != 0);
  long long cap4 = 0;
  cudaError_t e = var ? cta_mode<S, D, MODE, true, kCtaWarps>(a, st, false, &cap4)
                      : cta_mode<S, D, MODE, false, kCtaWarps>(a, st, false, &cap4);
  if (e != cudaSuccess) return e;
  *launched = true;
  if (a.num_queries <= cap4 || var) {
    if (a.num_queries > cap4 && !forced) {
      *launched = false;
      return cudaSuccess;
    }
    return var ? cta_mode<S, D, MODE, true, kCtaWarps>(a, st, true, nullptr)
               : cta_mode<S, D, MODE, false, kCtaWarps>(a, st, true, nullptr);
  }
  long long cap2 = 0;
  e = cta_mode<S, D, MODE, false, kCtaWarpsWide>(a, st, false, &cap2);
  if (e != cudaSuccess) return e;
  if (a.num_queries <= cap2) return cta_mode<S, D, MODE, false, kCtaWarpsWide>(a, st, true, nullptr);
  if (!forced) {
    *launched = false;
    return cudaSuccess;
  }
  return cta_mode<S, D, MODE, false, kCtaWarps>(a, st, true, nullptr);
}

template <int MODE>
cudaError_t dispatch_cta(const QueryArgs& a, int d, int score_bits, cudaStream_t st, bool forced,
                         bool* launched) {
  if (d == 64)
    return score_bits == 32 ? cta_dispatch<int, 64, MODE>(a, st, forced, launched)
                            : cta_dispatch<long long, 64, MODE>(a, st, forced, launched);
  return score_bits == 32 ? cta_dispatch<int, 128, MODE>(a, st, forced, launched)
                          : cta_dispatch<long long, 128, MODE>(a, st, forced, launched);
}

}  // namespace

cudaError_t launch_query_cta(const QueryArgs& a, int d, int score_bits, int mode, bool forced,
                             bool* launched, cudaStream_t st) {
  switch (mode) {
    case kForwardPredict: return dispatch_cta<kForwardPredict>(a, d, score_bits, st, forced, launched);
    case kForwardOverride: return dispatch_cta<kForwardOverride>(a, d, score_bits, st, forced, launched);
    case kRouteOnly: return dispatch_cta<kRouteOnly>(a, d, score_bits, st, forced, launched);
    default: return dispatch_cta<kPredictOnly>(a, d, score_bits, st, forced, launched);
  }
}

}  // namespace alhr
