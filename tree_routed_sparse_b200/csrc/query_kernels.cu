// query_kernels.cu -- warp-per-query kernels of the ALHR inference path (sm_100a).
//
// Follows the README of ALHR ("Adaptive learnable Hierarchical routing"), section "Inference
// stage": budget predictor on the query and the causal key sum, the own key and its neighbour
// window first, then a budget-limited descent of the past-only forest, then exact attention
// over the selected keys.
//
// Per query (one warp):
//   1. q, the window rows i, i-1, ..., i-w+1 (key rows: scores for attention, and G_i) and the
//      roots of [0, i-w] (tree rows: first frontier, and G_i) -- G_i = roots + window costs no
//      extra bytes;
//   2. budget: predictor logits over 32 classes from W in shared memory (int64, ties -> lower
//      class), or the given budget;
//   3. descent: every step reads only the LEFT child of each expanded node; the right child's
//      score is parent - left (exact in integers), so a step costs one row per expansion;
//      keep-the-best-r is an exact bisection on the integer score (select_top_r);
//   4. routed leaves keep the scores computed during the descent, so their key rows are never
//      read again; attention gathers only the value rows.
#include <cuda_runtime.h>

#include "alhr_device.cuh"
#include "internal.h"

namespace alhr {

enum Mode : int { kForwardPredict = 0, kForwardOverride = 1, kRouteOnly = 2, kPredictOnly = 3 };

template <typename S, int DPL, int MODE>
__global__ void __launch_bounds__(kWarps * 32) query_kernel(const QueryArgs a) {
  constexpr int D = 32 * DPL;
  constexpr bool kUsesW = (MODE == kForwardPredict || MODE == kPredictOnly);
  constexpr bool kDescend = (MODE != kPredictOnly);
  constexpr bool kAttend = (MODE == kForwardPredict || MODE == kForwardOverride);
  constexpr int RB = (DPL == 2) ? 32 : 16;  // rows per expansion batch (64 registers of rows)

  __shared__ __align__(16) int8_t sW[kUsesW ? 64 * D : 16];
  __shared__ WarpBuf<S> wbuf[kWarps];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  if constexpr (kUsesW) {
    for (int k = threadIdx.x; k < 64 * D / 16; k += blockDim.x)
      reinterpret_cast<int4*>(sW)[k] = __ldg(reinterpret_cast<const int4*>(a.W) + k);
    __syncthreads();
  }
  WarpBuf<S>& B = wbuf[warp];
  const int n = a.n;
  const int w = a.window;
  const long long stride = (long long)gridDim.x * kWarps;

  for (long long g = (long long)blockIdx.x * kWarps + warp; g < a.num_queries; g += stride) {
    const long long bh = g / a.nq;
    const int i = a.q_start + int(g - bh * a.nq);
    const int8_t* Kh = a.K + bh * (long long)n * D;
    const int32_t* Nh = a.nodes + bh * (long long)(n - 1) * D;

    int qv[DPL];
    load_i8<DPL>(a.Q + g * D, lane, qv);
    {
      bool bad = false;
#pragma unroll
      for (int e = 0; e < DPL; ++e) bad |= (qv[e] > a.value_bound) | (qv[e] < -a.value_bound);
      if (__any_sync(kFull, bad) && lane == 0) flag(a.dev_err, ALHR_DEVERR_VALUE_RANGE);
    }

    const int nwin = min(w, i + 1);  // keys of the window
    const int M = i - w + 1;         // keys before the window: [0, M)
    const int nr = M > 0 ? __popc(M) : 0;

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
    if constexpr (!kUsesW) settle(__ldg(a.budget_in + g));

    int G[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) G[e] = 0;

    // ---- window rows: lane x ends with the score of key i - x. The predictor needs every
    // window key (G_i); with a given budget only the selected ones are read.
    S win_score = 0;
    if constexpr (kUsesW || kAttend) {
      const int nload = kUsesW ? nwin : nsel_win;
      for (int c0 = 0; c0 < nload; c0 += 16) {
        int v[16][DPL];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          if (c0 + k < nload) {
            load_i8<DPL>(Kh + (long long)(i - c0 - k) * D, lane, v[k]);
          } else {
#pragma unroll
            for (int e = 0; e < DPL; ++e) v[k][e] = 0;
          }
        }
        S part[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          part[k] = lane_dot<S, DPL>(qv, v[k]);
          if constexpr (kUsesW) {
#pragma unroll
            for (int e = 0; e < DPL; ++e) G[e] += v[k][e];
          }
        }
        const S res = transpose_reduce<S, 16>(part, lane);
        if ((lane >> 4) == (c0 >> 4)) win_score = res;
      }
    }

    // ---- roots of [0, M), largest first: lane k ends with root k
    S root_score = 0;
    int root_desc = 0;
    const bool load_roots = kUsesW || (r > 0 && M > 0);
    if (load_roots) {
      int rest = M;
      for (int c0 = 0; c0 < nr; c0 += 16) {
        int v[16][DPL];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          if (c0 + k < nr) {
            const int lvl = 31 - __clz(rest);
            rest ^= 1 << lvl;
            const int start = M & ~((2 << lvl) - 1);
            if (lane == c0 + k) root_desc = make_desc(start, lvl);
            load_node<DPL>(Kh, Nh, n, lvl, start >> lvl, lane, v[k]);
          } else {
#pragma unroll
            for (int e = 0; e < DPL; ++e) v[k][e] = 0;
          }
        }
        S part[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          part[k] = lane_dot<S, DPL>(qv, v[k]);
          if constexpr (kUsesW) {
#pragma unroll
            for (int e = 0; e < DPL; ++e) G[e] += v[k][e];
          }
        }
        const S res = transpose_reduce<S, 16>(part, lane);
        if ((lane >> 4) == (c0 >> 4)) root_score = res;
      }
    }

    // ---- budget predictor: logit_c = W[c][:d] . q + W[c][d:] . G_i, argmax, ties -> lower c
    if constexpr (kUsesW) {
      long long logit = 0;
#pragma unroll
      for (int c0 = 0; c0 < 32; c0 += 16) {
        long long part[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const int8_t* wr = sW + (c0 + k) * 2 * D;
          int wq[DPL], wg[DPL];
          if constexpr (DPL == 2) {
            const int tq = reinterpret_cast<const short*>(wr)[lane];
            const int tg = reinterpret_cast<const short*>(wr + D)[lane];
            wq[0] = (tq << 24) >> 24; wq[1] = (tq << 16) >> 24;
            wg[0] = (tg << 24) >> 24; wg[1] = (tg << 16) >> 24;
          } else {
            const int tq = reinterpret_cast<const int*>(wr)[lane];
            const int tg = reinterpret_cast<const int*>(wr + D)[lane];
            wq[0] = (tq << 24) >> 24; wq[1] = (tq << 16) >> 24;
            wq[2] = (tq << 8) >> 24;  wq[3] = tq >> 24;
            wg[0] = (tg << 24) >> 24; wg[1] = (tg << 16) >> 24;
            wg[2] = (tg << 8) >> 24;  wg[3] = tg >> 24;
          }
          long long s = 0;
#pragma unroll
          for (int e = 0; e < DPL; ++e) s += (long long)(wq[e] * qv[e]) + (long long)wg[e] * G[e];
          part[k] = s;
        }
        const long long res = transpose_reduce<long long, 16>(part, lane);
        if ((lane >> 4) == (c0 >> 4)) logit = res;
      }
      // largest logit, then lowest class: pack (logit, 31 - class) and take the maximum
      const long long key = warp_max<long long>(logit * 32 + (31 - lane));
      const int cls = 31 - int(key & 31);
      settle(3 * (cls + 1));
    }

    if constexpr (MODE == kPredictOnly) {
      if (lane == 0) a.budget_out[g] = budget;
      continue;
    }

    // ---- descent of the past-only forest
    int nf = 0, exp_hi = 0, exp_l1 = 0;
    if (kDescend && r > 0 && M > 0) {
      __syncwarp();
      if (lane < nr) {
        B.cdesc[lane] = root_desc;
        B.cscore[lane] = root_score;
      }
      nf = nr;
      for (int step = 0; step < 32; ++step) {
        __syncwarp();
        int fd[kFrontSlots];
        S fs[kFrontSlots];
        bool inner[kFrontSlots], leaf[kFrontSlots];
        int nx = 0, nl = 0, nhi = 0;
        unsigned bi[kFrontSlots], bl[kFrontSlots];
#pragma unroll
        for (int s = 0; s < kFrontSlots; ++s) {
          const int e = lane + 32 * s;
          const bool ok = e < nf;
          fd[s] = ok ? B.cdesc[e] : 0;
          fs[s] = ok ? B.cscore[e] : S(0);
          inner[s] = ok && desc_level(fd[s]) > 0;
          leaf[s] = ok && !inner[s];
          bi[s] = __ballot_sync(kFull, inner[s]);
          bl[s] = __ballot_sync(kFull, leaf[s]);
          nx += __popc(bi[s]);
          nl += __popc(bl[s]);
          nhi += warp_count(inner[s] && desc_level(fd[s]) >= 2);
        }
        if (nx == 0) break;
        exp_hi += nhi;
        exp_l1 += nx - nhi;
        __syncwarp();
        {
          int xo = 0, lo = 0;
#pragma unroll
          for (int s = 0; s < kFrontSlots; ++s) {
            const unsigned below = lanemask_lt(lane);
            if (inner[s]) {
              const int pos = xo + __popc(bi[s] & below);
              B.xdesc[pos] = fd[s];
              B.xscore[pos] = fs[s];
            }
            if (leaf[s]) {
              const int pos = lo + __popc(bl[s] & below);
              B.cdesc[pos] = fd[s];
              B.cscore[pos] = fs[s];
            }
            xo += __popc(bi[s]);
            lo += __popc(bl[s]);
          }
        }
        __syncwarp();
        for (int base = 0; base < nx; base += RB) {
          int v[RB][DPL];
#pragma unroll
          for (int k = 0; k < RB; ++k) {
            if (base + k < nx) {
              const int pd = B.xdesc[base + k];
              const int cl = desc_level(pd) - 1;
              load_node<DPL>(Kh, Nh, n, cl, desc_start(pd) >> cl, lane, v[k]);
            } else {
#pragma unroll
              for (int e = 0; e < DPL; ++e) v[k][e] = 0;
            }
          }
          S part[RB];
#pragma unroll
          for (int k = 0; k < RB; ++k) part[k] = lane_dot<S, DPL>(qv, v[k]);
          const S left = transpose_reduce<S, RB>(part, lane);
          const int x = base + lane;
          if (lane < RB && x < nx) {
            const int pd = B.xdesc[x];
            const S ps = B.xscore[x];
            const int cl = desc_level(pd) - 1;
            const int st = desc_start(pd);
            B.cdesc[nl + 2 * x] = make_desc(st, cl);
            B.cscore[nl + 2 * x] = left;
            B.cdesc[nl + 2 * x + 1] = make_desc(st + (1 << cl), cl);
            B.cscore[nl + 2 * x + 1] = ps - left;
          }
        }
        const int C = nl + 2 * nx;
        if (C > r) {
          select_top_r<S>(B, C, r, lane);
          nf = r;
        } else {
          nf = C;
          __syncwarp();
        }
      }
    }
    __syncwarp();

    // ---- optional outputs of the route
    const int count = nsel_win + nf;
    if (a.count_out && lane == 0) a.count_out[g] = count;
    if (a.exp_out && lane == 0) {
      a.exp_out[2 * g] = exp_hi;
      a.exp_out[2 * g + 1] = exp_l1;
    }
    if (a.budget_out && lane == 0) a.budget_out[g] = budget;
    if (a.idx_out) {
      int32_t* io = a.idx_out + g * a.max_keys;
#pragma unroll
      for (int s = 0; s < kFrontSlots; ++s) {
        const int e = lane + 32 * s;
        if (e < nf) {
          const int st = desc_start(B.cdesc[e]);
          int rank = 0;
          for (int f = 0; f < nf; ++f) rank += desc_start(B.cdesc[f]) < st ? 1 : 0;
          io[rank] = st;
        }
      }
      if (lane < nsel_win) io[nf + nsel_win - 1 - lane] = i - lane;
      for (int p = count + lane; p < a.max_keys; p += 32) io[p] = -1;
    }

    // ---- exact attention over window + routed keys
    if constexpr (kAttend) {
      const float scale = a.scale;
      const float sw = lane < nsel_win ? float(win_score) * scale : -INFINITY;
      float sr[kFrontSlots];
      int kr[kFrontSlots];
#pragma unroll
      for (int s = 0; s < kFrontSlots; ++s) {
        const int e = lane + 32 * s;
        sr[s] = e < nf ? float(B.cscore[e]) * scale : -INFINITY;
        kr[s] = e < nf ? desc_start(B.cdesc[e]) : 0;
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
      const uint16_t* Vh = a.V + bh * (long long)n * D;
      float acc[DPL];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
#pragma unroll 4
      for (int x = 0; x < nsel_win; ++x) {
        const float px = __shfl_sync(kFull, pw, x);
        float v[DPL];
        load_bf16<DPL>(Vh + (long long)(i - x) * D, lane, v);
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[e] = fmaf(px, v[e], acc[e]);
      }
#pragma unroll
      for (int s = 0; s < kFrontSlots; ++s) {
        const int cnt = min(32, nf - 32 * s);
#pragma unroll 4
        for (int x = 0; x < cnt; ++x) {
          const float px = __shfl_sync(kFull, pr[s], x);
          const int key = __shfl_sync(kFull, kr[s], x);
          float v[DPL];
          load_bf16<DPL>(Vh + (long long)key * D, lane, v);
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[e] = fmaf(px, v[e], acc[e]);
        }
      }
      const float inv = 1.f / den;
      float* o = a.out + g * D + lane * DPL;
      if constexpr (DPL == 2) {
        *reinterpret_cast<float2*>(o) = make_float2(acc[0] * inv, acc[1] * inv);
      } else {
        *reinterpret_cast<float4*>(o) =
            make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
      }
    }
  }
}

// Exact attention over a given selection (idx, count): key rows for the scores, value rows for
// the sum. Entries outside [0, i] are skipped and flagged.
template <int DPL>
__global__ void __launch_bounds__(kWarps * 32) attend_kernel(const QueryArgs a) {
  constexpr int D = 32 * DPL;
  constexpr int RB = (DPL == 2) ? 32 : 16;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int n = a.n;
  const long long stride = (long long)gridDim.x * kWarps;
  for (long long g = (long long)blockIdx.x * kWarps + warp; g < a.num_queries; g += stride) {
    const long long bh = g / a.nq;
    const int i = a.q_start + int(g - bh * a.nq);
    const int8_t* Kh = a.K + bh * (long long)n * D;
    const uint16_t* Vh = a.V + bh * (long long)n * D;
    int qv[DPL];
    load_i8<DPL>(a.Q + g * D, lane, qv);
    const int cnt = min(__ldg(a.count_in + g), a.max_keys);
    float* o = a.out + g * D + lane * DPL;
    int key[kFrontSlots];
    bool ok[kFrontSlots];
    bool bad = false;
#pragma unroll
    for (int s = 0; s < kFrontSlots; ++s) {
      const int e = lane + 32 * s;
      key[s] = e < cnt ? __ldg(a.idx_in + g * a.max_keys + e) : -1;
      ok[s] = e < cnt && key[s] >= 0 && key[s] <= i;
      bad |= e < cnt && !ok[s];
    }
    if (__any_sync(kFull, bad) && lane == 0) flag(a.dev_err, ALHR_DEVERR_INDEX);
    float sc[kFrontSlots];
#pragma unroll
    for (int s = 0; s < kFrontSlots; ++s) {
      sc[s] = -INFINITY;
#pragma unroll
      for (int h = 0; h < 32 / RB; ++h) {
        const int base = 32 * s + RB * h;
        if (base < cnt) {
          int v[RB][DPL];
#pragma unroll
          for (int k = 0; k < RB; ++k) {
            const int kk = __shfl_sync(kFull, key[s], RB * h + k);
            const bool okk = __shfl_sync(kFull, ok[s], RB * h + k);
            if (okk) {
              load_i8<DPL>(Kh + (long long)kk * D, lane, v[k]);
            } else {
#pragma unroll
              for (int e = 0; e < DPL; ++e) v[k][e] = 0;
            }
          }
          int part[RB];
#pragma unroll
          for (int k = 0; k < RB; ++k) part[k] = lane_dot<int, DPL>(qv, v[k]);
          const int res = transpose_reduce<int, RB>(part, lane);
          if (lane / RB == h && ok[s]) sc[s] = float(res) * a.scale;
        }
      }
    }
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
    float acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
#pragma unroll
    for (int s = 0; s < kFrontSlots; ++s) {
      const int c = min(32, cnt - 32 * s);
#pragma unroll 4
      for (int x = 0; x < c; ++x) {
        const float px = __shfl_sync(kFull, pr[s], x);
        const int kk = __shfl_sync(kFull, key[s], x);
        if (px != 0.f) {
          float v[DPL];
          load_bf16<DPL>(Vh + (long long)kk * D, lane, v);
#pragma unroll
          for (int e = 0; e < DPL; ++e) acc[e] = fmaf(px, v[e], acc[e]);
        }
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    if constexpr (DPL == 2) {
      *reinterpret_cast<float2*>(o) = make_float2(acc[0] * inv, acc[1] * inv);
    } else {
      *reinterpret_cast<float4*>(o) =
          make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    }
  }
}

// ------------------------------------------------------------------ launchers

namespace {

struct Occ {
  int sms = 0;
  int per_sm[20] = {0};
};

template <typename KernelT>
int blocks_for(KernelT kernel, int slot, long long queries) {
  static thread_local int cached_dev = -1;
  static thread_local Occ occ;
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev != cached_dev) {
    occ = Occ{};
    cudaDeviceGetAttribute(&occ.sms, cudaDevAttrMultiProcessorCount, dev);
    cached_dev = dev;
  }
  if (occ.per_sm[slot] == 0) {
    int b = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, kWarps * 32, 0);
    occ.per_sm[slot] = b > 0 ? b : 1;
  }
  const long long need = (queries + kWarps - 1) / kWarps;
  const long long cap = (long long)occ.sms * occ.per_sm[slot];
  return int(need < cap ? need : cap);
}

template <typename S, int DPL, int MODE>
cudaError_t launch_query(const QueryArgs& a, cudaStream_t st) {
  constexpr int slot = (MODE * 2 + (DPL == 4 ? 1 : 0)) * 2 + (sizeof(S) == 8 ? 1 : 0);
  static_assert(slot < 16, "occupancy cache slot");
  auto kern = query_kernel<S, DPL, MODE>;
  const int blocks = blocks_for(kern, slot, a.num_queries);
  if (blocks <= 0) return cudaSuccess;
  kern<<<blocks, kWarps * 32, 0, st>>>(a);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t dispatch_query(const QueryArgs& a, int d, int score_bits, cudaStream_t st) {
  if (d == 64) {
    return score_bits == 32 ? launch_query<int, 2, MODE>(a, st)
                            : launch_query<long long, 2, MODE>(a, st);
  }
  return score_bits == 32 ? launch_query<int, 4, MODE>(a, st)
                          : launch_query<long long, 4, MODE>(a, st);
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

cudaError_t launch_attend(const QueryArgs& a, int d, cudaStream_t st) {
  if (d == 64) {
    const int blocks = blocks_for(attend_kernel<2>, 16, a.num_queries);
    attend_kernel<2><<<blocks, kWarps * 32, 0, st>>>(a);
  } else {
    const int blocks = blocks_for(attend_kernel<4>, 17, a.num_queries);
    attend_kernel<4><<<blocks, kWarps * 32, 0, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace alhr
