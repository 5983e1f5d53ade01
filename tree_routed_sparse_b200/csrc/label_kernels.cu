// label_kernels.cu -- phase-2 labels of ALHR on sm_100a: the top-k keys of every query's dense
// causal attention row.
//
// README of ALHR, section "Training stage", Phase 2: the dense teacher's attention matrix is
// read and the top-k keys of every query are labelled; section "Results and Variables": k = 16.
// Softmax keeps the order of the scores, so the labels are the k largest exact q . k over the
// causal keys t <= i, equal scores to the lower position.
//
// One CTA of 4 warps takes 128 queries of one (b,h). For every 64-key tile up to the tile's
// last query position, the scores Q_tile . K_tile^T (int8 x int8 -> int32, exact) are computed by
// the 5th-generation tensor core (tcgen05.mma kind::i8, M = 128, N = 64, K = 32 per instruction)
// into one of two 128 x 64 int32 accumulators in tensor memory, so that the next tile's cp.async
// load and MMA run while this one is scanned; thread t reads row t of the accumulator
// (tcgen05.ld, one TMEM lane per thread) 32 columns at a time, queues the columns that beat its
// 16th best in shared memory, and inserts the queued ones in deferred rounds into a sorted
// 16-entry list held in registers. Operand tiles are staged with cp.async in the no-swizzle K-major
// core-matrix layout (8 rows x 16 bytes per 128-byte core matrix). Every wait on the MMA's
// mbarrier is bounded; on timeout the CTA stops, sets ALHR_DEVERR_TIMEOUT, writes none of its
// rows, waits (bounded) for the one MMA that can still be in flight and frees its tensor memory.
#include <climits>
#include <cstdint>
#include <cuda_runtime.h>

#include "alhr_device.cuh"
#include "internal.h"

namespace alhr {

namespace {

constexpr int kLT = 128;          // queries per CTA tile (M)
constexpr int kNT = 64;           // keys per key tile (N): two accumulators in flight
constexpr int kLThreads = 128;    // warp w reads TMEM lanes 32w .. 32w+31: one query row each
constexpr int kListK = 16;        // labels kept per query (k <= 16 is returned)
constexpr int kTmemCols = 128;    // two 128 x 64 int32 accumulators
constexpr uint32_t kWaitLimit = 1u << 24;  // bounded mbarrier polling

template <int D>
struct LabelSmem {
  static constexpr int q_bytes = kLT * D;                     // int8 query tile
  static constexpr int k_bytes = kNT * D;                     // one int8 key tile
  static constexpr int q_off = 0;
  static constexpr int k_off = q_bytes;                       // two key tiles
  // Requested size: at most 4 CTAs per SM (3 at d = 128), so that their accumulators (128
  // columns each) fit the 512 columns of tensor memory and no allocation ever waits on another
  // CTA.
  static constexpr int bytes = (D == 64 ? 56 : 74) * 1024 - 64;
  static constexpr int misc_bytes = 64;
  static constexpr int row_off = q_bytes + 2 * k_bytes;       // [128][36] int32: a chunk per row
  static constexpr int queue_off = row_off + kLThreads * 36 * 4;  // [kQueue][128] int32
  // candidates queued per thread before they are inserted (at least two chunks' worth)
  static constexpr int kQueue = (bytes - misc_bytes - queue_off) / (kLThreads * 4);
  static constexpr int misc_off = queue_off + kQueue * kLThreads * 4;
  static constexpr int used = misc_off + misc_bytes;
  static_assert(kQueue >= 40, "label queue");
  static_assert(used <= bytes, "label kernel shared memory");
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Shared-memory matrix descriptor of tcgen05 (no swizzle): start address, leading byte offset
// (between the 16-byte column blocks of a K-major tile), stride byte offset (between 8-row
// groups), descriptor version 1 at bits 46-47, base offset 0, no swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::i8: int32 accumulator, signed int8 A and B, both
// K-major, N >> 3 at bits 17-22, M >> 4 at bits 24-28.
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(kNT >> 3) << 17) |
                              (static_cast<uint32_t>(kLT >> 4) << 24);

// Byte offset of (row, byte column kb) of an R x D int8 tile in the core-matrix layout.
template <int D>
__device__ __forceinline__ int core_offset(int row, int kb) {
  return ((row >> 3) * (D / 16) + (kb >> 4)) * 128 + (row & 7) * 16 + (kb & 15);
}

// cp.async of a 16-byte row piece; src_bytes = 0 fills zeros (rows outside the matrix).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}

template <int D, int ROWS>
__device__ __forceinline__ void load_tile(unsigned char* tile, const int8_t* base, int first_row,
                                          int valid_rows, int tid) {
  constexpr int CPR = D / 16;  // 16-byte chunks per row
  for (int c = tid; c < ROWS * CPR; c += kLThreads) {
    const int r = c / CPR, kc = c - r * CPR;
    const bool ok = r < valid_rows;
    const int8_t* src = ok ? base + (static_cast<long long>(first_row) + r) * D + kc * 16 : base;
    cp_async16(smem_u32(tile + core_offset<D>(r, kc * 16)), src, ok ? 16 : 0);
  }
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t mbar, uint32_t phase) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(mbar), "r"(phase)
      : "memory");
  return done != 0;
}

// Insert (v, key) into the list sorted by score (descending); v beats the 16th entry, and key
// is larger than every key in the list, so an equal score stays below the older entry.
__device__ __forceinline__ void list_insert(int (&s)[kListK], int (&ix)[kListK], int v, int key) {
#pragma unroll
  for (int j = kListK - 1; j >= 1; --j) {
    const bool up = v > s[j - 1];
    const bool here = !up && v > s[j];
    s[j] = up ? s[j - 1] : (here ? v : s[j]);
    ix[j] = up ? ix[j - 1] : (here ? key : ix[j]);
  }
  const bool top = v > s[0];
  s[0] = top ? v : s[0];
  ix[0] = top ? key : ix[0];
}

// Candidates are queued in shared memory as score * 512 + (key - epoch), epoch a multiple of
// 512 keys: |score| <= 128 * 128 * 128 = 2^21, so the word never overflows. They are inserted
// in rounds (one per queued entry of the fullest lane of the warp), and only when the queue could
// overflow or the 512-key epoch ends: rows add candidates rarely once their list is full, and a
// round serves every lane at once, so deferring rounds saves most of them.
constexpr int kEpochKeys = 512;

// Queue the columns of 32 scores that beat the row's 16th best as of the last insertion round.
// lim: columns j <= lim are causal keys of this row (lim >= 31: all of them).
// The candidates are found as a bit mask (two instructions per score); the chunk is parked in the
// thread's row of shared memory so that only the candidates are read back and queued.
__device__ __forceinline__ int* queue_chunk(const uint32_t (&v)[32], int lim, int T, int key0,
                                            int* qp, int* rowp) {
  unsigned mask = 0u;
#pragma unroll
  for (int j = 0; j < 32; ++j)
    if (static_cast<int>(v[j]) > T) mask |= 1u << j;
  if (lim < 31) mask &= lim < 0 ? 0u : ((2u << lim) - 1u);
  int4* r4 = reinterpret_cast<int4*>(rowp);
#pragma unroll
  for (int j = 0; j < 8; ++j)
    r4[j] = make_int4(static_cast<int>(v[4 * j]), static_cast<int>(v[4 * j + 1]),
                      static_cast<int>(v[4 * j + 2]), static_cast<int>(v[4 * j + 3]));
  while (mask) {
    const int j = __ffs(mask) - 1;
    mask &= mask - 1u;
    *qp = rowp[j] * 512 + key0 + j;
    qp += kLThreads;
  }
  return qp;
}

// Insert this warp's queued candidates into the lists and empty the queues.
__device__ __forceinline__ int* flush_queue(int* qbase, int* qp, int epoch, int (&s)[kListK],
                                            int (&ix)[kListK]) {
  const int cnt = static_cast<int>(qp - qbase) / kLThreads;
  const int rounds = __reduce_max_sync(0xffffffffu, cnt);
  for (int e = 0; e < rounds; ++e) {
    if (e < cnt) {
      const int p = qbase[e * kLThreads];
      const int sc = p >> 9;  // floor division by 512: the key offset is the low 9 bits
      if (sc > s[kListK - 1]) list_insert(s, ix, sc, epoch + (p & (kEpochKeys - 1)));
    }
  }
  return qbase;
}

template <int D>
__global__ void __launch_bounds__(kLThreads, D == 64 ? 4 : 3)
    topk_label_kernel(const int8_t* __restrict__ Q, const int8_t* __restrict__ K,
                      int32_t* __restrict__ labels, int32_t* __restrict__ scores, int n,
                      int q_start, int nq, int k, long long bh_count, int tiles_per_head,
                      uint32_t* dev_err) {
  using L = LabelSmem<D>;
  extern __shared__ __align__(1024) unsigned char lsm[];
  unsigned char* sQ = lsm + L::q_off;
  unsigned char* sK = lsm + L::k_off;  // key tile b at sK + b * k_bytes
  int* queue = reinterpret_cast<int*>(lsm + L::queue_off);
  int* rowp = reinterpret_cast<int*>(lsm + L::row_off) + threadIdx.x * 36;
  uint64_t* mbar = reinterpret_cast<uint64_t*>(lsm + L::misc_off);  // two barriers
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lsm + L::misc_off + 16);
  int* abort_flag = reinterpret_cast<int*>(lsm + L::misc_off + 32);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  // the longest tiles (the last queries of every head) first
  const long long bid = blockIdx.x;
  const int qt = tiles_per_head - 1 - static_cast<int>(bid / bh_count);
  const long long bh = bid - (bid / bh_count) * bh_count;
  const int q0 = qt * kLT;
  const int rows = min(kLT, nq - q0);
  const int8_t* Qh = Q + bh * static_cast<long long>(nq) * D;
  const int8_t* Kh = K + bh * static_cast<long long>(n) * D;
  const int i_last = q_start + q0 + rows - 1;
  const int ntiles = i_last / kNT + 1;  // key tiles [0, 64), [64, 128), ... up to i_last

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(mbar)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_u32(mbar + 1)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
    *abort_flag = 0;
  }
  // group 0: the query tile and key tile 0; group 1: key tile 1
  load_tile<D, kLT>(sQ, Qh, q0, rows, tid);
  load_tile<D, kNT>(sK, Kh, 0, min(kNT, n), tid);
  if (ntiles > 1) load_tile<D, kNT>(sK + L::k_bytes, Kh, kNT, min(kNT, n - kNT), tid);
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  const uint32_t tmem = *tmem_slot;

  const int r = tid;  // this thread's query row in the tile (= its TMEM lane)
  const bool row_ok = r < rows;
  const int i = q_start + q0 + r;  // its position
  int s[kListK], ix[kListK];
#pragma unroll
  for (int j = 0; j < kListK; ++j) {
    s[j] = INT_MIN;
    ix[j] = -1;
  }

  const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK);
  constexpr uint32_t kLbo = 128, kSbo = 8 * D;
  // MMA of key tile t into accumulator t & 1, arriving on barrier t & 1 (thread 0)
  auto issue_mma = [&](int t) {
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    const uint32_t kb = ka + (t & 1) * L::k_bytes;
#pragma unroll
    for (int ks = 0; ks < D / 32; ++ks) {
      const uint64_t adesc = smem_desc(qa + ks * 256, kLbo, kSbo);
      const uint64_t bdesc = smem_desc(kb + ks * 256, kLbo, kSbo);
      asm volatile(
          "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
          " tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(
              tmem + (t & 1) * kNT),
          "l"(adesc), "l"(bdesc), "r"(kIdescI8), "r"(ks)
          : "memory");
    }
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
            smem_u32(mbar + (t & 1)))
        : "memory");
  };

  // prologue: wait for the query tile and key tile 0, start their MMA
  if (ntiles > 1) asm volatile("cp.async.wait_group 1;\n" ::: "memory");
  else asm volatile("cp.async.wait_group 0;\n" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
  __syncthreads();
  if (tid == 0) issue_mma(0);

  uint32_t phases = 0u;  // bit b: the parity to wait for on barrier b
  int* const qbase = queue + tid;  // this thread's queue column
  int* qp = qbase;                 // next free entry
  int epoch = 0;                   // key base of the queued entries
  int drain_b = -1;                // after an abort: the barrier of the MMA still in flight
  uint32_t drain_parity = 0u;
  for (int t = 0; t < ntiles; ++t) {
    const int b = t & 1;
    // 1. MMA t done (as this thread sees it): its accumulator is ready, its key buffer free
    bool ok = false;
    for (uint32_t w = 0; w < kWaitLimit && !ok; ++w)
      ok = mbar_try_wait(smem_u32(mbar + b), (phases >> b) & 1u);
    phases ^= 1u << b;
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
    // 2. key tile t + 2 into the freed buffer (its own cp.async group)
    if (ok && t + 2 < ntiles) {
      const int k2 = (t + 2) * kNT;
      load_tile<D, kNT>(sK + b * L::k_bytes, Kh, k2, min(kNT, n - k2), tid);
    }
    // 3. the tile's one CTA barrier: every thread's copies of key tile t + 1 have landed, every
    //    thread has read accumulator (t + 1) & 1 (tile t - 1, in the previous iteration), and
    //    a wait that ran out on any thread stops all of them here together
    if (t + 1 < ntiles) {
      if (t + 2 < ntiles) asm volatile("cp.async.wait_group 1;\n" ::: "memory");
      else asm volatile("cp.async.wait_group 0;\n" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
    }
    if (__syncthreads_or(!ok)) {
      if (tid == 0) {
        *abort_flag = 1;
        if (dev_err) atomicOr(dev_err, ALHR_DEVERR_TIMEOUT);
      }
      drain_b = b;
      drain_parity = ((phases >> b) & 1u) ^ 1u;  // the parity waited for above
      break;
    }
    if (t + 1 < ntiles && tid == 0) issue_mma(t + 1);
    // 4. this thread's row of scores for tile t, 64 columns as two loads of 32
    uint32_t v0[32], v1[32];
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16) + b * kNT;
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(v0[0]), "=r"(v0[1]), "=r"(v0[2]), "=r"(v0[3]), "=r"(v0[4]), "=r"(v0[5]),
          "=r"(v0[6]), "=r"(v0[7]), "=r"(v0[8]), "=r"(v0[9]), "=r"(v0[10]), "=r"(v0[11]),
          "=r"(v0[12]), "=r"(v0[13]), "=r"(v0[14]), "=r"(v0[15]), "=r"(v0[16]), "=r"(v0[17]),
          "=r"(v0[18]), "=r"(v0[19]), "=r"(v0[20]), "=r"(v0[21]), "=r"(v0[22]), "=r"(v0[23]),
          "=r"(v0[24]), "=r"(v0[25]), "=r"(v0[26]), "=r"(v0[27]), "=r"(v0[28]), "=r"(v0[29]),
          "=r"(v0[30]), "=r"(v0[31])
        : "r"(taddr)
        : "memory");
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
        : "=r"(v1[0]), "=r"(v1[1]), "=r"(v1[2]), "=r"(v1[3]), "=r"(v1[4]), "=r"(v1[5]),
          "=r"(v1[6]), "=r"(v1[7]), "=r"(v1[8]), "=r"(v1[9]), "=r"(v1[10]), "=r"(v1[11]),
          "=r"(v1[12]), "=r"(v1[13]), "=r"(v1[14]), "=r"(v1[15]), "=r"(v1[16]), "=r"(v1[17]),
          "=r"(v1[18]), "=r"(v1[19]), "=r"(v1[20]), "=r"(v1[21]), "=r"(v1[22]), "=r"(v1[23]),
          "=r"(v1[24]), "=r"(v1[25]), "=r"(v1[26]), "=r"(v1[27]), "=r"(v1[28]), "=r"(v1[29]),
          "=r"(v1[30]), "=r"(v1[31])
        : "r"(taddr + 32)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
    const int k0 = t * kNT;
    const int lim = row_ok ? i - k0 : -1;  // columns j <= lim are causal keys of this row
    if (k0 - epoch >= kEpochKeys) {        // the queued key offsets are relative to the epoch
      qp = flush_queue(qbase, qp, epoch, s, ix);
      epoch = k0;
    }
    if (__any_sync(0xffffffffu, qp - qbase > (L::kQueue - 32) * kLThreads))
      qp = flush_queue(qbase, qp, epoch, s, ix);
    qp = queue_chunk(v0, lim, s[kListK - 1], k0 - epoch, qp, rowp);
    if (__any_sync(0xffffffffu, qp - qbase > (L::kQueue - 32) * kLThreads))
      qp = flush_queue(qbase, qp, epoch, s, ix);
    qp = queue_chunk(v1, lim - 32, s[kListK - 1], k0 + 32 - epoch, qp, rowp);
    // 5. accumulator t & 1 is read; the next iteration's barrier orders this before the MMA of
    //    tile t + 2 overwrites it
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  }

  qp = flush_queue(qbase, qp, epoch, s, ix);
  if (row_ok && !*abort_flag) {
    const long long o = (bh * nq + q0 + r) * static_cast<long long>(k);
#pragma unroll
    for (int j = 0; j < kListK; ++j) {
      if (j < k) {
        labels[o + j] = ix[j];
        if (scores) scores[o + j] = ix[j] >= 0 ? s[j] : 0;
      }
    }
  }
  asm volatile("cp.async.wait_all;\n" ::: "memory");  // nothing in flight after an abort
  if (drain_b >= 0) {
    // After an abort exactly one committed MMA can still be writing tensor memory: the MMA of
    // tile t, whose wait ran out. (MMA t + 1 is issued only after the tile's barrier has agreed
    // that no wait ran out, and the wait of every earlier tile succeeded on every thread, so
    // their MMAs are complete.) Wait for its commit once more, bounded like every wait, before
    // the accumulators are freed below; once the commit has been observed nothing targets them.
    // Should even this wait run out, the tensor core has lost a committed MMA: the memory is
    // still freed (a CTA must free what it allocated before it exits, and a leaked allocation
    // would starve the CTAs that come after it on this SM), and ALHR_DEVERR_TIMEOUT, already
    // set, tells the caller that no output of this launch can be trusted.
    bool done = false;
    for (uint32_t w = 0; w < kWaitLimit && !done; ++w)
      done = mbar_try_wait(smem_u32(mbar + drain_b), drain_parity);
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
}

template <int D>
cudaError_t launch_labels_d(const int8_t* Q, const int8_t* K, int32_t* labels, int32_t* scores,
                            int n, int q_start, int nq, int k, long long bh, uint32_t* dev_err,
                            cudaStream_t st) {
  static thread_local bool configured[128] = {};  // per host thread: no shared state
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 128 || !configured[dev]) {
    const cudaError_t e = cudaFuncSetAttribute(
        topk_label_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, LabelSmem<D>::bytes);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 128) configured[dev] = true;
  }
  const int tiles = (nq + kLT - 1) / kLT;
  const long long grid = bh * tiles;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  topk_label_kernel<D><<<static_cast<unsigned>(grid), kLThreads, LabelSmem<D>::bytes, st>>>(
      Q, K, labels, scores, n, q_start, nq, k, bh, tiles, dev_err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_topk_labels(const int8_t* Q, const int8_t* K, int32_t* labels,
                               int32_t* scores, int n, int d, int q_start, int nq, int k,
                               long long bh, uint32_t* dev_err, cudaStream_t st) {
  if (nq == 0 || bh == 0) return cudaSuccess;
  return d == 64 ? launch_labels_d<64>(Q, K, labels, scores, n, q_start, nq, k, bh, dev_err, st)
                 : launch_labels_d<128>(Q, K, labels, scores, n, q_start, nq, k, bh, dev_err, st);
}

}  // namespace alhr
