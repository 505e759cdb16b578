// Partition kernel on the 5th-generation tensor cores, for 32-head tiles at
// head_dim 128 (large GQA groups and MQA, where the group's QK and PV are dense
// enough -- 32 flop per K/V byte -- to be a real contraction).
//
// Same work unit and result as partition_kernel (pad_partition.cu): one CTA per
// (sequence b, KV head, head tile, partition s), the query heads of the tile
// against tokens [s*P, min((s+1)*P, L_b)) ("perf(rocke): prepare saved paged
// decode bindings once", section "Summary"), every head served from one K/V read
// ("spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm", section "It is a
// mirror of merged work, not new design").  Two CTAs share an SM, so one's
// start, epilogue and split merge overlap the other's streaming.  The
// partition is processed in chunks of 128 tokens:
//
//   producer warp:  TMA of the chunk's K and V, boxes of 8 tokens x 128 head_dim
//                   (two 64-element column blocks, 128-byte swizzle), so that
//                   8-token groups sit 2 KB apart: the canonical tcgen05
//                   operand layout for K (K-major) and for V (MN-major).  The
//                   q rows of the tile arrive the same way.  One K and one V
//                   chunk buffer: K(c+1) streams once S(c) has read K(c), V(c+1)
//                   once PV(c) has read V(c).
//   MMA thread:     S^T[128 tok x 32 heads] = K . Q^T        (tcgen05.mma, TMEM)
//                   O^T[128 d x 32 heads]  += V^T . P^T      (tcgen05.mma, TMEM)
//   softmax warps:  thread i owns token i (TMEM lane i): reads its 32 scores,
//                   lazy running max per head (moves only when a score passes
//                   it by more than 2^8: each thread tests its token and one
//                   barrier-reduce decides; only then the chunk's per-head
//                   maximum, a shuffle transpose-reduce and a 4-warp combine),
//                   weights in fp32 summed per thread, P^T row written to shared
//                   memory (MN-major, 128-byte swizzle) as the B operand of the
//                   PV product.  At the end thread i owns head_dim row i of O^T.
//
// S^T and P^T are double buffered.  A rescale of O^T waits for PV(c-1); a P^T
// buffer is rewritten once PV(c-2) has read it.
//
// Output and split handling are those of partition_kernel: one non-empty
// partition writes bf16 out (+ lse), otherwise fp32 partials and the last CTA of
// the set merges them by log-sum-exp.  Every wait is bounded (error bit 0x4).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "pad_device.cuh"
#include "pad_internal.h"
#include "pad_merge.cuh"

namespace pad {
namespace {

constexpr float kLn2u = 0.69314718055994530942f;
constexpr float kSlack = 8.f;                   // lazy-rescale threshold, log2 units
constexpr uint64_t kWaitNs = 1000000000ull;      // 1 s
constexpr int kChunk = 128;                      // tokens per chunk (MMA M)
constexpr int kHeads = 32;                       // heads per tile (MMA N)
constexpr int kD = 128;                          // head_dim (MMA K of QK, M of PV)
constexpr int kBoxRows = 8;                      // tokens per TMA box
constexpr uint32_t kBoxBytes = kBoxRows * kD * 2;          // 2 KB
constexpr uint32_t kHalfBytes = kChunk * kD * 2;           // K (or V) of a chunk: 32 KB
constexpr uint32_t kQBytes = kHeads * kD * 2;              // 8 KB
constexpr uint32_t kPBytes = kChunk * 128;                 // one P^T buffer: 128 rows of 128 B
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4, kMmaWarp = 5;
constexpr int kUmmaThreads = 6 * 32;

// ---- tcgen05 wrappers (sm_100a) ----------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }
// D(tmem) (+)= A(smem desc) * B(smem desc), bf16 in, fp32 accumulate
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          bool accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Arrive on `bar` once every tcgen05 operation this thread issued so far completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive1(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(bar) : "memory");
}
// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp gets lane
// (taddr lane + t), columns taddr col .. +31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory"); }
__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }
// Barrier of the 128 softmax threads that also ANDs a predicate over them: the
// way every loop exit among them is made uniform (a thread left waiting at
// bar.sync would never return).
__device__ __forceinline__ bool softmax_bar_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n bar.red.and.pred q, 1, 128, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// Shared-memory matrix descriptor: start, leading / stride byte offsets (all in
// 16-byte units), descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, M=128, N=32.
__host__ __device__ constexpr uint32_t umma_idesc(bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(kHeads >> 3) << 17) | ((uint32_t)(kChunk >> 4) << 24);
}

// Waits for the phase of `bar` with this parity, at most kWaitNs; gives up at
// once when another role has already given up, unless `drain` (the waits that
// make sure nothing is left in flight before the CTA exits).
__device__ bool wait_bounded(uint32_t bar, uint32_t parity, uint32_t *err, volatile int *abort_flag,
                             bool drain = false) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (!drain && *abort_flag) return false;
    if (global_timer_ns() - start > kWaitNs) {
      atomicOr(err, kErrTimeout);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// Per-head maximum over the warp's 32 lanes for 32 heads at once: after the
// reduce-scatter, lane h holds the maximum for head h.
__device__ __forceinline__ float warp_max_scatter(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send = upper ? v[j] : v[j + off];
      const float keep = upper ? v[j + off] : v[j];
      v[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
    }
  }
  return v[0];
}
__device__ __forceinline__ float warp_sum_scatter(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send = upper ? v[j] : v[j + off];
      const float keep = upper ? v[j + off] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

}  // namespace

// Shared memory (1024-byte aligned base): q 8 KB | K chunk 32 KB | V chunk
// 32 KB | P^T 2 x 16 KB | reductions 1 KB | barriers and words.  The K and V
// chunk buffers are reused for the split merge's weights after the last chunk.
// TMEM: S^T in two 32-column buffers, O^T after them (128 columns; two CTAs per
// SM take 256 of the 512).
struct UmmaSmem {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t k = kQBytes;
  static constexpr uint32_t v = k + kHalfBytes;
  static constexpr uint32_t pt = v + kHalfBytes;
  static constexpr uint32_t red = pt + 2 * kPBytes;
  static constexpr uint32_t bars = red + 1024;
  static constexpr uint32_t total = bars + 256 + 1024 /* alignment slack */;
};
static_assert(2 * kHalfBytes >= kHeads * kMaxSplits * 4, "merge weights fit the K and V buffers");

// One CTA per work unit (sequence b, KV head, head tile, partition s), two
// CTAs per SM: while one streams, the other's start, epilogue and split merge
// proceed.  (Double-buffering the K and V chunks, ~171 KB of shared memory and
// so one CTA per SM, was slower on the ragged MQA batch on B200: 200 against
// 162 us -- a per-CTA timeline of this layout showed two CTAs resident on
// every SM, 1.6 on average over the launch.)  Roles: warps 0-3 softmax and epilogue (thread i = token i of a
// chunk, then head_dim row i of O^T), warp 4 copies (TMA), warp 5 issues the
// MMAs (one thread).  Per chunk c of 128 tokens:
//   K(c) lands -> S(c) = K(c).Q^T into S buffer c%2 -> K buffer refilled with K(c+1)
//   softmax(c) reads S(c), writes P^T(c) -> PV(c): O^T += V(c)^T.P^T(c)
//   -> V buffer refilled with V(c+1)
// The MMA thread issues S(0), then PV(c), S(c+1) for each c, so K(c+1) and
// V(c+1) stream while the softmax works on chunk c.
__global__ void __launch_bounds__(kUmmaThreads, kUmmaCtasPerSm) umma_kernel(const __grid_constant__ PartitionParams p) {
  using SM = UmmaSmem;
  static_assert(SM::total <= (uint32_t)kSmemBudget, "shared-memory plan over budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SM::bars);
  const uint32_t q_full = smem_addr(bars + 0);
  const uint32_t k_full = smem_addr(bars + 1), k_free = smem_addr(bars + 2);
  const uint32_t v_full = smem_addr(bars + 3), v_free = smem_addr(bars + 4);
  const uint32_t s_full0 = smem_addr(bars + 5), s_free0 = smem_addr(bars + 7);
  const uint32_t p_full0 = smem_addr(bars + 9), p_free0 = smem_addr(bars + 11);
  const uint32_t o_done = smem_addr(bars + 13), mma_idle = smem_addr(bars + 14);
  uint32_t *words = reinterpret_cast<uint32_t *>(bars + 16);  // [0] tmem, [1] flag, [2] abort
  volatile int *abort_flag = reinterpret_cast<volatile int *>(words + 2);
  float *red = reinterpret_cast<float *>(smem + SM::red);  // [4][32]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (blockIdx.x == 0 && tid == 0)  // which kernel ran, and with what plan
    *p.witness = LaunchWitness{2, kD, kHeads, (int32_t)PAD_BF16, 1, kChunk, p.S, p.P, (int32_t)gridDim.x, kUmmaWarps,
                               kUmmaCtasPerSm};
  // Unit order as in partition_kernel: p.order (longest units first) when the
  // launch schedules its units, else partition index descending, outermost.
  uint32_t u = p.order != nullptr ? __ldg(p.order + blockIdx.x) : blockIdx.x;
  const uint32_t pairs = (uint32_t)p.B * p.Hkv * p.HT;
  const int s = p.S - 1 - (int)(u / pairs);
  u %= pairs;
  const int ht = (int)(u % (uint32_t)p.HT);
  u /= (uint32_t)p.HT;
  const int kvh = (int)(u % (uint32_t)p.Hkv);
  const int b = (int)(u / (uint32_t)p.Hkv);
  const int h0 = kvh * p.g + ht * kHeads;
  const int gl = min(kHeads, p.g - ht * kHeads);
  const int capacity = p.max_blocks << p.bs_log2;
  int L = __ldg(p.seq_lens + b);
  if (L < 0 || L > capacity) {
    if (tid == 0 && s == 0 && kvh == 0 && ht == 0) atomicOr(p.err, kErrSeqLen);
    L = L < 0 ? 0 : capacity;
  }
  const int t0 = s * p.P, t1 = min(t0 + p.P, L);
  if (t0 >= t1) {
    if (L == 0 && s == 0) {  // empty sequence: out = 0, lse = -inf
      for (int x = tid; x < gl * kD; x += kUmmaThreads)
        p.out[b * p.o_sb + (int64_t)(h0 + x / kD) * p.o_sh + (x % kD)] = 0;
      if (p.lse != nullptr && tid < gl) p.lse[b * p.lse_sb + (int64_t)(h0 + tid) * p.lse_sh] = -INFINITY;
    }
    return;  // nothing issued, nothing allocated
  }
  const int ns = (L + p.P - 1) / p.P;
  const int nch = (t1 - t0 + kChunk - 1) / kChunk;

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(k_full, 1);
    mbar_init(k_free, 1);
    mbar_init(v_full, 1);
    mbar_init(v_free, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full0 + 8 * i, 1);                   // QK commit
      mbar_init(s_free0 + 8 * i, kSoftmaxWarps * 32);  // every softmax thread has read S^T
      mbar_init(p_full0 + 8 * i, kSoftmaxWarps * 32);  // every softmax thread has written its P^T row
      mbar_init(p_free0 + 8 * i, 1);                   // PV commit
    }
    mbar_init(o_done, 1);
    mbar_init(mma_idle, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {  // 128 TMEM columns: S^T buffers at +0 and +32, O^T at +64
    tmem_alloc(smem_addr(words), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = words[0];
  const uint32_t tmem_o = tmem + 64;

  if (warp == kProducerWarp) {
    // ---------------- TMA: q, then each chunk's K and V (lane l copies box l) ----------------
    const int32_t *trow = p.tables + (int64_t)b * p.table_stride;
    int kq = 0, vq = 0;  // K and V chunks issued
    bool ok = true;
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, kQBytes);
      tma_load_4d(smem_addr(smem + SM::q), &p.tmq, 0, h0, 0, b, q_full);
    }
    // block id of lane l's box of chunk c (one chunk ahead, so the table's
    // latency overlaps the waits for the buffers)
    auto box_id = [&](int c) -> int {
      const int tb = t0 + c * kChunk;
      const int nbox = min(kChunk / kBoxRows, (t1 - tb + kBoxRows - 1) / kBoxRows);
      return lane < nbox ? __ldg(trow + ((tb + kBoxRows * lane) >> p.bs_log2)) : 0;
    };
    int id_next = box_id(0);
    for (int c = 0; ok && c < nch; ++c) {
      const int tb = t0 + c * kChunk;
      const int nbox = min(kChunk / kBoxRows, (t1 - tb + kBoxRows - 1) / kBoxRows);
      const int tok = tb + kBoxRows * lane;
      const int id = id_next;
      if (c + 1 < nch) id_next = box_id(c + 1);
      const int slot0 = tok & ((1 << p.bs_log2) - 1);
      if (lane < nbox && (unsigned)id >= (unsigned)p.num_blocks) atomicOr(p.err, kErrBlockId);  // reads as zeros
      // K(c) once S(c-1) has read the K buffer
      if (c > 0 && !wait_bounded(k_free, (c - 1) & 1, p.err, abort_flag)) {
        ok = false;
        break;
      }
      if (lane == 0) mbar_arrive_expect_tx(k_full, (uint32_t)nbox * kBoxBytes);
      __syncwarp();
      if (lane < nbox) tma_load_5d(smem_addr(smem + SM::k + lane * kBoxBytes), &p.tmk, 0, slot0, 0, kvh, id, k_full);
      ++kq;
      // V(c) once PV(c-1) has read the V buffer
      if (c > 0 && !wait_bounded(v_free, (c - 1) & 1, p.err, abort_flag)) {
        ok = false;
        break;
      }
      if (lane == 0) mbar_arrive_expect_tx(v_full, (uint32_t)nbox * kBoxBytes);
      __syncwarp();
      if (lane < nbox) tma_load_5d(smem_addr(smem + SM::v + lane * kBoxBytes), &p.tmv, 0, slot0, 0, kvh, id, v_full);
      ++vq;
    }
    if (!ok && lane == 0) {
      // leave no copy in flight: the last K and V chunks and q
      if (kq > 0) wait_bounded(k_full, (kq - 1) & 1, p.err, abort_flag, true);
      if (vq > 0) wait_bounded(v_full, (vq - 1) & 1, p.err, abort_flag, true);
      wait_bounded(q_full, 0, p.err, abort_flag, true);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issue (one thread): S(0), then PV(c), S(c+1) ----------------
    if (lane == 0) {
      constexpr uint32_t IQK = umma_idesc(false, false), IPV = umma_idesc(true, true);
      bool ok = wait_bounded(q_full, 0, p.err, abort_flag);
      auto qk = [&](int c) -> bool {
        if (!wait_bounded(k_full, c & 1, p.err, abort_flag)) return false;
        if (c >= 2 && !wait_bounded(s_free0 + 8 * (c & 1), ((c >> 1) - 1) & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kb = smem_addr(smem + SM::k);
        const uint32_t qb = smem_addr(smem + SM::q);
        const uint32_t sd = tmem + (uint32_t)(c & 1) * 32;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          // K: rows of 128 B in 8-row groups 2 KB apart, column block kk/4 at +1 KB
          const uint64_t a = smem_desc(kb + (kk >> 2) * 1024 + (kk & 3) * 32, 16, 2 * 1024);
          // Q: 32 heads x 128 B per column block (4 KB), 8-head groups 1 KB apart
          const uint64_t bq = smem_desc(qb + (kk >> 2) * 4096 + (kk & 3) * 32, 16, 1024);
          umma_bf16(sd, a, bq, IQK, kk > 0);
        }
        umma_commit(s_full0 + 8 * (c & 1));
        umma_commit(k_free);  // the K buffer may take the next chunk
        return true;
      };
      auto pv = [&](int c) -> bool {
        if (!wait_bounded(p_full0 + 8 * (c & 1), (c >> 1) & 1, p.err, abort_flag)) return false;
        if (!wait_bounded(v_full, c & 1, p.err, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = smem_addr(smem + SM::v);
        const uint32_t pb = smem_addr(smem + SM::pt + (c & 1) * kPBytes);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk) {
          // V^T (MN-major): 64-d column blocks 1 KB apart, 8-token groups 2 KB apart
          const uint64_t a = smem_desc(vb + kk * 2 * kBoxBytes, 1024, 2 * 1024);
          // P^T (MN-major): token rows of 128 B, 8-token groups 1 KB apart
          const uint64_t bp = smem_desc(pb + kk * 2 * 1024, 1024, 1024);
          umma_bf16(tmem_o, a, bp, IPV, c > 0 || kk > 0);
        }
        umma_commit(p_free0 + 8 * (c & 1));  // P^T buffer free; O^T holds chunks ..c
        umma_commit(v_free);                 // the V buffer may take the next chunk
        return true;
      };
      ok = ok && qk(0);
      for (int c = 0; ok && c < nch; ++c) {
        ok = pv(c);
        if (ok && c + 1 < nch) ok = qk(c + 1);
      }
      if (ok) umma_commit(o_done);
      umma_commit(mma_idle);  // every MMA issued above has completed when this arrives
    }
  } else {
    // ---------------- softmax warps: thread i = token i of a chunk, then head_dim row i ----------------
    const int i = tid;  // 0..127 == TMEM lane
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float mr[32], lp[32];
#pragma unroll
    for (int h = 0; h < 32; ++h) {
      mr[h] = -INFINITY;
      lp[h] = 0.f;
    }
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
      // warp-uniform: tcgen05.ld is a warp-collective instruction
      const bool landed = __all_sync(0xffffffffu, wait_bounded(s_full0 + 8 * (c & 1), (c >> 1) & 1, p.err, abort_flag));
      uint32_t raw[32];
      if (landed) {
        tc_fence_after();
        tmem_ld32(tmem + (uint32_t)(c & 1) * 32 + lane_off, raw);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive1(s_free0 + 8 * (c & 1));  // the next-but-one QK may overwrite this buffer
      }
      const int tb = t0 + c * kChunk;
      const bool live = landed && tb + i < t1;
      float sc[32];
      bool over = false;  // a score of this token passes its head's reference by more than the slack
#pragma unroll
      for (int h = 0; h < 32; ++h) {
        sc[h] = live ? __uint_as_float(raw[h]) * p.scale_log2 : -INFINITY;
        over |= sc[h] > mr[h] + kSlack;
      }
      if (!softmax_bar_and(landed)) {  // one decision for all 128 threads
        ok = false;
        break;
      }
      // The reference maxima are the same in every thread, so each thread
      // tests its own token and one barrier-reduce decides; the chunk's
      // per-head maximum (a transpose-reduce and a 4-warp combine) is taken
      // only when a reference moves.  Token 0 of a chunk is live and the first
      // reference is -inf, so the first chunk always sets it.
      if (!softmax_bar_and(!over)) {  // the same decision in every thread
        float cm[32];
#pragma unroll
        for (int h = 0; h < 32; ++h) cm[h] = sc[h];
        red[warp * 32 + lane] = warp_max_scatter(cm, lane);
        softmax_bar();
        const float mh = fmaxf(fmaxf(red[lane], red[32 + lane]), fmaxf(red[64 + lane], red[96 + lane]));  // head = lane
#pragma unroll
        for (int h = 0; h < 32; ++h) cm[h] = __shfl_sync(0xffffffffu, mh, h);
        softmax_bar();  // every warp has read `red` before its next use
        float al[32];
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          const float mn = fmaxf(mr[h], cm[h]);
          al[h] = fast_exp2(mr[h] - mn);
          mr[h] = mn;
          lp[h] *= al[h];
        }
        // row i of O^T holds chunks 0..c-1 once PV(c-1) has completed
        if (c > 0 &&
            __all_sync(0xffffffffu, wait_bounded(p_free0 + 8 * ((c - 1) & 1), ((c - 1) >> 1) & 1, p.err, abort_flag))) {
          tc_fence_after();
          uint32_t o[32];
          tmem_ld32(tmem_o + lane_off, o);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < 32; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * al[h]);
          tmem_st32(tmem_o + lane_off, o);
          tmem_wait_st();
        }
      }
      // weights, the fp32 running sums, and the P^T row of token i (into the
      // buffer PV(c-2) has finished reading)
      if (c >= 2) wait_bounded(p_free0 + 8 * (c & 1), ((c >> 1) - 1) & 1, p.err, abort_flag);
      uint8_t *pt = smem + SM::pt + (c & 1) * kPBytes;
      uint32_t pk[16];
#pragma unroll
      for (int h = 0; h < 32; h += 2) {
        const float e0 = fast_exp2(sc[h] - mr[h]), e1 = fast_exp2(sc[h + 1] - mr[h + 1]);
        lp[h] += e0;
        lp[h + 1] += e1;
        pk[h / 2] = pack_bf16x2(e0, e1);
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
        *reinterpret_cast<uint4 *>(pt + i * 128 + ((q4 ^ (i & 7)) << 4)) =
            make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
      if (!live) {
        // V row of a token past t1 (a slot past L_b or a box not copied):
        // zeros, after the chunk's copies have landed
        wait_bounded(v_full, c & 1, p.err, abort_flag);
        uint8_t *vrow = smem + SM::v + (i >> 3) * kBoxBytes + (i & 7) * 128;
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) {
          *reinterpret_cast<uint4 *>(vrow + q8 * 16) = make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4 *>(vrow + 1024 + q8 * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();  // P^T and zeroed rows, before the tensor core reads them
      tc_fence_before();
      mbar_arrive1(p_full0 + 8 * (c & 1));
    }

    // ---- the unit's output: thread i = head_dim row i of O^T
    if (ok) ok = softmax_bar_and(wait_bounded(o_done, 0, p.err, abort_flag));
    if (ok) {
      tc_fence_after();
      float tmp[32];
#pragma unroll
      for (int h = 0; h < 32; ++h) tmp[h] = lp[h];
      red[warp * 32 + lane] = warp_sum_scatter(tmp, lane);  // per-head sums over the token threads
      uint32_t o[32];
      tmem_ld32(tmem_o + lane_off, o);
      tmem_wait_ld();
      tc_fence_before();
      softmax_bar();
      const float lh = red[lane] + red[32 + lane] + red[64 + lane] + red[96 + lane];  // head = lane
      float mrl = 0.f;  // mr[lane]
#pragma unroll
      for (int h = 0; h < 32; ++h) mrl = h == lane ? mr[h] : mrl;
      if (ns == 1) {
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          const float inv = 1.f / __shfl_sync(0xffffffffu, lh, h);
          if (h < gl) p.out[b * p.o_sb + (int64_t)(h0 + h) * p.o_sh + i] = to_bf16_bits(__uint_as_float(o[h]) * inv);
        }
        if (warp == 0 && lane < gl && p.lse != nullptr)
          p.lse[b * p.lse_sb + (int64_t)(h0 + lane) * p.lse_sh] = (mrl + log2f(lh)) * kLn2u;
      } else {
        const int64_t row0 = ((int64_t)b * p.Hq + h0) * p.S + s;
#pragma unroll
        for (int h = 0; h < 32; ++h) {
          const float inv = 1.f / __shfl_sync(0xffffffffu, lh, h);
          if (h < gl) p.o_part[(row0 + (int64_t)h * p.S) * kD + i] = __uint_as_float(o[h]) * inv;
        }
        if (warp == 0 && lane < gl) p.lse_part[row0 + (int64_t)lane * p.S] = (mrl + log2f(lh)) * kLn2u;
      }
      softmax_bar();  // `red` is read by every warp before the merge reuses shared memory
      // every chunk has been consumed: the K and V buffers hold the merge's weights
      if (ns > 1 && claim_last_partition(p, b, kvh, ht, ns, reinterpret_cast<int *>(words + 1), Warps0to3Sync()))
        merge_partials<kD, kSoftmaxWarps * 32>(p, b, h0, gl, 0, ns, reinterpret_cast<float *>(smem + SM::k),
                                               Warps0to3Sync());
    }
  }

  // ---------------- all warps: release TMEM ----------------
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    // every MMA has completed before its accumulators are freed
    wait_bounded(mma_idle, 0, p.err, abort_flag, true);
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

int umma_stages() { return 1; }

cudaError_t launch_umma(const PartitionParams &p, int grid, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)UmmaSmem::total);
    if (e != cudaSuccess) return e;
    // all of the unified L1 / shared memory as shared memory: two CTAs of
    // ~106 KB need more than the carveout the driver picks by itself, with
    // which a timeline of the ragged MQA batch showed one CTA per SM
    e = cudaFuncSetAttribute(umma_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  umma_kernel<<<grid, kUmmaThreads, UmmaSmem::total, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace pad
