// Partition kernel: persistent split-KV decode with the split reduce folded into
// the same launch.
//
// Work unit = (sequence b, KV head, head tile, partition s): the query heads of
// one GQA group (up to 32 per tile) against tokens [s*P, min((s+1)*P, L_b)).
// One CTA per SM claims units from a global counter ("perf(rocke): prepare saved
// paged decode bindings once", section "Summary": one-token split-KV attention
// with a reduce pass; here the pass boundaries are per unit, not per launch).
//
// Warp roles (6 warps):
//  * scheduler (warp 4): claims units (the next claim and its seq_len and
//    block-table entries are always in flight), bulk-copies each unit's q rows
//    to shared memory, and writes one descriptor per 64-token stage -- token
//    range, flags and the block id of every page the stage covers, checked
//    against num_blocks -- into a ring of descriptors.  Partitions past
//    ceil(L_b / P) are skipped by pushing the claim counter past them.
//  * workers (warps 0-3): worker w owns the 16-token sub-tile w of every stage.
//    It gathers that sub-tile's K and V rows itself with 16-byte cp.async into
//    its own shared-memory ring (rows XOR-swizzled so ldmatrix is conflict free;
//    rows past L_b zero-filled without a read), NST-1 stages ahead of its math,
//    so the loads of all four workers are spread over the four SM sub-partitions
//    and no worker ever waits for another within a unit.  Per sub-tile and
//    8-head n-tile:
//      S^T = K.Q^T                    (mma.m16n8k16 bf16, fp32 accumulate)
//      running max / sum per head     (the warp-strided online softmax of
//                                      "spec(BACKEND-ROCM): the ROCm head_dim=128
//                                      decode arm", section "It is a mirror of
//                                      merged work, not new design")
//      O^T += V^T.P^T                 (P^T moved into the B-operand layout with
//                                      movmatrix)
//    All heads of the GQA group are served from that one K/V read (same
//    section: PagedAttnDecodeGqaBf16 fuses a GQA group).  At the end of a unit
//    the four workers merge through shared memory; a sequence with one
//    non-empty partition writes bf16 out (+ lse) directly, otherwise each
//    partition writes its fp32 output (normalised by its own sum) and its lse
//    and hands the unit to the merger.
//  * merger (warp 5): counts finished partitions per (b, KV head, head tile); the
//    CTA that completes the set merges them by log-sum-exp while they are in L2:
//      M = max_s lse_s,  out = sum_s exp(lse_s - M) o_s / sum_s exp(lse_s - M),
//      lse = M + log sum_s exp(lse_s - M).
//
// Every mbarrier wait is bounded in time: on expiry it sets an error bit and the
// kernel returns instead of hanging.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "pad_device.cuh"
#include "pad_internal.h"

namespace pad {

__device__ uint32_t g_err_word;

namespace {

constexpr uint32_t kFlagFirst = 1u, kFlagLast = 2u, kFlagTerminate = 4u, kFlagEmptySeq = 8u;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // no wait here can legitimately take 2 s
constexpr float kLn2 = 0.69314718055994530942f;
constexpr int kMergeQueue = 4;
constexpr int kSchedWarp = kWorkers, kMergerWarp = kWorkers + 1;
constexpr int kMaxStagePages = kStageTokens;  // block_size 1

struct StageDesc {
  int32_t b, kvh, ht, s;
  int32_t tb;  // first token of the stage
  int32_t t1;  // end of the unit's token range
  int32_t ns;  // non-empty partitions of sequence b
  uint32_t flags;
  int32_t pages[kMaxStagePages];  // block id of each page the stage covers; -1 = invalid id
};
static_assert(sizeof(StageDesc) == kDescBytes, "descriptor size");

struct MergeMeta {
  int32_t b, kvh, ht, ns;  // ns < 0: no more units
};

// Waits for the phase of `bar` with this parity.  Gives up after kWaitLimitNs
// (flagging kErrTimeout and the CTA-wide abort flag) or, when `honor_abort`, as
// soon as another role of the CTA has given up.
__device__ bool wait_phase(uint32_t bar, uint32_t parity, volatile int *abort_flag, uint32_t *err,
                           bool honor_abort = true) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_timer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (honor_abort && *abort_flag) return false;
    if (global_timer_ns() - start > kWaitLimitNs) {
      *abort_flag = 1;
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
}

}  // namespace

template <int D, int HPT>
__global__ void __launch_bounds__(kThreads, 1) partition_kernel(const __grid_constant__ PartitionParams p) {
  constexpr SmemPlan SP = smem_plan_for(D, HPT);
  constexpr int NST = SP.stages;                        // stages in each worker's ring
  constexpr int ND = NST + 2;                           // stage descriptors
  constexpr int NQ = SP.q_slots;                        // q ring slots (== NST)
  constexpr int HALVES = D / 64;                        // 128-byte column blocks of a row
  constexpr int KT = D / 16;                            // QK k-steps == PV m-tiles
  constexpr int NT = HPT / 8;                           // 8-head n-tiles per head tile
  constexpr int CH = D / 8;                             // 16-byte chunks per K/V row
  constexpr uint32_t HALF_BYTES = 16 * 128;             // 16 rows x 128 B
  constexpr uint32_t TILE_BYTES = HALF_BYTES * HALVES;  // K (or V) of one sub-tile
  constexpr uint32_t QROW = (uint32_t)SP.q_row_bytes;
  constexpr int MROW = D + 4;                           // merge row stride (floats)
  constexpr int MSLOT = HPT * MROW + 2 * HPT;           // floats per merge slot
  constexpr int MS = SP.merge_slots;
  constexpr int NWT = kWorkers * 32;                    // worker threads
  constexpr bool SPLIT_QK = NT <= 2;                    // two QK chains when registers allow
  static_assert(NST >= 2, "shared memory too small for a 2-stage ring");
  static_assert(ND <= kMaxDescs, "descriptor ring");
  static_assert(SP.total <= (size_t)kSmemBudget, "shared-memory plan over budget");
  static_assert(NQ >= NST, "q ring shallower than the stage lookahead: short units would deadlock");
  static_assert(2 * ND + 2 * NQ + 1 + 2 * kMergeQueue <= 52, "mbarrier area");

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *ring = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *qbuf = ring + SP.ring_bytes;
  float *merge = reinterpret_cast<float *>(qbuf + SP.q_bytes);
  StageDesc *desc = reinterpret_cast<StageDesc *>(reinterpret_cast<uint8_t *>(merge) + SP.merge_bytes);
  uint8_t *misc = reinterpret_cast<uint8_t *>(desc) + SP.desc_bytes;
  // mbarriers: dfull[ND] dempty[ND] qfull[NQ] qempty[NQ] cbar mqfull[4] mqempty[4]
  uint64_t *bars = reinterpret_cast<uint64_t *>(misc);
  MergeMeta *mqmeta = reinterpret_cast<MergeMeta *>(misc + 480 - kMergeQueue * sizeof(MergeMeta));
  volatile int *abort_flag = reinterpret_cast<volatile int *>(misc + 480);

  const uint32_t dfull0 = smem_addr(bars), dempty0 = smem_addr(bars + ND);
  const uint32_t qfull0 = smem_addr(bars + 2 * ND), qempty0 = smem_addr(bars + 2 * ND + NQ);
  const uint32_t cbar = smem_addr(bars + 2 * ND + 2 * NQ);
  const uint32_t mqf0 = smem_addr(bars + 2 * ND + 2 * NQ + 1);
  const uint32_t mqe0 = smem_addr(bars + 2 * ND + 2 * NQ + 1 + kMergeQueue);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    for (int i = 0; i < ND; ++i) {
      mbar_init(dfull0 + 8 * i, 32);    // every scheduler lane, after writing its page ids
      mbar_init(dempty0 + 8 * i, NWT);  // every worker thread, after computing the stage
    }
    for (int i = 0; i < NQ; ++i) {
      mbar_init(qfull0 + 8 * i, 1);
      mbar_init(qempty0 + 8 * i, NWT);
    }
    mbar_init(cbar, NWT);
    for (int i = 0; i < kMergeQueue; ++i) {
      mbar_init(mqf0 + 8 * i, NWT);
      mbar_init(mqe0 + 8 * i, 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // padded q rows must hold finite values: zero the q buffers once
  for (uint32_t i = tid; i < SP.q_bytes / 16; i += kThreads)
    reinterpret_cast<uint4 *>(qbuf)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  __syncthreads();

  const int capacity = p.max_blocks << p.bs_log2;
  const int bs = 1 << p.bs_log2;

  // ======================= scheduler warp =======================
  if (warp == kSchedWarp) {
    const int pages_per_stage = bs < kStageTokens ? kStageTokens / bs : 1;
    uint32_t st = 0, k = 0, issued = 0;  // stages written, units with q, q copies issued
    bool ok = true;
    auto decode_unit = [&](uint32_t u, int &s, uint32_t &pair, int &ht, int &kvh, int &b) {
      s = (int)(u % (uint32_t)p.S);
      pair = u / (uint32_t)p.S;
      ht = (int)(pair % (uint32_t)p.HT);
      const int rest = (int)(pair / (uint32_t)p.HT);
      kvh = rest % p.Hkv;
      b = rest / p.Hkv;
    };
    // table entries of one 64-page chunk: lane j holds pages base + j, base + 32 + j
    auto load_chunk = [&](int b, int base, int (&ph)[2]) {
      const int32_t *trow = p.tables + (int64_t)b * p.table_stride;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int pg = base + lane + 32 * r;
        ph[r] = pg < p.max_blocks ? __ldg(trow + pg) : -1;
      }
    };
    // Everything a unit needs from global memory (its claim, seq_len and first
    // 64 block-table entries) is fetched one unit ahead.
    uint32_t claim = 0;  // lane 0: the unit after the prefetched one
    uint32_t un = 0;     // prefetched unit
    int Ln = 0;          // lane 0: its raw seq_len
    int tabn[2] = {-1, -1};
    auto prefetch = [&]() {
      un = __shfl_sync(0xffffffffu, claim, 0);
      if (un < p.n_units) {
        int s_, ht_, kvh_, b_;
        uint32_t pair_;
        decode_unit(un, s_, pair_, ht_, kvh_, b_);
        if (lane == 0) Ln = __ldg(p.seq_lens + b_);
        load_chunk(b_, (s_ * p.P) >> p.bs_log2, tabn);
      }
      if (lane == 0) claim = atomicAdd(p.ctl, 1u);
    };
    if (lane == 0) claim = atomicAdd(p.ctl, 1u);
    prefetch();
    while (true) {
      const uint32_t u = un;
      if (u >= p.n_units) break;
      int s, ht, kvh, b;
      uint32_t pair;
      decode_unit(u, s, pair, ht, kvh, b);
      int L = Ln;
      int tab[2] = {tabn[0], tabn[1]};
      if (lane == 0) {
        if (L < 0 || L > capacity) {
          if (s == 0 && kvh == 0 && ht == 0) atomicOr(p.err, kErrSeqLen);
          L = L < 0 ? 0 : capacity;
        }
        // no later partition of this (b, kv head, tile) has tokens: skip them all
        if (s + 1 >= (L + p.P - 1) / p.P) atomicMax(p.ctl, (pair + 1) * (uint32_t)p.S);
      }
      L = __shfl_sync(0xffffffffu, L, 0);
      prefetch();  // the next unit's loads overlap this unit
      const int ns = (L + p.P - 1) / p.P;
      const bool empty_seq = L == 0;
      if (s >= ns && !(empty_seq && s == 0)) continue;

      const int h0 = kvh * p.g + ht * HPT;
      const int gl = min(HPT, p.g - ht * HPT);
      const int t0 = s * p.P;
      const int t1 = min(t0 + p.P, L);
      const int nst = t1 > t0 ? (t1 - t0 + kStageTokens - 1) / kStageTokens : 1;
      const int first_page = t0 >> p.bs_log2;
      const int last_page = t1 > t0 ? (t1 - 1) >> p.bs_log2 : -1;
      // further 64-page chunks of this unit, each loaded a chunk ahead
      int chunk = 0;
      int tabx[2] = {-1, -1};
      if (!empty_seq && first_page + 64 <= last_page) load_chunk(b, first_page + 64, tabx);

      if (!empty_seq) {  // this head tile's q rows -> q slot k % NQ
        const int qs = k % NQ;
        if (!wait_phase(qempty0 + 8 * qs, ((k / NQ) & 1) ^ 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        if (lane == 0) mbar_arrive_expect_tx(qfull0 + 8 * qs, (uint32_t)gl * D * 2);
        __syncwarp();
        if (lane < gl)
          bulk_load(smem_addr(qbuf + (qs * HPT + lane) * QROW), p.q + b * p.q_sb + (int64_t)(h0 + lane) * p.q_sh,
                    D * 2, qfull0 + 8 * qs);
        ++issued;
      }

      for (int i = 0; i < nst; ++i, ++st) {
        const int tb = t0 + i * kStageTokens;
        // the stage's pages start at offset rel of the unit; a stage never
        // straddles a 64-page chunk (64 is a multiple of the pages per stage)
        const int rel = (tb >> p.bs_log2) - first_page;
        if (!empty_seq && (rel >> 6) > chunk) {
          ++chunk;
          tab[0] = tabx[0];
          tab[1] = tabx[1];
          if (first_page + 64 * (chunk + 1) <= last_page) load_chunk(b, first_page + 64 * (chunk + 1), tabx);
        }
        const uint32_t slot = st % ND;
        if (!wait_phase(dempty0 + 8 * slot, ((st / ND) & 1) ^ 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        StageDesc &d = desc[slot];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int j = lane + 32 * r;
          const int idx = (rel & 63) + j;  // position in the chunk
          const int lo = __shfl_sync(0xffffffffu, tab[0], idx & 31);
          const int hi = __shfl_sync(0xffffffffu, tab[1], idx & 31);
          int phys = idx < 32 ? lo : hi;
          if (!empty_seq && j < pages_per_stage && first_page + rel + j <= last_page) {
            if ((unsigned)phys >= (unsigned)p.num_blocks) {
              atomicOr(p.err, kErrBlockId);
              phys = -1;
            }
            d.pages[j] = phys;
          }
        }
        if (lane == 0) {
          d.b = b;
          d.kvh = kvh;
          d.ht = ht;
          d.s = s;
          d.tb = tb;
          d.t1 = t1;
          d.ns = ns;
          d.flags = (i == 0 ? kFlagFirst : 0u) | (i == nst - 1 ? kFlagLast : 0u) | (empty_seq ? kFlagEmptySeq : 0u);
        }
        mbar_arrive(dfull0 + 8 * slot);  // releases this lane's writes
      }
      if (!ok) break;
      if (!empty_seq) ++k;
    }
    if (ok) {
      const uint32_t slot = st % ND;
      if (wait_phase(dempty0 + 8 * slot, ((st / ND) & 1) ^ 1, abort_flag, p.err)) {
        if (lane == 0) desc[slot].flags = kFlagTerminate;
        mbar_arrive(dfull0 + 8 * slot);
      }
    } else {
      // q copies already issued must land before the CTA exits: the latest
      // copy into each slot completes that slot's phase (issued-1-i) / NQ
      for (uint32_t i = 0; i < (uint32_t)NQ && i < issued; ++i) {
        const uint32_t c = issued - 1 - i;
        wait_phase(qfull0 + 8 * (c % NQ), (c / NQ) & 1, abort_flag, p.err, false);
      }
    }
    if (lane == 0) {
      __threadfence();
      if (atomicAdd(p.ctl + 1, 1u) == gridDim.x - 1) {  // every CTA has stopped claiming
        atomicExch(p.ctl, 0u);
        atomicExch(p.ctl + 1, 0u);
      }
    }
    return;
  }

  // ======================= merger warp =======================
  if (warp == kMergerWarp) {
    constexpr int D4 = D / 4;
    uint32_t nm = 0;
    while (true) {
      const uint32_t mq = nm % kMergeQueue;
      if (!wait_phase(mqf0 + 8 * mq, (nm / kMergeQueue) & 1, abort_flag, p.err)) break;
      const MergeMeta mm = mqmeta[mq];
      mbar_arrive(mqe0 + 8 * mq);  // the entry has been copied
      if (mm.ns < 0) break;
      uint32_t last = 0;
      if (lane == 0) {
        // the workers' partial stores happen-before this (CTA barrier above)
        __threadfence();
        const uint32_t pair = ((uint32_t)mm.b * p.Hkv + mm.kvh) * p.HT + mm.ht;
        const uint32_t done = atomicAdd(p.counters + pair, 1u);
        last = done + 1 == (uint32_t)mm.ns;
        if (last) atomicExch(p.counters + pair, 0u);
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      ++nm;
      if (!last) continue;
      __threadfence();
      const int h0 = mm.kvh * p.g + mm.ht * HPT;
      const int gl = min(HPT, p.g - mm.ht * HPT);
      for (int i = lane; i < gl * D4; i += 32) {
        const int hl = i / D4, d = (i % D4) * 4;
        const int64_t row0 = ((int64_t)mm.b * p.Hq + h0 + hl) * p.S;
        float M = -INFINITY;
        for (int s0 = 0; s0 < mm.ns; s0 += 8) {
          float v[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) v[j] = s0 + j < mm.ns ? ld_cg_f32(p.lse_part + row0 + s0 + j) : -INFINITY;
#pragma unroll
          for (int j = 0; j < 8; ++j) M = fmaxf(M, v[j]);
        }
        float sum = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < mm.ns; s0 += 4) {
          float lv[4];
          float4 ov[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const bool in = s0 + j < mm.ns;
            lv[j] = in ? ld_cg_f32(p.lse_part + row0 + s0 + j) : -INFINITY;
            ov[j] = in ? ld_cg_f4(p.o_part + (row0 + s0 + j) * D + d) : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float w = __expf(lv[j] - M);
            sum += w;
            acc.x += w * ov[j].x;
            acc.y += w * ov[j].y;
            acc.z += w * ov[j].z;
            acc.w += w * ov[j].w;
          }
        }
        const float inv = 1.f / sum;
        uint2 packed;
        packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        *reinterpret_cast<uint2 *>(p.out + mm.b * p.o_sb + (int64_t)(h0 + hl) * p.o_sh + d) = packed;
        if (d == 0 && p.lse != nullptr) p.lse[mm.b * p.lse_sb + (int64_t)(h0 + hl) * p.lse_sh] = M + logf(sum);
      }
    }
    return;
  }

  // ======================= worker warps =======================
  const int w = warp;  // this worker's sub-tile of every stage
  uint8_t *my_ring = ring + w * SP.sub_bytes;
  uint32_t jl = 0, jc = 0;  // next stage to load, next stage to compute
  uint32_t k = 0, cph = 0, nm = 0;
  bool ended = false, ok = true;
  uint32_t qf[NT][KT][2];
  float oacc[NT][KT][4];
  float m_run[NT][2], l_run[NT][2];

  auto cbar_sync = [&]() -> bool {
    mbar_arrive(cbar);
    const bool r = wait_phase(cbar, cph, abort_flag, p.err);
    cph ^= 1u;
    return r;
  };
  // hand one entry to the merger (ns < 0: no more units)
  auto push_merge = [&](int b, int kvh, int ht, int ns) -> bool {
    const uint32_t mq = nm % kMergeQueue;
    if (!wait_phase(mqe0 + 8 * mq, ((nm / kMergeQueue) & 1) ^ 1, abort_flag, p.err)) return false;
    if (tid == 0) {
      MergeMeta mm;
      mm.b = b;
      mm.kvh = kvh;
      mm.ht = ht;
      mm.ns = ns;
      mqmeta[mq] = mm;
    }
    mbar_arrive(mqf0 + 8 * mq);  // releases every worker thread's partial stores
    ++nm;
    return true;
  };
  // Gather this worker's 16 rows of stage jl into ring slot jl % NST.  Always
  // commits exactly one cp.async group, so group i is stage i.
  auto issue = [&]() {
    if (!ended && ok) {
      const uint32_t ds = jl % ND;
      if (!wait_phase(dfull0 + 8 * ds, (jl / ND) & 1, abort_flag, p.err)) {
        ok = false;
      } else {
        const StageDesc &d = desc[ds];
        if (d.flags & kFlagTerminate) {
          ended = true;
        } else {
          const int tok0 = d.tb + 16 * w;
          if (!(d.flags & kFlagEmptySeq) && tok0 < d.t1) {
            const int page0 = d.tb >> p.bs_log2;
            uint8_t *sK = my_ring + (jl % NST) * SP.stage_bytes;
            uint8_t *sV = sK + TILE_BYTES;
            const int64_t kh_k = (int64_t)d.kvh * p.k_sh, kh_v = (int64_t)d.kvh * p.v_sh;
#pragma unroll
            for (int e = lane; e < 16 * CH; e += 32) {
              const int r = e / CH, c = e % CH;
              const int t = tok0 + r;
              const int phys = t < d.t1 ? d.pages[(t >> p.bs_log2) - page0] : -1;
              const bool ld = phys >= 0;
              const int slot = t & (bs - 1);
              const uint32_t off = (c >> 3) * HALF_BYTES + r * 128 + (((c & 7) ^ (r & 7)) << 4);
              cp_async_16(smem_addr(sK + off), ld ? p.k + (int64_t)phys * p.k_sblk + kh_k + slot * p.k_ss + c * 8 : p.k, ld);
              cp_async_16(smem_addr(sV + off), ld ? p.v + (int64_t)phys * p.v_sblk + kh_v + slot * p.v_ss + c * 8 : p.v, ld);
            }
          }
          ++jl;
        }
      }
    }
    cp_async_commit();
  };

#pragma unroll 1
  for (int i = 0; i < NST - 1; ++i) issue();
  while (ok) {
    issue();  // stage jc + NST - 1
    if (!ok || jc >= jl) break;
    cp_async_wait<NST - 1>();  // this worker's rows of stage jc have landed
    __syncwarp();
    const uint32_t ds = jc % ND;
    const StageDesc &d = desc[ds];
    const uint32_t flags = d.flags;
    const int h0 = d.kvh * p.g + d.ht * HPT;
    const int gl = min(HPT, p.g - d.ht * HPT);

    if (flags & kFlagEmptySeq) {  // L_b = 0: out = 0, lse = -inf
      if (w == 0) {
        for (int i = lane; i < gl * D; i += 32) p.out[d.b * p.o_sb + (int64_t)(h0 + i / D) * p.o_sh + (i % D)] = 0;
        if (p.lse != nullptr && lane < gl) p.lse[d.b * p.lse_sb + (int64_t)(h0 + lane) * p.lse_sh] = -INFINITY;
      }
      mbar_arrive(dempty0 + 8 * ds);
      ++jc;
      continue;
    }

    if (flags & kFlagFirst) {
      const int qs = k % NQ;
      if (!wait_phase(qfull0 + 8 * qs, (k / NQ) & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      // Q^T fragments (B operand): head nt*8 + lane/4, dims 16kk + 2(lane%4) + {0,1}, {8,9}
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const uint8_t *qrow = qbuf + (qs * HPT + nt * 8 + (lane >> 2)) * QROW + (lane & 3) * 4;
#pragma unroll
        for (int kk = 0; kk < KT; ++kk) {
          qf[nt][kk][0] = *reinterpret_cast<const uint32_t *>(qrow + kk * 32);
          qf[nt][kk][1] = *reinterpret_cast<const uint32_t *>(qrow + kk * 32 + 16);
        }
      }
      mbar_arrive(qempty0 + 8 * qs);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          m_run[nt][j] = -INFINITY;
          l_run[nt][j] = 0.f;
        }
#pragma unroll
        for (int mt = 0; mt < KT; ++mt)
#pragma unroll
          for (int i = 0; i < 4; ++i) oacc[nt][mt][i] = 0.f;
      }
    }

    const int tok0 = d.tb + 16 * w;
    const int t1 = d.t1;
    if (tok0 < t1) {
      const uint8_t *sK = my_ring + (jc % NST) * SP.stage_bytes;
      const uint8_t *sV = sK + TILE_BYTES;
      // ---- S^T = K . Q^T over this sub-tile's 16 tokens
      float sc[NT][4], sc2[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[nt][i] = sc2[nt][i] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
        const int c = kk * 2 + (lane >> 4);
        uint32_t a[4];
        ldsm_x4(a, smem_addr(sK + (c >> 3) * HALF_BYTES + r * 128 + (((c & 7) ^ (r & 7)) << 4)));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (SPLIT_QK && (kk & 1))
            mma_16816(sc2[nt], a, qf[nt][kk][0], qf[nt][kk][1]);
          else
            mma_16816(sc[nt], a, qf[nt][kk][0], qf[nt][kk][1]);
        }
      }
      // ---- online softmax (rows lane/4 and lane/4 + 8; columns 2(lane%4) + {0,1})
      const bool okA = tok0 + (lane >> 2) < t1;
      const bool okB = tok0 + (lane >> 2) + 8 < t1;
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        if (SPLIT_QK)
#pragma unroll
          for (int i = 0; i < 4; ++i) sc[nt][i] += sc2[nt][i];
        const float s0 = okA ? sc[nt][0] * p.scale_log2 : -INFINITY;
        const float s1 = okA ? sc[nt][1] * p.scale_log2 : -INFINITY;
        const float s2 = okB ? sc[nt][2] * p.scale_log2 : -INFINITY;
        const float s3 = okB ? sc[nt][3] * p.scale_log2 : -INFINITY;
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        // row 0 of the sub-tile is a live token, so the new maxima are finite
        const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
        const float al0 = fast_exp2(m_run[nt][0] - mn0), al1 = fast_exp2(m_run[nt][1] - mn1);
        m_run[nt][0] = mn0;
        m_run[nt][1] = mn1;
        const float e0 = fast_exp2(s0 - mn0), e1 = fast_exp2(s1 - mn1);
        const float e2 = fast_exp2(s2 - mn0), e3 = fast_exp2(s3 - mn1);
        const uint32_t pA = pack_bf16x2(e0, e1);
        const uint32_t pB = pack_bf16x2(e2, e3);
        // The running sum takes the fp32 weights: summing the bf16-rounded ones
        // moves the LSE of a short sequence by up to 2^-9 (one weight's rounding).
        l_run[nt][0] = l_run[nt][0] * al0 + e0 + e2;
        l_run[nt][1] = l_run[nt][1] * al1 + e1 + e3;
#pragma unroll
        for (int mt = 0; mt < KT; ++mt) {
          oacc[nt][mt][0] *= al0;
          oacc[nt][mt][1] *= al1;
          oacc[nt][mt][2] *= al0;
          oacc[nt][mt][3] *= al1;
        }
        pb[nt][0] = movmatrix_t(pA);
        pb[nt][1] = movmatrix_t(pB);
      }
      // ---- O^T += V^T . P^T  (rows past t1 were zero-filled, weights are 0)
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) {
        const int j = lane >> 3;
        const int r = (lane & 7) + (j >> 1) * 8;
        const int c = mt * 2 + (j & 1);
        uint32_t a[4];
        ldsm_x4_t(a, smem_addr(sV + (c >> 3) * HALF_BYTES + r * 128 + (((c & 7) ^ (r & 7)) << 4)));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(oacc[nt][mt], a, pb[nt][0], pb[nt][1]);
      }
    }
    const int b = d.b, kvh = d.kvh, ht = d.ht, s = d.s, ns = d.ns;
    mbar_arrive(dempty0 + 8 * ds);  // done with the descriptor and this ring slot's data

    if (flags & kFlagLast) {
      // ---------------- epilogue of the unit: merge the four workers ----------------
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) l_run[nt][j] += __shfl_xor_sync(0xffffffffu, l_run[nt][j], off);
      auto write_slot = [&](float *ms) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int mt = 0; mt < KT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
              ms[(nt * 8 + 2 * (lane & 3) + (i & 1)) * MROW + mt * 16 + (lane >> 2) + 8 * (i >> 1)] = oacc[nt][mt][i];
          if (lane < 4)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              ms[HPT * MROW + nt * 8 + 2 * lane + j] = m_run[nt][j];
              ms[HPT * MROW + HPT + nt * 8 + 2 * lane + j] = l_run[nt][j];
            }
        }
      };
      auto combine_slot = [&](const float *ms) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int col = nt * 8 + 2 * (lane & 3) + j;
            const float mo = ms[HPT * MROW + col], lo = ms[HPT * MROW + HPT + col];
            const float mn = fmaxf(m_run[nt][j], mo);
            const float fa = m_run[nt][j] == -INFINITY ? 0.f : fast_exp2(m_run[nt][j] - mn);
            const float fb = mo == -INFINITY ? 0.f : fast_exp2(mo - mn);
            l_run[nt][j] = l_run[nt][j] * fa + lo * fb;
            m_run[nt][j] = mn;
#pragma unroll
            for (int mt = 0; mt < KT; ++mt)
#pragma unroll
              for (int hi = 0; hi < 2; ++hi) {
                const int i = 2 * hi + j;
                oacc[nt][mt][i] = oacc[nt][mt][i] * fa + fb * ms[col * MROW + mt * 16 + (lane >> 2) + 8 * hi];
              }
          }
      };
      if constexpr (MS == kWorkers - 1) {
        if (w > 0) write_slot(merge + (w - 1) * MSLOT);
        if (!cbar_sync()) {
          ok = false;
          break;
        }
        if (w == 0)
#pragma unroll 1
          for (int t2 = 0; t2 < kWorkers - 1; ++t2) combine_slot(merge + t2 * MSLOT);
      } else {
        bool good = true;
#pragma unroll 1
        for (int t2 = 1; t2 < kWorkers && good; ++t2) {
          if (w == t2) write_slot(merge);
          good = cbar_sync();
          if (good && w == 0) combine_slot(merge);
          good = good && cbar_sync();
        }
        if (!good) {
          ok = false;
          break;
        }
      }
      if (w == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float inv[2], lse_nat[2];
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            inv[j] = 1.f / l_run[nt][j];
            lse_nat[j] = (m_run[nt][j] + log2f(l_run[nt][j])) * kLn2;
          }
          const int hl0 = nt * 8 + 2 * (lane & 3);
          if (ns <= 1) {
#pragma unroll
            for (int mt = 0; mt < KT; ++mt)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int hl = hl0 + (i & 1);
                if (hl < gl)
                  p.out[b * p.o_sb + (int64_t)(h0 + hl) * p.o_sh + mt * 16 + (lane >> 2) + 8 * (i >> 1)] =
                      to_bf16_bits(oacc[nt][mt][i] * inv[i & 1]);
              }
            if (lane < 4 && p.lse != nullptr)
#pragma unroll
              for (int j = 0; j < 2; ++j)
                if (hl0 + j < gl) p.lse[b * p.lse_sb + (int64_t)(h0 + hl0 + j) * p.lse_sh] = lse_nat[j];
          } else {
#pragma unroll
            for (int mt = 0; mt < KT; ++mt)
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int hl = hl0 + (i & 1);
                if (hl < gl) {
                  const int64_t row = ((int64_t)b * p.Hq + h0 + hl) * p.S + s;
                  p.o_part[row * D + mt * 16 + (lane >> 2) + 8 * (i >> 1)] = oacc[nt][mt][i] * inv[i & 1];
                }
              }
            if (lane < 4)
#pragma unroll
              for (int j = 0; j < 2; ++j)
                if (hl0 + j < gl) p.lse_part[((int64_t)b * p.Hq + h0 + hl0 + j) * p.S + s] = lse_nat[j];
          }
        }
      }
      if (ns > 1 && !push_merge(b, kvh, ht, ns)) {
        ok = false;
        break;
      }
      if constexpr (MS == kWorkers - 1) {
        if (!cbar_sync()) {  // merge slots free for the next unit
          ok = false;
          break;
        }
      }
      ++k;
    }
    ++jc;
  }
  if (ok) push_merge(0, 0, 0, -1);  // no more units for the merger
  cp_async_wait_all();               // never exit with copies in flight
}

int partition_stages(int D, int hpt) {
  switch (D) {
    case 64: return hpt == 8 ? smem_plan_for(64, 8).stages : hpt == 16 ? smem_plan_for(64, 16).stages : smem_plan_for(64, 32).stages;
    case 128: return hpt == 8 ? smem_plan_for(128, 8).stages : hpt == 16 ? smem_plan_for(128, 16).stages : smem_plan_for(128, 32).stages;
    case 256: return hpt == 8 ? smem_plan_for(256, 8).stages : smem_plan_for(256, 16).stages;
  }
  return 0;
}

template <int D, int HPT>
static cudaError_t launch_t(const PartitionParams &p, int grid, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  constexpr SmemPlan SP = smem_plan_for(D, HPT);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(partition_kernel<D, HPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SP.total);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  partition_kernel<D, HPT><<<grid, kThreads, SP.total, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_partition(const PartitionParams &p, int D, int heads_per_tile, int grid, cudaStream_t s) {
  if (heads_per_tile > max_heads_per_tile(D)) return cudaErrorInvalidValue;
  switch (D * 64 + heads_per_tile) {
    case 64 * 64 + 8: return launch_t<64, 8>(p, grid, s);
    case 64 * 64 + 16: return launch_t<64, 16>(p, grid, s);
    case 64 * 64 + 32: return launch_t<64, 32>(p, grid, s);
    case 128 * 64 + 8: return launch_t<128, 8>(p, grid, s);
    case 128 * 64 + 16: return launch_t<128, 16>(p, grid, s);
    case 128 * 64 + 32: return launch_t<128, 32>(p, grid, s);
    case 256 * 64 + 8: return launch_t<256, 8>(p, grid, s);
    case 256 * 64 + 16: return launch_t<256, 16>(p, grid, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t device_error_word(int device, uint32_t **ptr) {
  static std::atomic<uint32_t *> cache[64];
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  uint32_t *v = cache[device].load(std::memory_order_acquire);
  if (v == nullptr) {
    void *addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_err_word);
    if (e != cudaSuccess) return e;
    v = static_cast<uint32_t *>(addr);
    cache[device].store(v, std::memory_order_release);
  }
  *ptr = v;
  return cudaSuccess;
}

}  // namespace pad
