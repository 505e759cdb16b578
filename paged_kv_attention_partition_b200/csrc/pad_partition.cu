// Partition kernel: split-KV single-token decode with the split reduce folded
// into the same launch.
//
// One CTA per work unit (sequence b, KV head, head tile, partition s): the query
// heads of one GQA group (up to 32 per tile) against tokens [s*P, min((s+1)*P,
// L_b)) ("perf(rocke): prepare saved paged decode bindings once", section
// "Summary": one-token split-KV attention followed by a reduce pass).  Several
// CTAs share each SM (the ring is sized for it), so one CTA's start -- table and
// q latency -- and finish -- merge and stores -- overlap the others' streaming.
//
// The CTA streams its partition's K and V pages for one KV head from HBM into a
// small shared-memory ring (16-byte cp.async per thread; rows XOR-swizzled so the
// tensor-core operand loads are bank-conflict free; rows past L_b zero-filled
// without a read).  Each thread's page ids for the next stage are loaded one
// stage ahead, so the loads never wait on the block table.  Every query head of
// the GQA group is served from that one K/V read ("spec(BACKEND-ROCM): the ROCm
// head_dim=128 decode arm", section "It is a mirror of merged work, not new
// design": PagedAttnDecodeGqaBf16 fuses a GQA group over one K/V read).
//
// Warp w computes tokens 16w .. 16w+15 of every 64-token stage and keeps its own
// running max and sum per head (the warp-strided online softmax of the same
// section; the four warps are merged at the end, so the sum is taken in another
// order than a sequential kernel's).  Per 16-token tile and 8-head n-tile:
//   S^T = K . Q^T                 (mma.m16n8k16 bf16, fp32 accumulate)
//   P^T = exp2(S^T * scale*log2e - m)
//   O^T += V^T . P^T              (P^T moved into the B-operand layout by movmatrix)
//
// A sequence with one non-empty partition writes bf16 out (+ lse) directly.
// Otherwise each partition writes its fp32 output (normalised by its own sum)
// and its lse, and the CTA that finishes the last partition of the (b, KV head,
// head tile) merges them by log-sum-exp while they are in L2:
//   M = max_s lse_s,  w_s = exp(lse_s - M) / sum_s' exp(lse_s' - M),
//   out = sum_s w_s o_s,  lse = M + log sum_s exp(lse_s - M).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "pad_device.cuh"
#include "pad_internal.h"

namespace pad {

__device__ uint32_t g_err_word;

namespace {
constexpr float kLn2 = 0.69314718055994530942f;
}

template <int D, int HPT>
__global__ void __launch_bounds__(kThreads, ctas_per_sm_for(D, HPT))
    partition_kernel(const __grid_constant__ PartitionParams p) {
  constexpr SmemPlan SP = smem_plan_for(D, HPT);
  constexpr int NST = SP.stages;
  constexpr uint32_t STAGE_BYTES = (uint32_t)SP.stage_bytes;
  constexpr int NT = HPT / 8;              // 8-head n-tiles
  constexpr int KT = D / 16;               // QK k-steps == PV m-tiles
  constexpr int CH = D / 8;                // 16-byte chunks per K/V row
  constexpr int ROWB = D * 2;
  constexpr int RPP = kThreads / CH;       // rows per loader pass
  constexpr int NR = kStageTokens / RPP;   // rows each thread loads per stage
  constexpr bool SPLIT_QK = NT <= 2;       // two QK accumulation chains when registers allow
  static_assert(kStageTokens % RPP == 0, "loader shape");
  static_assert(NST == 2 || NST == 3, "prologue handles 2 or 3 stages");
  static_assert(SP.total <= (size_t)kSmemBudget, "shared-memory plan over budget");
  extern __shared__ __align__(128) uint8_t smem[];
  int *flag = reinterpret_cast<int *>(smem + SP.total - 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint32_t u = blockIdx.x;
  const int s = (int)(u % (uint32_t)p.S);
  u /= (uint32_t)p.S;
  const int ht = (int)(u % (uint32_t)p.HT);
  u /= (uint32_t)p.HT;
  const int kvh = (int)(u % (uint32_t)p.Hkv);
  const int b = (int)(u / (uint32_t)p.Hkv);
  const int h0 = kvh * p.g + ht * HPT;  // this unit serves query heads h0 .. h0+gl-1
  const int gl = min(HPT, p.g - ht * HPT);
  const int capacity = p.max_blocks << p.bs_log2;

  int L = __ldg(p.seq_lens + b);
  if (L < 0 || L > capacity) {
    if (tid == 0 && s == 0 && kvh == 0 && ht == 0) atomicOr(p.err, kErrSeqLen);
    L = L < 0 ? 0 : capacity;
  }
  const int t0 = s * p.P;
  const int t1 = min(t0 + p.P, L);
  if (t0 >= t1) {
    if (L == 0 && s == 0) {  // empty sequence: out = 0, lse = -inf
      for (int i = tid; i < gl * D; i += kThreads)
        p.out[b * p.o_sb + (int64_t)(h0 + i / D) * p.o_sh + (i % D)] = 0;
      if (p.lse != nullptr && tid < gl) p.lse[b * p.lse_sb + (int64_t)(h0 + tid) * p.lse_sh] = -INFINITY;
    }
    return;
  }
  const int ns = (L + p.P - 1) / p.P;  // non-empty partitions of sequence b
  const int nstages = (t1 - t0 + kStageTokens - 1) / kStageTokens;

  // ---- K/V loader: thread (lr, lc) copies 16-byte chunk lc of rows lr, lr+RPP,
  // ... of a stage; row r, chunk c lands at r*ROWB + ((c ^ (r & 7)) * 16).
  const int32_t *trow = p.tables + (int64_t)b * p.table_stride;
  const int lc = tid % CH, lr = tid / CH;
  const int64_t kh_k = (int64_t)kvh * p.k_sh + lc * 8, kh_v = (int64_t)kvh * p.v_sh + lc * 8;
  int pid[NR];  // block ids of this thread's rows in the next stage to issue
  auto load_ids = [&](int (&ids)[NR], int st) {
    const int base = t0 + st * kStageTokens + lr;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int t = base + i * RPP;
      ids[i] = t < t1 ? __ldg(trow + (t >> p.bs_log2)) : 0;
    }
  };
  auto issue = [&](const int (&ids)[NR], int st) {
    uint8_t *sK = smem + (st % NST) * STAGE_BYTES;
    uint8_t *sV = sK + kStageTokens * ROWB;
    const int base = t0 + st * kStageTokens;
#pragma unroll
    for (int i = 0; i < NR; ++i) {
      const int r = lr + i * RPP;
      const int t = base + r;
      bool valid = t < t1;
      const uint16_t *ks = p.k, *vs = p.v;
      if (valid) {
        const int phys = ids[i];
        if ((unsigned)phys < (unsigned)p.num_blocks) {
          const int slot = t & ((1 << p.bs_log2) - 1);
          ks = p.k + (int64_t)phys * p.k_sblk + kh_k + (int64_t)slot * p.k_ss;
          vs = p.v + (int64_t)phys * p.v_sblk + kh_v + (int64_t)slot * p.v_ss;
        } else {
          atomicOr(p.err, kErrBlockId);  // never dereferenced: the row reads as zero
          valid = false;
        }
      }
      const uint32_t off = r * ROWB + ((lc ^ (r & 7)) << 4);
      cp_async_16(smem_addr(sK + off), ks, valid);
      cp_async_16(smem_addr(sV + off), vs, valid);
    }
  };

  // Q^T fragments (B operand of S^T = K.Q^T), loaded first so their latency
  // overlaps the block-table reads: lane holds head nt*8 + lane/4,
  // dims 16kk + 2(lane%4) + {0,1} and + {8,9}.  Padded heads are zero.
  uint32_t qf[KT][NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    const int hl = nt * 8 + (lane >> 2);
    const bool ok = hl < gl;
    const uint16_t *qr = p.q + b * p.q_sb + (int64_t)(h0 + (ok ? hl : 0)) * p.q_sh + (lane & 3) * 2;
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      qf[kk][nt][0] = ok ? __ldg(reinterpret_cast<const uint32_t *>(qr + kk * 16)) : 0u;
      qf[kk][nt][1] = ok ? __ldg(reinterpret_cast<const uint32_t *>(qr + kk * 16 + 8)) : 0u;
    }
  }

  // Prologue: the page ids of the first two stages are fetched together, then
  // stages 0 .. NST-2 are issued; pid ends up holding stage NST-1's ids.
  {
    int pid2[NR];
    load_ids(pid, 0);
    if (nstages > 1) load_ids(pid2, 1);
    issue(pid, 0);
    cp_async_commit();
    if constexpr (NST == 3) {
      if (nstages > 1) {
        issue(pid2, 1);
        if (nstages > 2) load_ids(pid, 2);
      }
      cp_async_commit();
    } else {
#pragma unroll
      for (int i = 0; i < NR; ++i) pid[i] = pid2[i];
    }
  }

  float oacc[KT][NT][4];
  float m_run[NT][2], l_run[NT][2];
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
      for (int i = 0; i < 4; ++i) oacc[mt][nt][i] = 0.f;
  }

#pragma unroll 1
  for (int st = 0; st < nstages; ++st) {
    const int nx = st + NST - 1;
    if (nx < nstages) {
      issue(pid, nx);                          // ids fetched one stage ago
      if (nx + 1 < nstages) load_ids(pid, nx + 1);  // in flight during this stage's math
    }
    cp_async_commit();
    cp_async_wait<NST - 1>();  // stage st has landed (this thread's copies)
    __syncthreads();           // ... and every other thread's

    const uint8_t *sK = smem + (st % NST) * STAGE_BYTES;
    const uint8_t *sV = sK + kStageTokens * ROWB;
    const int tbase = t0 + st * kStageTokens + warp * 16;
    if (tbase < t1) {
      // ---- S^T = K . Q^T over this warp's 16 tokens
      float sc[NT][4], sc2[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[nt][i] = sc2[nt][i] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = kk * 2 + (lane >> 4);
        uint32_t a[4];
        ldsm_x4(a, smem_addr(sK + r * ROWB + ((ch ^ (r & 7)) << 4)));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (SPLIT_QK && (kk & 1))
            mma_16816(sc2[nt], a, qf[kk][nt][0], qf[kk][nt][1]);
          else
            mma_16816(sc[nt], a, qf[kk][nt][0], qf[kk][nt][1]);
        }
      }

      // ---- online softmax (rows lane/4 and lane/4 + 8; columns 2(lane%4) + {0,1})
      const bool okA = tbase + (lane >> 2) < t1;
      const bool okB = tbase + (lane >> 2) + 8 < t1;
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
        // row 0 of the tile is a live token, so the new maxima are finite
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
          oacc[mt][nt][0] *= al0;
          oacc[mt][nt][1] *= al1;
          oacc[mt][nt][2] *= al0;
          oacc[mt][nt][3] *= al1;
        }
        pb[nt][0] = movmatrix_t(pA);
        pb[nt][1] = movmatrix_t(pB);
      }

      // ---- O^T += V^T . P^T  (rows past t1 were zero-filled, their weights are 0)
#pragma unroll
      for (int mt = 0; mt < KT; ++mt) {
        const int j = lane >> 3;
        const int r = warp * 16 + (lane & 7) + (j >> 1) * 8;
        const int ch = mt * 2 + (j & 1);
        uint32_t a[4];
        ldsm_x4_t(a, smem_addr(sV + r * ROWB + ((ch ^ (r & 7)) << 4)));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(oacc[mt][nt], a, pb[nt][0], pb[nt][1]);
      }
    }
    __syncthreads();  // every warp is done with slot st % NST before it is refilled
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- merge the four warps' states through shared memory (the ring is free);
  // rows padded to D+4 floats so the fragment stores below are conflict free
  constexpr int MROW = D + 4;
  float *sm_o = reinterpret_cast<float *>(smem);  // [kWarps][HPT][MROW]
  float *sm_m = sm_o + kWarps * HPT * MROW;        // [kWarps][HPT]
  float *sm_l = sm_m + kWarps * HPT;               // [kWarps][HPT]
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[nt][j];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      if (lane < 4) {
        sm_m[warp * HPT + nt * 8 + 2 * lane + j] = m_run[nt][j];
        sm_l[warp * HPT + nt * 8 + 2 * lane + j] = l;
      }
    }
#pragma unroll
    for (int mt = 0; mt < KT; ++mt) {
      const int d = mt * 16 + (lane >> 2);
      float *o0 = sm_o + (warp * HPT + nt * 8 + (lane & 3) * 2) * MROW;
      o0[d] = oacc[mt][nt][0];
      o0[MROW + d] = oacc[mt][nt][1];
      o0[d + 8] = oacc[mt][nt][2];
      o0[MROW + d + 8] = oacc[mt][nt][3];
    }
  }
  __syncthreads();

  constexpr int D4 = D / 4;
  for (int i = tid; i < gl * D4; i += kThreads) {
    const int hl = i / D4, d = (i % D4) * 4;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) m = fmaxf(m, sm_m[w * HPT + hl]);
    float l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = sm_m[w * HPT + hl];
      if (mw == -INFINITY) continue;  // warp saw no token of this partition
      const float f = fast_exp2(mw - m);
      l += f * sm_l[w * HPT + hl];
      const float4 ow = *reinterpret_cast<const float4 *>(sm_o + (w * HPT + hl) * MROW + d);
      o.x += f * ow.x;
      o.y += f * ow.y;
      o.z += f * ow.z;
      o.w += f * ow.w;
    }
    const float inv = 1.f / l;
    const float lse_nat = (m + log2f(l)) * kLn2;
    const int h = h0 + hl;
    if (ns == 1) {
      uint2 packed;
      packed.x = pack_bf16x2(o.x * inv, o.y * inv);
      packed.y = pack_bf16x2(o.z * inv, o.w * inv);
      *reinterpret_cast<uint2 *>(p.out + b * p.o_sb + (int64_t)h * p.o_sh + d) = packed;
      if (d == 0 && p.lse != nullptr) p.lse[b * p.lse_sb + (int64_t)h * p.lse_sh] = lse_nat;
    } else {
      const int64_t row = ((int64_t)b * p.Hq + h) * p.S + s;
      *reinterpret_cast<float4 *>(p.o_part + row * D + d) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      if (d == 0) p.lse_part[row] = lse_nat;
    }
  }
  if (ns == 1) return;

  // ---- split reduce: the CTA that finishes the set's last partition merges it.
  // The barrier orders every thread's partial stores before thread 0's fence,
  // which publishes them (cumulatively) before the count.
  __syncthreads();
  if (tid == 0) {
    const uint32_t pair = ((uint32_t)b * p.Hkv + kvh) * p.HT + ht;
    __threadfence();
    const uint32_t done = atomicAdd(p.counters + pair, 1u);
    const int last = done + 1 == (uint32_t)ns;
    if (last) {
      atomicExch(p.counters + pair, 0u);  // ready for the next launch
      __threadfence();                    // the other partials' stores, before the loads below
    }
    *flag = last;
  }
  __syncthreads();
  if (!*flag) return;

  // weights w[hl][s] = exp(lse_s - M) / sum, in shared memory (the ring is free)
  float *wt = reinterpret_cast<float *>(smem);  // [HPT][ns]
  const int64_t row0 = ((int64_t)b * p.Hq + h0) * p.S;
  for (int i = tid; i < gl * ns; i += kThreads) {
    const int hl = i / ns, si = i % ns;
    wt[hl * ns + si] = ld_cg_f32(p.lse_part + row0 + (int64_t)hl * p.S + si);
  }
  __syncthreads();
  for (int hl = warp; hl < gl; hl += kWarps) {
    float M = -INFINITY;
    for (int si = lane; si < ns; si += 32) M = fmaxf(M, wt[hl * ns + si]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float sum = 0.f;
    for (int si = lane; si < ns; si += 32) sum += __expf(wt[hl * ns + si] - M);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float inv = 1.f / sum;
    __syncwarp();
    for (int si = lane; si < ns; si += 32) wt[hl * ns + si] = __expf(wt[hl * ns + si] - M) * inv;
    if (lane == 0 && p.lse != nullptr) p.lse[b * p.lse_sb + (int64_t)(h0 + hl) * p.lse_sh] = M + logf(sum);
  }
  __syncthreads();
  for (int i = tid; i < gl * D4; i += kThreads) {
    const int hl = i / D4, d = (i % D4) * 4;
    const float *orow = p.o_part + (row0 + (int64_t)hl * p.S) * D + d;
    const float *w = wt + hl * ns;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int si = 0;
    for (; si + 4 <= ns; si += 4) {
      float4 ov[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) ov[j] = ld_cg_f4(orow + (int64_t)(si + j) * D);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float wj = w[si + j];
        acc.x += wj * ov[j].x;
        acc.y += wj * ov[j].y;
        acc.z += wj * ov[j].z;
        acc.w += wj * ov[j].w;
      }
    }
    for (; si < ns; ++si) {
      const float4 ov = ld_cg_f4(orow + (int64_t)si * D);
      const float wj = w[si];
      acc.x += wj * ov.x;
      acc.y += wj * ov.y;
      acc.z += wj * ov.z;
      acc.w += wj * ov.w;
    }
    uint2 packed;
    packed.x = pack_bf16x2(acc.x, acc.y);
    packed.y = pack_bf16x2(acc.z, acc.w);
    *reinterpret_cast<uint2 *>(p.out + b * p.o_sb + (int64_t)(h0 + hl) * p.o_sh + d) = packed;
  }
}

int partition_stages(int D, int hpt) { return stages_for(D, hpt); }

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
