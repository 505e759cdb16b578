// Partition kernel: one CTA per (sequence b, KV head, head tile, token partition s).
//
// The CTA streams its partition's K and V pages for one KV head from HBM into a
// 3-stage shared-memory ring (16-byte cp.async per lane, XOR-swizzled rows so the
// tensor-core operand loads are bank-conflict free), and serves every query head
// of the GQA group from that single read ("spec(BACKEND-ROCM): the ROCm
// head_dim=128 decode arm", section "It is a mirror of merged work, not new
// design": PagedAttnDecodeGqaBf16 fuses a GQA group over one K/V read; its
// vectorised 16-byte loads).
//
// Each warp owns 16 tokens of every 64-token stage and keeps its own running max
// and sum per head (the warp-strided online softmax of the same section: warps
// walk disjoint token subsets and are merged at the end, so the sum is taken in
// a different order than a sequential kernel, not bitwise equal to it).
//
// Per 16-token tile, with the group's heads padded to NT*8 columns:
//   S^T[16 tok x 8 heads] = K[16 x D] . Q^T          (mma.m16n8k16, fp32 accum)
//   P^T = exp2(S^T * scale*log2e - m)                 (per-head running max m)
//   O^T[D x 8 heads]     += V^T[D x 16 tok] . P^T     (P^T moved from the S^T
//                                                      accumulator layout into the
//                                                      B-operand layout by movmatrix)
// With one partition per sequence the CTA writes bf16 out (+ lse); otherwise it
// writes the fp32 partial out (normalised by its own sum) and its lse for the
// split-reduce kernel ("perf(rocke): prepare saved paged decode bindings once",
// section "Summary": split-KV attention followed by a reduce pass).
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "pad_device.cuh"
#include "pad_internal.h"

namespace pad {

__device__ uint32_t g_err_word;

template <int D, int NT>
__global__ void __launch_bounds__(kThreads, (D <= 128 ? 2 : 1))
    partition_kernel(const PartitionParams p) {
  constexpr int CH = D / 8;  // 16-byte chunks per K/V row
  constexpr int ROWB = D * 2;
  constexpr int KT = D / 16;  // QK k-steps == PV m-tiles
  constexpr int NSTAGE = 3;
  constexpr int STAGE_BYTES = 2 * kStageTokens * ROWB;
  constexpr int HPT = NT * 8;
  constexpr int ROWS_PER_PASS = kThreads / CH;
  static_assert(kStageTokens % ROWS_PER_PASS == 0, "loader shape");
  extern __shared__ __align__(128) uint8_t smem[];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int s = blockIdx.x % p.S;
  int rest = blockIdx.x / p.S;
  const int ht = rest % p.HT;
  rest /= p.HT;
  const int kvh = rest % p.Hkv;
  const int b = rest / p.Hkv;
  // this CTA serves query heads h0 .. h0+gl-1 of KV head kvh's group
  const int h0 = kvh * p.g + ht * HPT;
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
    if (p.S == 1) {  // empty sequence: out = 0, lse = -inf
      for (int i = tid; i < gl * D; i += kThreads)
        p.out[b * p.o_sb + (int64_t)(h0 + i / D) * p.o_sh + (i % D)] = 0;
      if (p.lse != nullptr && tid < gl)
        p.lse[b * p.lse_sb + (int64_t)(h0 + tid) * p.lse_sh] = -INFINITY;
    }
    return;
  }

  // Q^T fragments (B operand of S^T = K.Q^T): lane holds head nt*8 + lane/4,
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

  // ---- K/V page loader: token row r of a stage, 16-byte chunk c lands at
  //      r*ROWB + ((c ^ (r & 7)) * 16).  Tokens past the partition are zero-filled
  //      without reading memory, so cache slots past L_b are never touched.
  const int32_t *trow = p.tables + (int64_t)b * p.table_stride;
  const int bs_mask = (1 << p.bs_log2) - 1;
  const int lc = tid % CH;
  const int lr = tid / CH;
  const int nstages = (t1 - t0 + kStageTokens - 1) / kStageTokens;

  auto issue = [&](int st) {
    uint8_t *sK = smem + (st % NSTAGE) * STAGE_BYTES;
    uint8_t *sV = sK + kStageTokens * ROWB;
    const int base = t0 + st * kStageTokens;
#pragma unroll
    for (int r = lr; r < kStageTokens; r += ROWS_PER_PASS) {
      const int t = base + r;
      bool valid = t < t1;
      const uint16_t *ks = p.k, *vs = p.v;
      if (valid) {
        const int phys = __ldg(trow + (t >> p.bs_log2));
        if ((unsigned)phys < (unsigned)p.num_blocks) {
          const int slot = t & bs_mask;
          ks = p.k + phys * p.k_sblk + kvh * p.k_sh + slot * p.k_ss + lc * 8;
          vs = p.v + phys * p.v_sblk + kvh * p.v_sh + slot * p.v_ss + lc * 8;
        } else {
          atomicOr(p.err, kErrBlockId);
          valid = false;
        }
      }
      const uint32_t off = r * ROWB + ((lc ^ (r & 7)) << 4);
      cp_async_16(smem_addr(sK + off), ks, valid);
      cp_async_16(smem_addr(sV + off), vs, valid);
    }
  };

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
  for (int st = 0; st < NSTAGE - 1; ++st) {
    if (st < nstages) issue(st);
    cp_async_commit();
  }

#pragma unroll 1
  for (int st = 0; st < nstages; ++st) {
    if (st + NSTAGE - 1 < nstages) issue(st + NSTAGE - 1);
    cp_async_commit();
    cp_async_wait<NSTAGE - 1>();
    __syncthreads();

    const uint8_t *sK = smem + (st % NSTAGE) * STAGE_BYTES;
    const uint8_t *sV = sK + kStageTokens * ROWB;
    const int tbase = t0 + st * kStageTokens + warp * 16;
    if (tbase < t1) {
      // S^T = K . Q^T
      float sc[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sc[nt][i] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        const int r = warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = kk * 2 + (lane >> 4);
        uint32_t a[4];
        ldsm_x4(a, smem_addr(sK + r * ROWB + ((ch ^ (r & 7)) << 4)));
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(sc[nt], a, qf[kk][nt][0], qf[kk][nt][1]);
      }

      // online softmax over this tile's 16 tokens (rows lane/4 and lane/4 + 8)
      const bool okA = tbase + (lane >> 2) < t1;
      const bool okB = tbase + (lane >> 2) + 8 < t1;
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
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
        // Row 0 of the tile is a live token, so the new maxima are finite.
        const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
        const float al0 = fast_exp2(m_run[nt][0] - mn0), al1 = fast_exp2(m_run[nt][1] - mn1);
        m_run[nt][0] = mn0;
        m_run[nt][1] = mn1;
        const uint32_t pA = pack_bf16x2(fast_exp2(s0 - mn0), fast_exp2(s1 - mn1));
        const uint32_t pB = pack_bf16x2(fast_exp2(s2 - mn0), fast_exp2(s3 - mn1));
        // the running sum uses the same bf16-rounded weights the MMA sees
        l_run[nt][0] = l_run[nt][0] * al0 + __uint_as_float(pA << 16) + __uint_as_float(pB << 16);
        l_run[nt][1] = l_run[nt][1] * al1 + __uint_as_float(pA & 0xffff0000u) +
                       __uint_as_float(pB & 0xffff0000u);
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

      // O^T += V^T . P^T
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
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- merge the four warps' states through shared memory (the ring is free now)
  float *sm_o = reinterpret_cast<float *>(smem);  // [kWarps][HPT][D]
  float *sm_m = sm_o + kWarps * HPT * D;           // [kWarps][HPT]
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
      float *o0 = sm_o + (warp * HPT + nt * 8 + (lane & 3) * 2) * D;
      o0[d] = oacc[mt][nt][0];
      o0[D + d] = oacc[mt][nt][1];
      o0[d + 8] = oacc[mt][nt][2];
      o0[D + d + 8] = oacc[mt][nt][3];
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
      const float4 ow = *reinterpret_cast<const float4 *>(sm_o + (w * HPT + hl) * D + d);
      o.x += f * ow.x;
      o.y += f * ow.y;
      o.z += f * ow.z;
      o.w += f * ow.w;
    }
    const float inv = 1.f / l;
    const float lse_nat = (m + log2f(l)) * 0.69314718055994530942f;
    const int h = h0 + hl;
    if (p.S == 1) {
      uint2 packed;
      packed.x = pack_bf16x2(o.x * inv, o.y * inv);
      packed.y = pack_bf16x2(o.z * inv, o.w * inv);
      *reinterpret_cast<uint2 *>(p.out + b * p.o_sb + (int64_t)h * p.o_sh + d) = packed;
      if (d == 0 && p.lse != nullptr) p.lse[b * p.lse_sb + (int64_t)h * p.lse_sh] = lse_nat;
    } else {
      const int64_t row = ((int64_t)b * p.Hq + h) * p.S + s;
      *reinterpret_cast<float4 *>(p.o_part + row * D + d) =
          make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      if (d == 0) p.lse_part[row] = lse_nat;
    }
  }
}

template <int D, int NT>
static cudaError_t launch_t(const PartitionParams &p, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  const size_t smem = partition_smem_bytes(D, NT * 8);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(partition_kernel<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  const unsigned grid = (unsigned)p.B * (unsigned)p.Hkv * (unsigned)p.HT * (unsigned)p.S;
  partition_kernel<D, NT><<<grid, kThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_d(const PartitionParams &p, int hpt, cudaStream_t s) {
  if (hpt > max_heads_per_tile(D)) return cudaErrorInvalidValue;
  switch (hpt) {
    case 8: return launch_t<D, 1>(p, s);
    case 16: return launch_t<D, 2>(p, s);
    case 32: return launch_t<D, (D <= 128 ? 4 : 2)>(p, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_partition(const PartitionParams &p, int D, int heads_per_tile, cudaStream_t s) {
  switch (D) {
    case 64: return launch_d<64>(p, heads_per_tile, s);
    case 128: return launch_d<128>(p, heads_per_tile, s);
    case 256: return launch_d<256>(p, heads_per_tile, s);
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
