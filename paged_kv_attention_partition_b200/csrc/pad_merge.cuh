// The split reduce folded into the partition launches ("perf(rocke): prepare
// saved paged decode bindings once", section "Summary": split-KV attention
// followed by a reduce pass), shared by the mma.sync and tcgen05 kernels.
//
// Every partition of a sequence with ns > 1 non-empty partitions writes its
// partial output o_s (normalised by its own sum) and lse_s.  The CTA whose
// count brings the (b, KV head, head tile) counter to ns merges the set:
//   M = max_s lse_s,  lse = M + log sum_s exp(lse_s - M),
//   out = sum_s w_s o_s with w_s = exp(lse_s - lse).
// With attention sinks the head's sink logit joins the denominator:
//   lse' = logaddexp(lse, sink), w_s = exp(lse_s - lse').
#pragma once

#include <math.h>
#include <stdint.h>

#include "pad_device.cuh"
#include "pad_internal.h"

namespace pad {

// Barriers over the threads that take part: the whole CTA, or the 128 threads
// of warps 0-3 (named barrier 1) while other warps of the CTA run on.
struct CtaSync {
  __device__ __forceinline__ void operator()() const { __syncthreads(); }
};
struct Warps0to3Sync {
  __device__ __forceinline__ void operator()() const { asm volatile("bar.sync 1, 128;\n" ::: "memory"); }
};

// Counts this partition; true (in every participating thread) for the CTA that
// completes the set, which also resets the counter for the next launch.  The
// barrier orders every participant's partial stores before thread 0's count, a
// release-acquire atomic at GPU scope: its release publishes them
// (cumulatively), and in the CTA that completes the set its acquire orders the
// other partitions' stores, published by their releases to the same counter,
// before the merge's loads (which the next barrier passes on to every
// participant).  Every participating thread calls it; thread 0 must be one of
// them.
template <class Sync = CtaSync>
__device__ __forceinline__ bool claim_last_partition(const PartitionParams &p, int b, int kvh, int ht, int ns,
                                                     int *flag, Sync sync = Sync()) {
  sync();
  if (threadIdx.x == 0) {
    const uint32_t pair = ((uint32_t)b * p.Hkv + kvh) * p.HT + ht;
    uint32_t done;
    asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;\n" : "=r"(done) : "l"(p.counters + pair) : "memory");
    const int last = done + 1 == (uint32_t)ns;
    if (last) atomicExch(p.counters + pair, 0u);  // ready for the next launch
    *flag = last;
  }
  sync();
  const bool last = *flag != 0;
  sync();  // every participant has read the flag before it is written again
  return last;
}

// Merges partials s_first .. s_first+ns-1 of query heads h0 .. h0+gl-1 of
// sequence b into bf16 out (+ lse).  `wt` is shared memory for gl * ns floats.
// The NTHREADS participating threads (threadIdx.x 0 .. NTHREADS-1) call it.
template <int D, int NTHREADS, class Sync = CtaSync>
__device__ void merge_partials(const PartitionParams &p, int b, int h0, int gl, int s_first, int ns, float *wt,
                               Sync sync = Sync()) {
  constexpr int D4 = D / 4, NW = NTHREADS / 32;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t row0 = ((int64_t)b * p.Hq + h0) * p.S + s_first;
  for (int i = tid; i < gl * ns; i += NTHREADS) {
    const int hl = i / ns, si = i % ns;
    wt[hl * ns + si] = ld_cg_f32(p.lse_part + row0 + (int64_t)hl * p.S + si);
  }
  sync();
  for (int hl = warp; hl < gl; hl += NW) {
    float M = -INFINITY;
    for (int si = lane; si < ns; si += 32) M = fmaxf(M, wt[hl * ns + si]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float sum = 0.f;
    for (int si = lane; si < ns; si += 32) sum += __expf(wt[hl * ns + si] - M);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    float lse = M + logf(sum);
    if (p.sinks != nullptr) {
      const float sg = p.sinks[h0 + hl];
      lse = fmaxf(lse, sg) + log1pf(__expf(-fabsf(lse - sg)));
    }
    __syncwarp();
    for (int si = lane; si < ns; si += 32) wt[hl * ns + si] = __expf(wt[hl * ns + si] - lse);
    if (lane == 0 && p.lse != nullptr) p.lse[b * p.lse_sb + (int64_t)(h0 + hl) * p.lse_sh] = lse;
  }
  sync();
  for (int i = tid; i < gl * D4; i += NTHREADS) {
    const int hl = i / D4, d = (i % D4) * 4;
    const float *orow = p.o_part + (row0 + (int64_t)hl * p.S) * D + d;
    const float *w = wt + hl * ns;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    int si = 0;
    for (; si + 8 <= ns; si += 8) {  // eight partials in flight per thread
      float4 ov[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) ov[j] = ld_cg_f4(orow + (int64_t)(si + j) * D);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
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
  sync();  // `wt` is free again when the call returns
}

}  // namespace pad
