// Split-reduce kernel: merges the per-partition partial outputs of one
// (sequence, query head) by their log-sum-exp ("perf(rocke): prepare saved paged
// decode bindings once", section "Summary": the split-KV pass is followed by a
// reduce pass that takes the output pointer, the sequence lengths and, when
// requested, the LSE pointer).
//
//   M   = max_s lse_s
//   lse = M + log(sum_s exp(lse_s - M))
//   out = sum_s exp(lse_s - lse) * o_s        (o_s already normalised by its own sum)
//
// Only the ceil(L_b / P) partitions that hold tokens are read; empty ones were
// never written.  One warp per (b, h); each lane owns D/32 contiguous dims, so a
// partition row is one coalesced read per warp.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "pad_device.cuh"
#include "pad_internal.h"

namespace pad {

template <int D>
__global__ void __launch_bounds__(128) reduce_kernel(const ReduceParams p) {
  constexpr int E = D / 32;  // dims per lane: 2, 4 or 8
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int idx = blockIdx.x * 4 + warp;
  if (idx >= p.B * p.Hq) return;
  const int b = idx / p.Hq, h = idx % p.Hq;
  int L = __ldg(p.seq_lens + b);
  L = L < 0 ? 0 : (L > p.capacity ? p.capacity : L);
  const int ns = (L + p.P - 1) / p.P;
  uint16_t *orow = p.out + b * p.o_sb + (int64_t)h * p.o_sh + lane * E;
  float *lse_out = p.lse != nullptr ? p.lse + b * p.lse_sb + (int64_t)h * p.lse_sh : nullptr;

  if (ns == 0) {
#pragma unroll
    for (int e = 0; e < E; ++e) orow[e] = 0;
    if (lane == 0 && lse_out != nullptr) *lse_out = -INFINITY;
    return;
  }

  const int64_t row0 = ((int64_t)b * p.Hq + h) * p.S;
  const float *lp = p.lse_part + row0;
  float M = -INFINITY;
  for (int s = lane; s < ns; s += 32) M = fmaxf(M, __ldg(lp + s));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float sum = 0.f;
  for (int s = lane; s < ns; s += 32) sum += expf(__ldg(lp + s) - M);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);

  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  const float *op = p.o_part + row0 * D + lane * E;
#pragma unroll 4
  for (int s = 0; s < ns; ++s) {
    const float w = expf(__ldg(lp + s) - M);
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float2 v = __ldg(reinterpret_cast<const float2 *>(op + (int64_t)s * D + e));
      acc[e] += w * v.x;
      acc[e + 1] += w * v.y;
    }
  }
  const float inv = 1.f / sum;
#pragma unroll
  for (int e = 0; e < E; e += 2)
    *reinterpret_cast<uint32_t *>(orow + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
  if (lane == 0 && lse_out != nullptr) *lse_out = M + logf(sum);
}

cudaError_t launch_reduce(const ReduceParams &p, cudaStream_t s) {
  const unsigned pairs = (unsigned)p.B * (unsigned)p.Hq;
  const unsigned grid = (pairs + 3) / 4;
  switch (p.D) {
    case 64: reduce_kernel<64><<<grid, 128, 0, s>>>(p); break;
    case 128: reduce_kernel<128><<<grid, 128, 0, s>>>(p); break;
    case 256: reduce_kernel<256><<<grid, 128, 0, s>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace pad
