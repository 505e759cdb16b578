// Internal launch parameters shared by the host API and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace pad {

enum : uint32_t {
  kErrBlockId = 0x1u,  // a live table entry outside [0, num_blocks)
  kErrSeqLen = 0x2u,   // seq_lens[b] < 0 or > table capacity
};

struct PartitionParams {
  const uint16_t *q;
  int64_t q_sb, q_sh;  // element strides over (b, h); d is contiguous
  const uint16_t *k;
  const uint16_t *v;
  int64_t k_sblk, k_sh, k_ss;  // element strides over (block, kv head, slot)
  int64_t v_sblk, v_sh, v_ss;
  const int32_t *tables;
  int64_t table_stride;
  int32_t max_blocks;  // table width
  int32_t num_blocks;
  const int32_t *seq_lens;
  int32_t B, Hq, Hkv, g;
  int32_t HT;  // head tiles per KV head: ceil(g / heads per tile)
  int32_t bs_log2;
  int32_t P;  // tokens per partition
  int32_t S;  // partitions per sequence
  float scale_log2;  // scale * log2(e)
  uint16_t *out;
  int64_t o_sb, o_sh;
  float *lse;  // may be null
  int64_t lse_sb, lse_sh;
  float *o_part;    // [B, Hq, S, D] fp32, S > 1 only
  float *lse_part;  // [B, Hq, S] fp32 (natural log), S > 1 only
  uint32_t *err;
};

struct ReduceParams {
  const float *o_part;
  const float *lse_part;
  const int32_t *seq_lens;
  int32_t B, Hq, D, S, P, capacity;
  uint16_t *out;
  int64_t o_sb, o_sh;
  float *lse;
  int64_t lse_sb, lse_sh;
};

// Partition-kernel geometry (fixed for this kernel family).
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kStageTokens = 16 * kWarps;  // one 16-token MMA tile per warp per stage

inline int stages_for(int D) { return 3; }
// Largest query-head tile whose fp32 O^T accumulator (D x heads) fits in registers.
inline int max_heads_per_tile(int D) { return D <= 128 ? 32 : 16; }
inline size_t partition_smem_bytes(int D, int heads_per_tile) {
  size_t ring = (size_t)stages_for(D) * 2 * kStageTokens * D * 2;
  size_t merge = (size_t)kWarps * heads_per_tile * (D + 2) * 4;
  return ring > merge ? ring : merge;
}

cudaError_t launch_partition(const PartitionParams &p, int D, int heads_per_tile, cudaStream_t s);
cudaError_t launch_reduce(const ReduceParams &p, cudaStream_t s);
cudaError_t device_error_word(int device, uint32_t **ptr);

}  // namespace pad

namespace pad {
void set_last_error(const char *msg);
}  // namespace pad
