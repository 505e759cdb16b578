// Internal launch parameters shared by the host API and the kernel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pad.h"

namespace pad {

enum : uint32_t {
  kErrBlockId = 0x1u,   // a live table entry outside [0, num_blocks)
  kErrSeqLen = 0x2u,    // seq_lens[b] < 0 or > table capacity
  kErrTimeout = 0x4u,   // a bounded wait inside the kernel gave up (a bug); workspace counters may be stale
};

// Kernel geometry: 4 worker warps (each loads and computes one 16-token sub-tile
// of every 64-token stage), one scheduler warp, one merger warp.
constexpr int kWorkers = 4;
constexpr int kThreads = (kWorkers + 2) * 32;
constexpr int kStageTokens = 16 * kWorkers;
constexpr int kSmemBudget = 232448;  // 227 KiB per CTA
constexpr int kDescBytes = 288;      // one stage descriptor (header + 64 block ids)
constexpr int kMaxDescs = 10;

// Shared-memory plan of one (head_dim, heads-per-tile) instantiation.
//
// The q ring has one slot per pipeline stage.  A worker looks NST-1 stages
// past the one it computes, and those NST stages belong to at most NST units,
// so the scheduler never needs a q slot that only the worker's current
// computation would free (with fewer slots, short units deadlock the pipeline).
struct SmemPlan {
  int stages, merge_slots, q_slots;
  size_t sub_bytes, stage_bytes, ring_bytes, q_row_bytes, q_slot_bytes, q_bytes, merge_bytes, desc_bytes, misc_bytes,
      total;
};

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ constexpr SmemPlan smem_plan_with(int D, int hpt, int merge_slots) {
  SmemPlan s{};
  s.merge_slots = merge_slots;
  s.sub_bytes = (size_t)16 * D * 2 * 2;  // one worker's 16 rows of K and of V
  s.stage_bytes = s.sub_bytes * kWorkers;
  s.q_row_bytes = (size_t)D * 2 + 16;    // padded: conflict-free fragment loads
  s.q_slot_bytes = (size_t)hpt * s.q_row_bytes;
  // a merge slot holds one worker's (O^T, m, l) for the head tile
  s.merge_bytes = align_up((size_t)merge_slots * ((size_t)hpt * (D + 4) + 2 * hpt) * 4, 128);
  s.desc_bytes = (size_t)kMaxDescs * kDescBytes;
  s.misc_bytes = 512;  // mbarriers, flags
  const size_t fixed = 1024 /* ring alignment slack */ + 128 /* q rounding */ + s.merge_bytes + s.desc_bytes +
                       s.misc_bytes;
  int st = (int)((kSmemBudget - fixed) / (s.stage_bytes + s.q_slot_bytes));
  if (st > kMaxDescs - 2) st = kMaxDescs - 2;
  s.stages = st;
  s.q_slots = st;
  s.ring_bytes = (size_t)st * s.stage_bytes;
  s.q_bytes = align_up((size_t)st * s.q_slot_bytes, 128);
  s.total = fixed - 128 + s.ring_bytes + s.q_bytes;
  return s;
}

// Three merge slots (one per non-leading worker) unless that costs a pipeline stage.
__host__ __device__ constexpr SmemPlan smem_plan_for(int D, int hpt) {
  const SmemPlan a = smem_plan_with(D, hpt, kWorkers - 1), b = smem_plan_with(D, hpt, 1);
  return a.stages >= b.stages ? a : b;
}

// Largest query-head tile whose fp32 O^T accumulator (D x heads) fits one worker's registers.
inline int max_heads_per_tile(int D) { return D <= 128 ? 32 : 16; }

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
  int32_t HT;       // head tiles per KV head: ceil(g / heads per tile)
  int32_t bs_log2;
  int32_t P;        // tokens per partition (multiple of the block size)
  int32_t S;        // partitions per sequence (capacity / P)
  uint32_t n_units; // B * Hkv * HT * S
  float scale_log2; // scale * log2(e)
  uint16_t *out;
  int64_t o_sb, o_sh;
  float *lse;  // may be null
  int64_t lse_sb, lse_sh;
  float *o_part;       // [B, Hq, S, D] fp32
  float *lse_part;     // [B, Hq, S] fp32 (natural log)
  uint32_t *counters;  // [B * Hkv * HT] partitions finished per (b, kv head, head tile)
  uint32_t *ctl;       // [0] next unit to claim, [1] CTAs finished
  uint32_t *err;
};

// Partials layout inside a workspace buffer (offsets 256-byte aligned); empty
// when S == 1.
struct WorkspaceLayout {
  size_t o_part, lse_part, total;
};

inline WorkspaceLayout workspace_layout(int64_t B, int64_t Hq, int64_t S, int64_t D) {
  WorkspaceLayout w{};
  if (S <= 1) return w;
  w.o_part = 0;
  w.lse_part = align_up((size_t)(B * Hq * S * D * 4), 256);
  w.total = w.lse_part + align_up((size_t)(B * Hq * S * 4), 256);
  return w;
}

// Control block: the claim word and CTA count (first 256 bytes), then one merge
// counter per (b, kv head, head tile) when S > 1.  Must be zero when a launch
// starts; a launch that completes leaves it zero.
struct ControlLayout {
  size_t ctl, counters, total;
};

inline ControlLayout control_layout(int64_t B, int64_t Hkv, int64_t HT, int64_t S) {
  ControlLayout c{};
  c.ctl = 0;
  c.counters = 256;
  c.total = 256 + (S > 1 ? align_up((size_t)(B * Hkv * HT * 4), 256) : 0);
  return c;
}

cudaError_t launch_partition(const PartitionParams &p, int D, int heads_per_tile, int grid, cudaStream_t s);
int partition_stages(int D, int heads_per_tile);
cudaError_t device_error_word(int device, uint32_t **ptr);
void set_last_error(const char *msg);

// pad_decode with explicit buffers: `partials` (>= the plan's workspace_bytes,
// 256-byte aligned) and `control` (>= the plan's control_bytes, zero at launch).
// Used by the allocation-free entry point; allocates nothing itself.
pad_status decode_with_buffers(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                               const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                               int32_t num_splits, pad_tensor *out, pad_tensor *lse, void *partials,
                               size_t partials_bytes, void *control, size_t control_bytes, cudaStream_t stream);

}  // namespace pad
