// Internal launch parameters shared by the host API and the kernel.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pad.h"

namespace pad {

enum : uint32_t {
  kErrBlockId = 0x1u,  // a live table entry outside [0, num_blocks)
  kErrSeqLen = 0x2u,   // seq_lens[b] < 0 or > table capacity
  kErrTimeout = 0x4u,  // a bounded wait for a stage's copies gave up (internal error)
};

// Kernel geometry: one CTA of NW warps (4 or 8) per work unit; one thread
// issues the stage copies (TMA), all warps compute.  A warp is (token group tg,
// head group hg, head_dim part dh):
//   - head groups split a head tile's 8-head n-tiles between warps: with 16 or
//     32 heads per tile each warp owns one n-tile and computes every token of the
//     stage for it (a quarter or half of the accumulator a warp holding the whole
//     tile would need, and each head's softmax stays inside one warp);
//   - head_dim parts split O^T's rows between the two warps of a pair that
//     compute the same scores (D = 256, bf16 8-head tiles at D = 128, and E4M3
//     8-head tiles at D = 128 with 8 warps: where a stage and the accumulator
//     would otherwise limit residency);
//   - the remaining warps form token groups: group tg computes 16-token tiles
//     tg, tg + TG, ... of every stage, and the groups merge at the end.
constexpr int kSmemBudget = 232448;  // 227 KiB per CTA
constexpr int kMaxSplits = 256;      // partitions per sequence (bounds the merge's weight table)

__host__ __device__ constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Warps per CTA of each (head_dim, heads-per-tile, cache type) instantiation,
// the measured choice (4 and 8 were timed on every named workload on B200).
__host__ __device__ constexpr int warps_for(int D, int hpt, bool f8) { return 4; }

__host__ __device__ constexpr int dsplit_for(int D, int hpt, bool f8, int nw) {
  return D == 256 ? 2 : (D == 128 && hpt == 8 && (nw == 8 || !f8) ? 2 : 1);
}
__host__ __device__ constexpr int head_groups_for(int D, int hpt, bool f8, int nw) {
  return (hpt / 8) * dsplit_for(D, hpt, f8, nw) <= nw ? hpt / 8 : nw / dsplit_for(D, hpt, f8, nw);
}
__host__ __device__ constexpr int token_groups_for(int D, int hpt, bool f8, int nw) {
  return nw / (dsplit_for(D, hpt, f8, nw) * head_groups_for(D, hpt, f8, nw));
}
// Tokens of one pipeline stage: 64; 32 at D = 256, whose rows are twice as
// long, and for bf16 8- and 32-head tiles at D = 128, whose 16 KB stages let
// five and four CTAs share an SM; an E4M3 cache at D = 256 with 8 or 16 heads
// per tile doubles them, so its stage carries as many bytes as a bf16 one.  At
// least one 16-token tile per token group.
__host__ __device__ constexpr int stage_tokens_for(int D, int hpt, bool f8, int nw) {
  int st = (D == 256 || (D == 128 && (hpt == 32 || hpt == 8) && !f8) ? 32 : 64) * (f8 && D == 256 && hpt <= 16 ? 2 : 1);
  while (st < 16 * token_groups_for(D, hpt, f8, nw)) st *= 2;
  return st;
}
// 16-token tiles a warp computes per stage.
__host__ __device__ constexpr int tiles_per_group(int D, int hpt, bool f8, int nw) {
  return stage_tokens_for(D, hpt, f8, nw) / (16 * token_groups_for(D, hpt, f8, nw));
}

// Pipeline depth and resident CTAs per SM of one (head_dim, heads-per-tile,
// cache type, warps) instantiation.  The ring is kept small so that several
// CTAs share each SM: their loads, math and start/finish latencies overlap one
// another.  The math is latency bound, so resident warps decide the speed.
// With 4 warps: an E4M3 cache at D = 128 with 8 or 16 heads per tile keeps two
// 16 KB stages and runs five (8 heads) or four (16 heads, whose accumulators
// would spill at five) CTAs per SM, registers capped to fit -- measured against
// deeper rings and two-tile stages at 2-4 CTAs per SM, which were slower.
// At D = 64 its 64-byte rows sit in boxes of at least 128 bytes, which caps
// it at three stages.  32-head tiles at D = 128 (one n-tile per warp, 128
// registers) run three 16 KB stages and four CTAs per SM for either cache
// type, measured against two 32 KB stages at three CTAs (ragged MQA batch:
// 177 -> 157 us bf16, 165 -> 159 us E4M3).  The bf16 8-head tile at D = 128
// splits head_dim over warp pairs (two token groups of two head_dim halves),
// which halves its accumulator (93 registers) and its stage (32 tokens, 16 KB):
// two stages and five CTAs per SM, measured against two 32 KB stages of four
// token groups at three CTAs (Qwen3-14B-shaped batch 349 -> 338 us, Llama-8B-
// shaped unchanged) and against three or four 16 KB stages at three or four
// CTAs (339-373 us).  With 8 warps: the same rings,
// half the CTAs (a third for the E4M3 8-head tile, whose registers allow it),
// so about as many warps share an SM.
__host__ __device__ constexpr int stages_for(int D, int hpt, bool f8, int nw) {
  return f8 ? (D == 256 || (D == 128 && hpt <= 16) ? 2 : 3) : (D == 64 || (D == 128 && hpt == 32) ? 3 : 2);
}
__host__ __device__ constexpr int ctas_per_sm4(int D, int hpt, bool f8) {
  return f8 && D == 128 ? (hpt == 8 ? 5 : 4)
                        : D == 64 ? (hpt == 32 ? 3 : 4) : D == 128 ? (hpt == 32 ? 4 : hpt == 8 ? 5 : 3)
                        : (hpt == 16 ? 2 : 3);
}
__host__ __device__ constexpr int ctas_per_sm_for(int D, int hpt, bool f8, int nw) {
  return nw == 4 ? ctas_per_sm4(D, hpt, f8)
                 : (f8 && D == 128 && hpt == 8 ? 3 : (ctas_per_sm4(D, hpt, f8) + 1) / 2);
}
// Bytes of one K (or V) half-stage: bf16 rows of 2D bytes; E4M3 rows of D
// bytes, in boxes padded to at least 128 bytes (only D = 64 with one-row boxes
// needs it).
__host__ __device__ constexpr int half_stage_bytes(int D, int hpt, bool f8, int nw) {
  return stage_tokens_for(D, hpt, f8, nw) * (f8 ? (D < 128 ? 128 : D) : 2 * D);
}

// The same, for the warps each instantiation is built with.
__host__ __device__ constexpr int stage_tokens_for(int D, int hpt, bool f8 = false) {
  return stage_tokens_for(D, hpt, f8, warps_for(D, hpt, f8));
}
__host__ __device__ constexpr int stages_for(int D, int hpt, bool f8 = false) {
  return stages_for(D, hpt, f8, warps_for(D, hpt, f8));
}
__host__ __device__ constexpr int ctas_per_sm_for(int D, int hpt, bool f8 = false) {
  return ctas_per_sm_for(D, hpt, f8, warps_for(D, hpt, f8));
}

// Resident CTAs per SM a launch is built for (the kernel's launch bound).
// The 8-head tiles at D = 128 have a second, denser build at six CTAs per SM
// (80 registers instead of 88 for E4M3 and 93 for bf16).  On B200 the E4M3
// one measured 2.5-3.5% faster on launches of at least four full waves at five
// CTAs per SM and 4-13% slower on shorter ones (GQA batches of 1024-16384
// units: there the CTAs' own start and finish latency weighs more than the
// extra resident warps), so the host picks it by the unit count.
__host__ __device__ constexpr bool has_dense_build(int D, int hpt, bool f8) { return D == 128 && hpt == 8; }
constexpr int kDenseCtasPerSm = 6;
constexpr int kDenseMinWaves = 4;
inline int ctas_per_sm_choice(int D, int hpt, bool f8, int64_t units, int sms) {
  const int base = ctas_per_sm_for(D, hpt, f8);
  return has_dense_build(D, hpt, f8) && units >= (int64_t)kDenseMinWaves * base * sms ? kDenseCtasPerSm : base;
}

// Shared memory of one CTA (from a 1024-byte aligned base): the K/V ring,
// reused after the last stage for the token groups' merge (O^T, m, l) and then
// for the split merge's weight table; then one mbarrier per stage and two flag
// words.
struct SmemPlan {
  int stages, stage_tokens;
  size_t stage_bytes, ring_bytes, warp_merge_bytes, split_merge_bytes, region_bytes, total;
};

__host__ __device__ constexpr SmemPlan smem_plan_for(int D, int hpt, bool f8, int nw) {
  SmemPlan s{};
  s.stages = stages_for(D, hpt, f8, nw);
  s.stage_tokens = stage_tokens_for(D, hpt, f8, nw);
  s.stage_bytes = (size_t)half_stage_bytes(D, hpt, f8, nw) * 2;  // K and V rows of one stage
  s.ring_bytes = (size_t)s.stages * s.stage_bytes;
  s.warp_merge_bytes = (size_t)token_groups_for(D, hpt, f8, nw) * hpt * (D + 4 + 2) * 4;  // padded rows, m, l
  s.split_merge_bytes = (size_t)hpt * (kMaxSplits + 1) * 4;
  size_t m = s.ring_bytes;
  if (s.warp_merge_bytes > m) m = s.warp_merge_bytes;
  if (s.split_merge_bytes > m) m = s.split_merge_bytes;
  s.region_bytes = align_up(m, 128);
  s.total = 1024 /* alignment slack */ + s.region_bytes + 128 /* barriers, flags */;
  return s;
}

// Largest query-head tile whose fp32 O^T accumulator (D x heads) fits one warp's registers.
inline int max_heads_per_tile(int D) { return D <= 128 ? 32 : 16; }

// What a launch records from inside the kernel (pad_last_launch).
struct LaunchWitness {
  int32_t kernel, head_dim, heads_per_tile, kv_dtype, stages, stage_tokens, num_splits, partition_tokens, ctas, warps,
      ctas_per_sm;
};

struct PartitionParams {
  // K and V caches as 5-D tiled tensors (128 bytes of head_dim, slot, the
  // rest of head_dim in 128-byte blocks, kv head, block), one box = one page
  // (or a stage's worth of a larger page; 8 rows for the tcgen05 kernel) with
  // the 128-byte swizzle.  An E4M3 cache at D = 64 has one 64-byte block and
  // the 64-byte swizzle.
  CUtensorMap tmk, tmv;
  // q as a 4-D tiled tensor (64 head_dim elements, head, head_dim / 64, b), one
  // box = a 32-head tile (tcgen05 kernel only).
  CUtensorMap tmq;
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
  int32_t S;        // partitions per sequence (ceil(capacity / P) <= kMaxSplits)
  uint32_t n_units; // B * Hkv * HT * S, one CTA each
  float scale_log2; // scale * k_scale * log2(e)
  float v_scale;    // E4M3 V dequantisation scale (1 for bf16)
  int32_t window;     // 0: every token; W > 0: each sequence's last W tokens
  const float *sinks; // null, or a sink logit per query head [Hq] (natural log, units of scale q.k)
  uint16_t *out;
  int64_t o_sb, o_sh;
  float *lse;  // may be null
  int64_t lse_sb, lse_sh;
  float *o_part;       // [B, Hq, S, D] fp32
  float *lse_part;     // [B, Hq, S] fp32 (natural log)
  // The launch's unit order, longest first (written by schedule_kernel just
  // before the launch): CTA i runs unit order[i].  Null: CTA i runs unit i.
  uint32_t *order;
  uint32_t *counters;  // [B * Hkv * HT] partitions finished per (b, kv head, head tile)
  uint32_t *err;
  LaunchWitness *witness;  // written by block 0 of every launch
  // Failure-path test hook (pad_inject_stage_timeout): -1 normally; otherwise
  // the partition kernel's non-empty units of partition `stall_partition` wait,
  // where they would count themselves for the merge, on a barrier nothing
  // arrives on, give up after a short bounded wait (error bit 0x4) and return
  // uncounted.
  int32_t stall_partition;
};

// Whether a launch orders its units longest first: with several partitions per
// sequence (only then do units differ in length), when its (sequence,
// partition) pairs fit the one-CTA scheduling pass, and when a unit is heavy --
// P tokens x heads per tile of at least 32 K (a 2048-token partition of a
// 32-head tile; an 8-head tile from 4096 tokens).  Measured on B200: the
// ragged MQA batch (2048 x 32) gains 17% (162 -> 134 us; E4M3 167 -> 146 us),
// because its full units no longer wait behind a first wave for the end of
// the launch; light units of near-equal length lose (llama8b, 512 x 8: 57 ->
// 66 us) -- the pass and the order load cost a few us, and equal units
// dispatched together start and finish in lock-step, so their start and end
// phases stop overlapping other units' streaming.
constexpr int64_t kScheduleMaxPairs = 65536;
constexpr int64_t kScheduleMinUnitWork = 32768;
inline bool schedules_units(int64_t B, int64_t S, int64_t P, int64_t heads_per_tile) {
  return S > 1 && B * S <= kScheduleMaxPairs && P * heads_per_tile >= kScheduleMinUnitWork;
}

// Partials layout inside a workspace buffer (offsets 256-byte aligned), then
// the unit order (4 bytes per unit) when the launch schedules its units; empty
// when S == 1.
struct WorkspaceLayout {
  size_t o_part, lse_part, order, total;
};

inline WorkspaceLayout workspace_layout(int64_t B, int64_t Hq, int64_t S, int64_t D, int64_t units, bool ordered) {
  WorkspaceLayout w{};
  if (S <= 1) return w;
  w.o_part = 0;
  w.lse_part = align_up((size_t)(B * Hq * S * D * 4), 256);
  w.order = w.lse_part + align_up((size_t)(B * Hq * S * 4), 256);
  w.total = w.order + (ordered ? align_up((size_t)units * 4, 256) : 0);
  return w;
}

// Control block: one merge counter per (b, kv head, head tile), present only
// when S > 1.  Must be zero when a launch starts; a launch that completes
// leaves it zero (the CTA that merges a set resets its counter).
struct ControlLayout {
  size_t counters, total;
};

inline ControlLayout control_layout(int64_t B, int64_t Hkv, int64_t HT, int64_t S) {
  ControlLayout c{};
  c.counters = 0;
  c.total = S > 1 ? align_up((size_t)(B * Hkv * HT * 4), 256) : 0;
  return c;
}

// Launches the partition kernel instance for (D, heads_per_tile, cache type)
// built for `ctas_per_sm` resident CTAs per SM (ctas_per_sm_choice); an
// instance that does not exist is cudaErrorInvalidValue.
cudaError_t launch_partition(const PartitionParams &p, int D, int heads_per_tile, bool kv_fp8, int grid,
                             int ctas_per_sm, cudaStream_t s);
// The tcgen05 kernel (pad_umma.cu) takes 32-head tiles at head_dim 128 with
// pages of at least 8 tokens (its K/V boxes are 8 rows of one page).
inline bool umma_eligible(int D, int hpt, int block_size) { return D == 128 && hpt == 32 && block_size >= 8; }
cudaError_t launch_umma(const PartitionParams &p, int grid, cudaStream_t s);
int umma_stages();
constexpr int kUmmaStageTokens = 128;
constexpr int kUmmaWarps = 6;
constexpr int kUmmaCtasPerSm = 2;

// Rows of one TMA box: a page, or a stage's worth of rows of a larger page.
inline int box_rows(int block_size, int D, int hpt, bool f8) {
  const int st = stage_tokens_for(D, hpt, f8, warps_for(D, hpt, f8));
  return block_size < st ? block_size : st;
}
int partition_stages(int D, int heads_per_tile, bool kv_fp8);
// One-CTA pass that writes p.order (units longest first) on `s`; the decode
// launch that follows on the same stream reads it.
cudaError_t launch_schedule(const PartitionParams &p, cudaStream_t s);
cudaError_t device_error_word(int device, uint32_t **ptr);
cudaError_t device_witness(int device, LaunchWitness **ptr);
void set_last_error(const char *msg);

// pad_decode with its scratch in a fixed array of `scratch_bytes` bytes:
// validates and plans exactly as pad_decode, then rejects a shape whose control
// block and partials exceed the array (PAD_ERR_WORKSPACE), asks
// `scratch_address` for the array's device address (on every call that gets
// this far, so the first one does any set-up), clears the control block on
// `stream` and launches.  Used by the allocation-free entry point; allocates
// nothing itself.
pad_status decode_with_scratch_array(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                                     const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                                     int32_t num_splits, pad_tensor *out, pad_tensor *lse,
                                     pad_status (*scratch_address)(void **), size_t scratch_bytes,
                                     cudaStream_t stream);

}  // namespace pad
