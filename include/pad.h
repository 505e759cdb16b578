/*
 * pad.h -- C ABI of the paged-KV single-token decode attention library (libpad).
 *
 * The operation: for every sequence b of a decode batch, one query token per
 * query head attends over the L_b tokens of that sequence held in a paged KV
 * cache, the pages being named by the sequence's row of a block table.  This is
 * the problem of "spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm, the ROCm
 * half of #382" (vllm.cpp PR #564, section "The gap it specs": bf16 paged decode
 * attention for head_dim 128 GQA models, one K/V read serving a GQA group) and of
 * "perf(rocke): prepare saved paged decode bindings once" (rocm-libraries PR
 * #13700, section "Summary": one-token split-KV attention with an optional
 * log-sum-exp output; section "Runnable saved-binding HIP-event comparison":
 * batch, heads, kv-heads, head-dim, seqlen-q = 1, seqlen-k, kv-block-size).
 *
 * Math (natural log; `scale` multiplies q.k before the softmax):
 *   kh = h / (Hq / Hkv)                      consecutive query heads share a KV head
 *   token t < L_b sits in block block_tables[b][t / bs], slot t % bs
 *   s_t = scale * <q[b,h,:], K[block, kh, slot, :]>
 *   out[b,h,:] = sum_t softmax(s)_t * V[block, kh, slot, :]     (bf16, RNE once)
 *   lse[b,h]   = log(sum_t exp(s_t))                             (fp32)
 *   L_b = 0 gives out = 0 and lse = -inf.
 *
 * How it runs on the device: each sequence's tokens are cut into partitions of P
 * tokens (P a multiple of bs).  One kernel launch runs a CTA per (sequence, KV
 * head, head tile, partition) unit; each streams its partition's K/V pages for
 * one KV head through shared memory once, serves all query heads of the GQA
 * group from that read, and keeps a running max/sum (online softmax) in fp32.
 * When a sequence has more than one non-empty partition, the unit that finishes
 * last merges the partial outputs weighted by their log-sum-exp (the split
 * reduce, folded into the same launch).  When units are heavy (partition tokens
 * x heads per tile >= 32768), a one-CTA pass on the same stream first orders
 * the launch's units longest first from the device-resident lengths, so the
 * units the GPU dispatches last are the short ones (no host synchronisation).
 *
 * Conventions for every entry point:
 *  - All tensor data pointers are DEVICE pointers owned by the caller.  The
 *    library never frees them and keeps no reference after the call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Outputs are valid once the stream has completed the work; inputs
 *    must stay alive and unmodified until then.
 *  - On any validation failure the call returns before launching anything and
 *    writes nothing: `out` and `lse` are left untouched.
 *  - Device-resident data that cannot be checked without a synchronisation
 *    (block ids, seq_lens) must be valid: 0 <= block id < num_blocks for every
 *    live page, 0 <= seq_lens[b] <= max_blocks_per_seq * block_size.  The kernels
 *    check both anyway; a violation is never dereferenced (the page is skipped,
 *    the length clamped), and sets a sticky per-device error word reported by
 *    pad_check_device_errors().
 */
#ifndef PAD_H
#define PAD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PAD_ABI_VERSION 3

typedef enum pad_status {
  PAD_OK = 0,
  PAD_ERR_INVALID_ARG = 1,  /* bad dtype, shape, stride, alignment or scalar */
  PAD_ERR_UNSUPPORTED = 2,  /* valid problem outside the compiled envelope */
  PAD_ERR_WORKSPACE = 3,    /* split scratch could not be obtained (e.g. growth under capture) */
  PAD_ERR_CUDA = 4,         /* a CUDA runtime call failed; see pad_last_error() */
  PAD_ERR_DEVICE_CHECK = 5  /* a kernel saw an invalid block id or sequence length, or a
                               bounded wait gave up (pad_check_device_errors) */
} pad_status;

/* PAD_FP8_E4M3: OCP 8-bit floating point, E4M3 variant (sign, 4 exponent bits
 * with bias 7, 3 mantissa bits, subnormals, no infinities, S.1111.111 = NaN,
 * largest finite 448) -- torch.float8_e4m3fn.  Accepted for k_cache/v_cache. */
typedef enum pad_dtype { PAD_BF16 = 0, PAD_F32 = 1, PAD_I32 = 2, PAD_FP8_E4M3 = 3 } pad_dtype;

/* A strided tensor view.  `stride` is in ELEMENTS.  Unused trailing dims are
 * ignored.  `dtype` holds a pad_dtype value. */
typedef struct pad_tensor {
  void *data;
  int32_t dtype;
  int32_t ndim;
  int64_t shape[4];
  int64_t stride[4];
} pad_tensor;

/* Launch plan chosen for one problem shape. */
typedef struct pad_plan {
  int32_t num_splits;        /* effective number of partitions per sequence (S) */
  int32_t partition_tokens;  /* P, tokens per partition, a multiple of block_size */
  int32_t heads_per_tile;    /* query heads per work unit, padded (8, 16 or 32) */
  int32_t head_tiles;        /* work units per (sequence, KV head, partition): ceil(group / heads_per_tile) */
  int32_t warps_per_cta;     /* warps per CTA: 4 or 8 (mma.sync kernel, chosen per head_dim, heads
                                per tile and cache type), 6 (tcgen05 kernel: 4 softmax,
                                producer, MMA) */
  int32_t stage_tokens;      /* tokens per shared-memory pipeline stage */
  int32_t stages;            /* pipeline depth */
  int32_t ctas;              /* CTAs launched: one per unit (B * Hkv * head_tiles * num_splits) */
  int32_t ctas_per_sm;       /* resident CTAs per SM the launched kernel instance is built for
                                (its launch bound): fixed per head_dim, heads per tile and
                                cache type, except the 8-head tiles at D = 128, which
                                take their six-per-SM build for launches of at least four
                                full waves at five per SM (2 for the tcgen05 kernel) */
  int32_t reduce;            /* 1 when partitions may need merging (S > 1) */
  int64_t workspace_bytes;   /* partial-output scratch (0 when S == 1) */
  int64_t control_bytes;     /* merge counters, 0 when S == 1 (library-owned except
                                for pad_decode_static_scratch) */
} pad_plan;

/*
 * pad_decode -- paged single-token decode attention: the operation of
 * "spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm, the ROCm half of #382"
 * (section "The gap it specs") computed as the one-token split-KV attention of
 * "perf(rocke): prepare saved paged decode bindings once" (section "Summary"),
 * with the optional log-sum-exp output.
 *
 *  q             bf16 [B, Hq, D], stride[2] == 1, every row 16-byte aligned.
 *  k_cache       bf16 or FP8 E4M3 [num_blocks, Hkv, block_size, D], stride[3] ==
 *                1; dims 0-2 may have any non-negative strides whose byte size
 *                is a multiple of 16 (so both [blocks, Hkv, bs, D] "HND" and a
 *                permuted view of a [blocks, bs, Hkv, D] "NHD" cache are
 *                accepted).  Base 16-byte aligned.  An E4M3 cache holds codes
 *                dequantised as k_scale * code (pad_decode_options; 1 here).
 *  v_cache       same dtype and shape as k_cache, its own strides, same rules;
 *                E4M3 codes are dequantised as v_scale * code.
 *  block_tables  int32 [B, max_blocks_per_seq], stride[1] == 1.  Entries past
 *                ceil(L_b / block_size) may hold anything: their values are never
 *                used (the kernel may read them, within the row, before it knows
 *                L_b).
 *  seq_lens      int32 [B], contiguous.
 *  scale         finite; multiplies q.k before the softmax (commonly 1/sqrt(D)).
 *  num_splits    0 = let the library choose; S >= 1 asks for partitions of
 *                P = round_up(ceil(C / S), block_size) tokens, C =
 *                max_blocks_per_seq * block_size (the effective S = ceil(C / P) is
 *                reported by pad_decode_plan; at most 256).  With S == 1 no
 *                partial is ever written.
 *  out           bf16 [B, Hq, D], stride[2] == 1, rows 16-byte aligned.  Must not
 *                overlap any input.
 *  lse           NULL = no log-sum-exp output (nothing else is written); else
 *                fp32 [B, Hq], any strides.  A non-NULL lse whose shape is wrong
 *                is an error, never silently dropped.
 *  stream        cudaStream_t.
 *
 * Supported envelope: D in {64, 128, 256}; Hq / Hkv <= 256; block_size a power of
 * two in [1, 256]; B < 2^31, Hq <= 65536 and B * Hq <= 2^31; a table capacity C of
 * at most 2^30 tokens; at most 2^31 - 1 work units (B * Hkv * head tiles * S) per
 * launch.  Outside it: PAD_ERR_UNSUPPORTED, nothing launched.  Scratch (partials, and a control block of merge counters
 * that every launch leaves zero) is owned by the library, kept per (device,
 * stream) and grown on demand; growing it while `stream` is being captured into
 * a CUDA graph returns PAD_ERR_WORKSPACE (call once outside capture first).
 * Threads: any number of host threads may call at once on different streams
 * (each (device, stream) has its own scratch); calls on the same stream must be
 * serialised by the caller, as their launches would be unordered anyway (a call
 * may regrow that stream's scratch).
 */
pad_status pad_decode(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                      const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                      int32_t num_splits, pad_tensor *out, pad_tensor *lse, void *stream);

/*
 * Options of pad_decode_ex: two attention types that "Attention parity: run
 * every attention type on the best available path on both targets" (section
 * "Current state") lists next to dense GQA.
 *   window_left  0: every token; W > 0: each sequence attends to its last W
 *                tokens only (tokens L_b - W .. L_b - 1; all of them when
 *                W >= L_b).  Partitions and pages wholly before the window
 *                are never read.
 *   sinks        NULL, or a pad_tensor of fp32 [Hq] on the device: the sink
 *                logit of each query head, in the units of scale * q.k.  It
 *                joins the softmax with a zero value row:
 *                  M = max(max_t s_t, sink_h), Z = sum_t exp(s_t - M) +
 *                  exp(sink_h - M), out = sum_t exp(s_t - M) v_t / Z,
 *                  lse = M + ln Z;  L_b = 0 gives out = 0, lse = sink_h.
 *   k_scale,     dequantisation scales of an E4M3 cache (the FP8 decode path
 *   v_scale      "perf(rocke): prepare saved paged decode bindings once" names
 *                beside the non-FP8 one, section "Summary"; one scale per
 *                tensor is the reading taken): k_t = k_scale * code, v_t =
 *                v_scale * code.  0 reads as 1; otherwise finite and > 0.  With a
 *                bf16 cache both must be 0 or 1.
 * Zero-initialised options are pad_decode exactly.
 */
typedef struct pad_decode_options {
  int32_t window_left;
  const pad_tensor *sinks;
  float k_scale;
  float v_scale;
} pad_decode_options;

/*
 * pad_decode_ex -- pad_decode with options (NULL options = pad_decode): the
 * attention types "Attention parity: run every attention type on the best
 * available path on both targets" (section "Current state") lists next to
 * dense GQA, and the FP8 cache of "perf(rocke): prepare saved paged decode
 * bindings once" (section "Summary").  Same
 * arguments, scratch, results and errors; `options->window_left` < 0, a sinks
 * tensor that is not fp32 [Hq] device memory, or a scale that is negative,
 * non-finite, or other than 0/1 for a bf16 cache, is PAD_ERR_INVALID_ARG.
 */
pad_status pad_decode_ex(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                         const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                         int32_t num_splits, const pad_decode_options *options, pad_tensor *out,
                         pad_tensor *lse, void *stream);

/*
 * pad_decode_with_workspace -- pad_decode with its scratch supplied by the
 * caller instead of the library ("perf(rocke): prepare saved paged decode
 * bindings once", section "Technical Changes": a binding owns its private
 * scratch, kept alive until the work queued on it completes).
 *
 * Arguments are those of pad_decode plus `workspace`: DEVICE memory owned by the
 * caller, 256-byte aligned, of at least pad_decode_plan(...).workspace_bytes
 * bytes (may be NULL when that is 0, i.e. S == 1); its initial contents do not
 * matter.  It must not be shared by calls that may run concurrently.  Layout
 * (offsets rounded up to 256 bytes): fp32 partial outputs [B, Hq, S, D], each
 * normalised by its own softmax sum, then fp32 partial LSEs [B, Hq, S], then --
 * when the launch orders its units longest first (a unit is heavy: partition
 * tokens x heads per tile >= 32768, with B * S <= 65536) -- the unit order,
 * one uint32 per CTA, written on the stream by a one-CTA pass just before the
 * decode launch.  After
 * a call, the partials of every (b, head) whose sequence had more than one
 * non-empty partition are left in place; partitions past ceil(L_b / P) are
 * neither written nor read.  The small control block (merge counters,
 * control_bytes) stays library-owned per (device, stream), as for pad_decode:
 * allocated zeroed on first use and kept zero by every launch.
 */
pad_status pad_decode_with_workspace(const pad_tensor *q, const pad_tensor *k_cache,
                                     const pad_tensor *v_cache, const pad_tensor *block_tables,
                                     const pad_tensor *seq_lens, float scale, int32_t num_splits,
                                     pad_tensor *out, pad_tensor *lse, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * pad_decode_with_workspace_ex -- pad_decode_with_workspace with the options of
 * pad_decode_ex (window, sinks, E4M3 scales; NULL = none): caller-owned scratch
 * ("perf(rocke): prepare saved paged decode bindings once", section "Technical
 * Changes") for every attention type of pad_decode_ex.  Same arguments,
 * scratch rules, results and errors as those two.
 */
pad_status pad_decode_with_workspace_ex(const pad_tensor *q, const pad_tensor *k_cache,
                                        const pad_tensor *v_cache, const pad_tensor *block_tables,
                                        const pad_tensor *seq_lens, float scale, int32_t num_splits,
                                        const pad_decode_options *options, pad_tensor *out,
                                        pad_tensor *lse, void *workspace, size_t workspace_bytes,
                                        void *stream);

/*
 * pad_decode_static_scratch -- pad_decode for callers that cannot allocate device
 * memory.  The source pages have no counterpart of this entry point.
 *
 * Some callers must not call cudaMalloc (or anything that allocates) when they
 * decode: a runtime that plans all of its memory up front, a thread that may not
 * take the allocator's locks or absorb the synchronisation an allocation or a
 * free can cause, an embedding with no allocator to lend.  pad_decode grows
 * scratch on demand and pad_decode_with_workspace wants the caller's scratch;
 * this call uses neither.  Its split scratch is a fixed 32 MiB array
 * compiled into the library, which every GPU that loads the library holds until
 * the process exits.
 *
 * Arguments, results and validation are those of pad_decode, checked in the
 * same order with the same statuses.  It calls no allocating routine.  A valid
 * shape whose split scratch (pad_decode_plan(...).control_bytes +
 * .workspace_bytes) exceeds 32 MiB is then rejected with PAD_ERR_WORKSPACE
 * before anything is launched.
 *
 * Every call with a non-empty batch that passes validation looks up the
 * array's device address (cudaGetSymbolAddress, with the call's device current;
 * kept per device after the first), whether or not that call splits.  Under
 * CUDA's lazy module loading (the default since CUDA 12.2) that first lookup
 * loads the library module holding the array, which is when the 32 MiB are
 * reserved on the device: make the first call on each device before any stream
 * capture.  All calls on a device share the one array and it keeps the last
 * call's contents; each call clears, on `stream` after validating its
 * arguments and before its launch (cudaMemsetAsync, which allocates nothing),
 * the counter words that must start at zero.  Calls that may
 * overlap on the GPU -- on different streams without ordering between them, or
 * from different host threads -- race on the array and corrupt each other's
 * results: serialise them.
 */
pad_status pad_decode_static_scratch(const pad_tensor *q, const pad_tensor *k_cache,
                                     const pad_tensor *v_cache, const pad_tensor *block_tables,
                                     const pad_tensor *seq_lens, float scale, int32_t num_splits,
                                     pad_tensor *out, pad_tensor *lse, void *stream);

/*
 * pad_decode_tcgen05 -- pad_decode computed by the 5th-generation tensor-core
 * kernel: S^T = K.Q^T and O^T += V^T.P^T as tcgen05.mma with the accumulators in
 * tensor memory, K/V/q streamed by TMA in 8-token boxes, the softmax in four warps
 * that own one token (one TMEM lane) each, one CTA per (sequence, KV head,
 * partition) unit, two per SM -- the GQA-group fusion over one K/V read of
 * "spec(BACKEND-ROCM): the ROCm head_dim=128 decode arm, the ROCm half of #382"
 * (section "The gap it specs") on tensor memory.  Same arguments, results,
 * scratch and errors as pad_decode.  It takes a bf16 cache with groups of 17..32 query
 * heads per KV head at head_dim 128 and block_size >= 8, and returns
 * PAD_ERR_UNSUPPORTED otherwise.
 * pad_decode does not call it: on the workloads measured on B200 the mma.sync
 * kernel behind pad_decode is faster (ragged MQA batch: 132 against 162 us; a
 * 128-token chunk of K and V is 64 KB of shared memory, so two CTAs with one
 * chunk buffer each are all an SM holds, and each chunk waits for its own
 * copies).  Like pad_decode it orders heavy units longest first.
 */
pad_status pad_decode_tcgen05(const pad_tensor *q, const pad_tensor *k_cache, const pad_tensor *v_cache,
                              const pad_tensor *block_tables, const pad_tensor *seq_lens, float scale,
                              int32_t num_splits, pad_tensor *out, pad_tensor *lse, void *stream);

/*
 * pad_decode_plan -- the launch geometry pad_decode would use for this shape
 * (the per-shape heuristic when num_splits == 0): the geometry a saved binding
 * of "perf(rocke): prepare saved paged decode bindings once" prepares once and
 * reuses for compatible calls (section "Summary").  Pure host computation; no
 * launch.  `device` < 0 means the current device (its SM count feeds the
 * heuristic: a small batch gets shorter partitions, down to 64 tokens, so that
 * it still fills the GPU).  Returns PAD_ERR_INVALID_ARG / PAD_ERR_UNSUPPORTED exactly when
 * pad_decode would for the same shape.
 */
pad_status pad_decode_plan(int64_t batch, int64_t num_q_heads, int64_t num_kv_heads,
                           int64_t head_dim, int64_t block_size, int64_t max_blocks_per_seq,
                           int32_t num_splits, int32_t device, pad_plan *plan);

/*
 * pad_decode_plan_ex -- pad_decode_plan for a cache of dtype `kv_dtype`
 * (PAD_BF16, as pad_decode_plan, or PAD_FP8_E4M3: the same partitions and
 * scratch, deeper pipeline stages of half the bytes) -- the non-FP8 and FP8
 * decode paths of "perf(rocke): prepare saved paged decode bindings once"
 * (section "Summary").  Any other kv_dtype is
 * PAD_ERR_INVALID_ARG.
 */
pad_status pad_decode_plan_ex(int64_t batch, int64_t num_q_heads, int64_t num_kv_heads,
                              int64_t head_dim, int64_t block_size, int64_t max_blocks_per_seq,
                              int32_t num_splits, int32_t kv_dtype, int32_t device, pad_plan *plan);

/*
 * pad_launch_witness / pad_last_launch -- what the most recent decode launch
 * on the current device recorded from inside the kernel (thread 0 of block 0:
 * the partition kernel when its unit is done, the tcgen05 kernel at its
 * start): which kernel ran and the plan it was compiled and launched with.  A
 * launch whose block 0 gave up on an internal error (pad_check_device_errors
 * reports it) leaves the previous record.  A test compares it with pad_decode_plan[_ex] to show that the planned
 * kernel is the one that executed: kernel-resident witnesses of which arm ran
 * ("perf(BACKEND-ROCM): cooperate across Q8_K activation blocks", section
 * "What changed"), because selection can land silently on another path
 * ("Attention parity: run every attention type on the best available path on
 * both targets", opening summary).  pad_last_launch synchronises the device;
 * concurrent launches on several streams leave the record of whichever wrote
 * last.
 */
typedef struct pad_launch_witness {
  int32_t kernel;            /* 1: partition kernel (mma.sync), 2: tcgen05 kernel; 0: none yet */
  int32_t head_dim;          /* D the kernel was compiled for */
  int32_t heads_per_tile;    /* query heads per unit it was compiled for */
  int32_t kv_dtype;          /* pad_dtype of the cache it was compiled for */
  int32_t stages;            /* pipeline stages it was compiled with */
  int32_t stage_tokens;      /* tokens per stage (chunk) */
  int32_t num_splits;        /* S it was launched with */
  int32_t partition_tokens;  /* P it was launched with */
  int32_t ctas;              /* grid size */
  int32_t warps;             /* warps per CTA it was compiled for */
  int32_t ctas_per_sm;       /* resident CTAs per SM it was compiled for (its launch bound) */
} pad_launch_witness;

pad_status pad_last_launch(pad_launch_witness *witness);

/*
 * pad_status_string -- static name of a status code.  Every failure is reported
 * as a status with a message, never dropped: "perf(rocke): prepare saved paged
 * decode bindings once", review item N1 (an argument the call cannot honour
 * raises instead of being silently ignored).
 */
const char *pad_status_string(pad_status status);

/*
 * pad_last_error -- message for the last failure on the calling thread ("" if
 * none); the message half of the same rule ("perf(rocke): prepare saved paged
 * decode bindings once", review item N1).
 */
const char *pad_last_error(void);

/*
 * pad_check_device_errors -- synchronises `stream`, then reads and clears the
 * current device's sticky error word: the guards that "feat(rocm): wvSplitK
 * skinny GEMM for decode M<=4" (opening review, findings 1 and 3) asks of
 * every device access, reported instead of silently producing wrong numbers.
 * Returns PAD_ERR_DEVICE_CHECK if any kernel since the last check set a bit;
 * the bits are stored in *bits when bits != NULL:
 *   0x1  a live table entry outside [0, num_blocks) (the page read as zeros),
 *   0x2  a sequence length < 0 or > the table capacity (clamped),
 *   0x4  a bounded wait gave up: a stage's copies did not land within its
 *        limit (1 s; internal error) or pad_inject_stage_timeout stalled the
 *        launch.  The CTA that gave up waited (bounded) for its own copies and
 *        returned without writing its outputs; the merge counters it left set
 *        in the library-owned control blocks of this device are re-zeroed by
 *        this call, so the next call is correct.  That launch's out and lse
 *        are not valid.
 */
pad_status pad_check_device_errors(void *stream, uint32_t *bits);

/*
 * pad_inject_stage_timeout -- failure-path test hook ("perf(rocke): prepare
 * saved paged decode bindings once", section "Risk Assessment": focused tests
 * of failure recovery).  The next launch of the partition kernel made from the
 * calling thread (pad_decode, pad_decode_ex, the workspace and static-scratch
 * entry points; not pad_decode_tcgen05) runs with every non-empty unit of
 * partition `partition` giving up where it would count its partition for the
 * merge: it waits on a barrier that nothing arrives on, the wait gives up after
 * a short limit (about 20 us) and sets bit 0x4 of the device error word, as a
 * stage that never lands would, and the unit returns uncounted.  The other
 * partitions count themselves and leave their merge counters set, so no
 * sequence with several partitions including that one is merged (its out and
 * lse are left as they were); a sequence with one partition has already
 * written its result.  No GPU fault, trap or hang is involved.  One-shot: the
 * launch consumes it.  -1 disarms it; other values outside [0, 256) are
 * PAD_ERR_INVALID_ARG.
 */
pad_status pad_inject_stage_timeout(int32_t partition);

/*
 * pad_release_workspace -- frees the split scratch held for `device` (< 0: all
 * devices) after synchronising that device: the scratch a binding owns and
 * keeps until its queued work completes ("perf(rocke): prepare saved paged
 * decode bindings once", section "Technical Changes").  Safe to call at any
 * time outside stream capture; later calls re-grow scratch on demand.
 */
pad_status pad_release_workspace(int32_t device);

/* pad_abi_version -- PAD_ABI_VERSION of the loaded library.  The source pages
 * have no counterpart. */
int32_t pad_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAD_H */
