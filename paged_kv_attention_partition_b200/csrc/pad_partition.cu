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
// One thread streams the partition's K and V pages for one KV head from HBM
// into a small shared-memory ring with TMA: one tiled box per page (or per
// stage's worth of rows of a larger page) for K and one for V, completing on the
// stage's mbarrier.  The box is (64 head_dim elements, its rows, head_dim / 64)
// with the 128-byte swizzle, so the tensor-core operand loads below are bank
// conflict free; an out-of-range block id reads as zeros.  Every query head of
// the GQA group is served from that one K/V read ("spec(BACKEND-ROCM): the ROCm
// head_dim=128 decode arm", section "It is a mirror of merged work, not new
// design": PagedAttnDecodeGqaBf16 fuses a GQA group over one K/V read).  Pages
// are whole, so the last page's slots past L_b arrive too: their scores are
// masked and their V rows zeroed before use.
//
// With 8 heads per tile the warps form token groups: group tg computes 16-token
// tiles tg, tg + 4, ... of every stage and keeps its own running max and sum
// per head (the warp-strided online softmax of the same section; the groups
// are merged at the end, so the sum is taken in another order than a
// sequential kernel's).  With 16 or 32 heads per tile the warps are head
// groups instead: each owns one 8-head n-tile and computes every token of the
// stage for it.  At head_dim 256 two warps compute the same scores and each
// keep half of the head_dim rows of O^T, which halves the stage and the
// accumulator.
// Per 16-token tile and 8-head n-tile:
//   S^T = K . Q^T                 (mma.m16n8k16 bf16, fp32 accumulate)
//   P^T = exp2(S^T * scale*log2e - m)
//   O^T += V^T . P^T              (P^T moved into the B-operand layout by movmatrix)
//
// An E4M3 cache ("perf(rocke): prepare saved paged decode bindings once",
// section "Summary": the FP8 decode path beside the non-FP8 one) streams 8-bit
// codes, half the bytes, through the same stages.  K operands are loaded four
// codes per register and widened exactly to f16 (one cvt per pair: every E4M3
// value is an f16 value); q enters the f16 QK product scaled by a power of two
// per head tile so that its bf16 values stay exact.  The head_dim order inside
// each 16-wide k-step is permuted (codes 4c..4c+3 of a row go to k = 2c, 2c+1,
// 2c+8, 2c+9), and the q fragments take the same permutation, which a dot
// product allows.  V operands come from a transposed ldmatrix of the codes and
// a byte permute, widened to f16 (exact) for an f16 PV product with f16
// weights; the m-tile rows are head_dim 2i and 2i+1 instead of i and i+8.
// k_scale is folded into the score scale, v_scale into the final 1/l.
//
// A sequence with one non-empty partition writes bf16 out (+ lse) directly.
// Otherwise each partition writes its fp32 output (normalised by its own sum)
// and its lse, and the CTA that finishes the last partition of the (b, KV head,
// head tile) merges them by log-sum-exp while they are in L2:
//   M = max_s lse_s,  w_s = exp(lse_s - M) / sum_s' exp(lse_s' - M),
//   out = sum_s w_s o_s,  lse = M + log sum_s exp(lse_s - M).
//
// Every mbarrier wait is bounded in time: on expiry the CTA sets an error bit,
// waits (bounded again) for the copies it issued, and returns.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "pad_device.cuh"
#include "pad_internal.h"
#include "pad_merge.cuh"

namespace pad {

__device__ uint32_t g_err_word;
__device__ LaunchWitness g_witness;

namespace {
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kRescaleSlack = 8.f;                  // log2 units: weights stay below 256
constexpr uint64_t kWaitLimitNs = 1000000000ull;      // no stage can legitimately take 1 s
constexpr uint64_t kStallLimitNs = 20000ull;          // the test hook's wait on a barrier nothing arrives on

// Waits for the phase of `bar` with this parity; false (and the timeout bit)
// after `limit_ns`.
__device__ bool wait_stage(uint32_t bar, uint32_t parity, uint32_t *err, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t start = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - start > limit_ns) {
      atomicOr(err, kErrTimeout);
      return false;
    }
  }
  return true;
}

}  // namespace

// At a unit's exits.  (1) Which kernel ran, and with what plan: thread 0 of
// block 0 writes the record when its unit is done (empty, or through the
// epilogue); a unit that gives up on an internal error records nothing -- the
// error word reports that case.  (2) The failure-path test hook, at the exit
// after the unit's result is written (`spare`: an unused 8-byte barrier slot):
// a unit of partition p.stall_partition gives up there instead of counting
// its partition -- its thread 0 waits on a barrier nothing arrives on until the
// short limit runs out, as on a stage whose copies never land (error bit 0x4)
// -- and returns true in every thread.  Out of line, both leave the main
// loop's code as it is: any code added to the kernel body (the record inlined
// at the start or at the exits, or a hook of its own) changed the 32-head
// instances' schedules at their 128-register cap and cost the ragged MQA batch
// 6-10% on B200; as this one call it is within 1% of neither.
template <int D, int HPT, bool F8, int NST, int ST, int CPS>
__device__ __noinline__ bool unit_exit(const PartitionParams &p, int s, uint64_t *spare) {
  if (blockIdx.x == 0 && threadIdx.x == 0)
    *p.witness = LaunchWitness{1, D, HPT, F8 ? (int32_t)PAD_FP8_E4M3 : (int32_t)PAD_BF16, NST, ST, p.S, p.P,
                               (int32_t)gridDim.x, (int32_t)(blockDim.x / 32), CPS};
  if (s != p.stall_partition || spare == nullptr) return false;
  if (threadIdx.x == 0) {
    const uint32_t never = smem_addr(spare);
    mbar_init(never, 1);
    wait_stage(never, 0, p.err, kStallLimitNs);  // gives up: bit 0x4
  }
  return true;
}

template <int D, int HPT, bool F8, int NW, bool ORDERED, int CPS>
__global__ void __launch_bounds__(NW * 32, CPS) partition_kernel(const __grid_constant__ PartitionParams p) {
  constexpr int NTH = NW * 32;             // threads of the CTA
  constexpr SmemPlan SP = smem_plan_for(D, HPT, F8, NW);
  constexpr int NST = SP.stages;
  constexpr uint32_t STAGE_BYTES = (uint32_t)SP.stage_bytes;
  constexpr int ST = SP.stage_tokens;      // tokens per stage
  constexpr int ST_LOG2 = ST == 128 ? 7 : ST == 64 ? 6 : 5;
  constexpr int DS = dsplit_for(D, HPT, F8, NW);       // warps sharing a token group's scores (head_dim split)
  constexpr int HG = head_groups_for(D, HPT, F8, NW);  // warps splitting the tile's n-tiles
  constexpr int TG = token_groups_for(D, HPT, F8, NW);  // token groups
  constexpr int TPW = tiles_per_group(D, HPT, F8, NW);  // 16-token tiles per warp per stage
  constexpr int NT = HPT / 8;              // 8-head n-tiles of the head tile
  constexpr int NTW = NT / HG;             // n-tiles of one warp
  constexpr int KT = D / 16;               // QK k-steps
  constexpr int MT = KT / DS;              // PV m-tiles (16 head_dim rows each) per warp
  constexpr int ROWB = F8 ? D : D * 2;     // bytes per K/V row
  constexpr int RW = ROWB < 128 ? ROWB : 128;  // bytes of a row in one column block
  constexpr int CH = ROWB / 16;            // 16-byte chunks per K/V row
  constexpr int CPB = RW / 16;             // 16-byte chunks per column block
  constexpr int HALF = half_stage_bytes(D, HPT, F8, NW);  // K (or V) rows of one stage
  constexpr int IDW = (ST + 31) / 32;      // block ids per lane of warp 0 for one stage
  // independent QK accumulation chains per tile (four in all where registers allow)
  constexpr int NCH = NTW == 1 ? (TPW >= 4 ? 1 : 4 / TPW) : NTW == 2 && TPW == 1 ? 2 : 1;
  static_assert(KT % NCH == 0, "k-steps split evenly over the chains");
  static_assert(ST == 16 * TG * TPW && (1 << ST_LOG2) == ST, "stage shape");
  static_assert(DS * HG * TG == NW && NTW * HG == NT, "warp roles");
  static_assert(!F8 || (KT % 2 == 0 && MT % 2 == 0), "E4M3 operands are loaded two k-steps / m-tiles at a time");
  static_assert(NST >= 2 && NST <= 8, "at least one stage in flight during the math; barrier area");
  static_assert(SP.total <= (size_t)kSmemBudget, "shared-memory plan over budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + SP.region_bytes);  // one per stage slot
  int *flag = reinterpret_cast<int *>(smem + SP.region_bytes + 64);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int dh = warp % DS, hg = (warp / DS) % HG, tg = warp / (DS * HG);  // head_dim part, head group, token group
  // Unit order.  With several partitions per sequence, CTA i runs unit
  // p.order[i], written just before the launch by schedule_kernel from the
  // device-resident lengths: the longest units first, so the units dispatched
  // last (after the first wave) are the shortest.  Otherwise, and as the unit
  // numbering: partition index descending, outermost -- the highest partitions
  // exist only for the longest sequences, so their work starts first and the
  // empty ones (short sequences) exit early.
  // (The instantiations without an order leave the code as it was: the order
  // load, even untaken, cost the 8-head tiles ~2% on the Qwen3-14B-shaped batch.)
  uint32_t u = ORDERED ? __ldg(p.order + blockIdx.x) : blockIdx.x;
  const uint32_t pairs = (uint32_t)p.B * p.Hkv * p.HT;
  const int s = p.S - 1 - (int)(u / pairs);
  u %= pairs;
  const int ht = (int)(u % (uint32_t)p.HT);
  u /= (uint32_t)p.HT;
  const int kvh = (int)(u % (uint32_t)p.Hkv);
  const int b = (int)(u / (uint32_t)p.Hkv);
  const int h0 = kvh * p.g + ht * HPT;  // this unit serves query heads h0 .. h0+gl-1
  const int gl = min(HPT, p.g - ht * HPT);
  const int capacity = p.max_blocks << p.bs_log2;
  const int t0 = s * p.P;

  // A box holds bsb rows: a whole page, or a stage's worth of a larger page.
  // Boxes sit box_pitch bytes apart: their size, but at least 128 bytes (a
  // one-row E4M3 box at D = 64 is 64 bytes), so every copy lands 128-byte aligned.
  const int bsb_log2 = min(p.bs_log2, ST_LOG2);
  const int nbox = ST >> bsb_log2;  // boxes per stage
  const uint32_t box_bytes = (uint32_t)ROWB << bsb_log2;
  const uint32_t box_pitch = box_bytes < 128u ? 128u : box_bytes;
  const int32_t *trow = p.tables + (int64_t)b * p.table_stride;

  // Stages are counted from tu, the first stage holding a token of the unit:
  // t0 unless a sliding window starts later.  Warp 0 fetches the block ids of
  // the first NST stages while the length is still in flight (clamped to the
  // table row; an id is used only for a stage that holds live tokens): lane j
  // holds box j, j + 32, ... of a stage.
  int tu = t0;
  int ids[NST][IDW];
  auto load_ids = [&](int (&dst)[IDW], int st) {
    const int page0 = (tu + st * ST) >> p.bs_log2;
#pragma unroll
    for (int w = 0; w < IDW; ++w) {
      const int j = lane + 32 * w;
      dst[w] = j < nbox ? __ldg(trow + min(page0 + j, p.max_blocks - 1)) : 0;
    }
  };
  if (warp == 0) {
#pragma unroll
    for (int k = 0; k < NST; ++k) load_ids(ids[k], k);
  }
  if (tid == 0) {
#pragma unroll
    for (int i = 0; i < NST; ++i) mbar_init(smem_addr(full + i), 1);
    fence_mbar_init();
  }

  int L = __ldg(p.seq_lens + b);
  if (L < 0 || L > capacity) {
    if (tid == 0 && s == 0 && kvh == 0 && ht == 0) atomicOr(p.err, kErrSeqLen);
    L = L < 0 ? 0 : capacity;
  }
  // tokens that take part: [lo, L) -- the last window tokens under a sliding
  // window ("Attention parity: run every attention type on the best available
  // path on both targets", section "Current state": out-of-window block skip);
  // this unit covers [tlo, t1) of them
  const int lo = (p.window > 0 && L > p.window) ? L - p.window : 0;
  const int t1 = min(t0 + p.P, L);
  const int tlo = max(t0, lo);
  if (tlo >= t1) {
    if (L == 0 && s == 0) {  // empty sequence: out = 0, lse = -inf (or the sink)
      for (int i = tid; i < gl * D; i += NTH)
        p.out[b * p.o_sb + (int64_t)(h0 + i / D) * p.o_sh + (i % D)] = 0;
      if (p.lse != nullptr && tid < gl)
        p.lse[b * p.lse_sb + (int64_t)(h0 + tid) * p.lse_sh] = p.sinks != nullptr ? p.sinks[h0 + tid] : -INFINITY;
    }
    unit_exit<D, HPT, F8, NST, ST, CPS>(p, s, nullptr);
    return;  // pages wholly outside [lo, L) are never read
  }
  const int s_first = lo / p.P;                      // first non-empty partition of sequence b
  const int ns = (L + p.P - 1) / p.P - s_first;     // non-empty partitions
  if (tlo >= t0 + ST) {  // stages wholly before the window are skipped
    tu = t0 + ((tlo - t0) / ST) * ST;
    if (warp == 0) {
#pragma unroll
      for (int k = 0; k < NST; ++k) load_ids(ids[k], k);
    }
  }
  const int nstages = (t1 - tu + ST - 1) / ST;
  __syncthreads();  // the stage barriers are initialised

  // Stage st into ring slot st % NST (called by all of warp 0; lane 0 issues).
  // Only boxes holding live tokens ([tlo, t1)) are copied.
  auto issue = [&](const int (&sid)[IDW], int st) {
    const int tb = tu + st * ST;
    const int jb = tb < tlo ? (tlo - tb) >> bsb_log2 : 0;
    const int nb = min(nbox, (t1 - tb + (1 << bsb_log2) - 1) >> bsb_log2);
    uint8_t *sK = smem + (st % NST) * STAGE_BYTES;
    uint8_t *sV = sK + HALF;
    const uint32_t bar = smem_addr(full + st % NST);
    const int slot0 = tb & ((1 << p.bs_log2) - 1);  // row of the box inside its page
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(nb - jb) * box_bytes * 2);
#pragma unroll
    for (int w = 0; w < IDW; ++w) {
#pragma unroll 1
      for (int jj = max(0, jb - 32 * w); jj < 32 && 32 * w + jj < nb; ++jj) {
        const int j = 32 * w + jj;
        const int id = __shfl_sync(0xffffffffu, sid[w], jj);
        if (lane == 0) {
          if ((unsigned)id >= (unsigned)p.num_blocks) atomicOr(p.err, kErrBlockId);  // the box reads as zeros
          tma_load_5d(smem_addr(sK + j * box_pitch), &p.tmk, 0, slot0, 0, kvh, id, bar);
          tma_load_5d(smem_addr(sV + j * box_pitch), &p.tmv, 0, slot0, 0, kvh, id, bar);
        }
      }
    }
  };
  if (warp == 0) {
#pragma unroll
    for (int k = 0; k < NST - 1; ++k)
      if (k < nstages) issue(ids[k], k);
  }
  int (&idn)[IDW] = ids[NST - 1];  // block ids of the next stage to issue

  // Address of 16-byte chunk (column block h, chunk c of it) of row r in a K
  // or V half-stage: rows grouped in boxes of 2^bsb_log2 rows, each box laid out
  // [column blocks][rows][RW bytes].  The TMA's 128-byte swizzle XORs the chunk
  // index with address bits 7-9; the 64-byte swizzle (E4M3 rows at D = 64, one
  // column block) XORs chunk bits 4-5 with address bits 7-8.  rbase/rkey depend
  // on the row only.
  auto row_base = [&](int r, uint32_t &rbase, uint32_t &rkey) {
    const int slot = r & ((1 << bsb_log2) - 1);
    rbase = (uint32_t)(r >> bsb_log2) * box_pitch + (uint32_t)(slot * RW);
    rkey = rbase >> 7;
  };
  auto chunk = [&](uint32_t rbase, uint32_t rkey, int h, int c) -> uint32_t {
    if constexpr (RW == 128)
      return rbase + ((uint32_t)h << (bsb_log2 + 7)) + ((((uint32_t)c) ^ ((rkey + ((uint32_t)h << bsb_log2)) & 7u)) << 4);
    else
      return rbase + ((((uint32_t)c) ^ (rkey & 3u)) << 4);
  };
  // QK operand rows (ldmatrix of K) and PV operand rows (transposed ldmatrix
  // of V) of this warp's tiles: tile i of token group tg is stage rows
  // 16 (i TG + tg) .. +15.  (E4M3: both operands' matrices 0/1 are tokens
  // 0-7/8-15 of the first 16 bytes, matrices 2/3 the same tokens of the next 16.)
  // Each lane keeps, per tile and per column block it reads, the offset of its
  // row's chunk c0 (lane/16 for K and E4M3 V, bit 3 of the lane for bf16 V).
  // An operand x bytes into the column block is chunk c0 + x/16 with x/16
  // even, i.e. c0 XOR x/16, and the swizzle XORs the chunk index, so its
  // address is (stage address + offset) XOR x: one instruction per load,
  // instead of the swizzle arithmetic (the stage address is a multiple of 128
  // and an offset has c0's swizzled chunk in bits 4-6 only).  Written as
  // (offset XOR x) + stage address, the same value, the bf16 32-head tile at
  // D = 128 (at its 128-register cap) measured 1.5% faster on B200 and the
  // other measured instances 1-4% slower, so only that tile takes that form.
  constexpr int EB = F8 ? 1 : 2;                      // bytes per element
  constexpr int NKB = ROWB / RW;                      // column blocks of a K row
  constexpr int NVB = (MT * 16 * EB + RW - 1) / RW;   // column blocks of this warp's V rows
  static_assert(DS == 1 || (MT * 16 * EB) % RW == 0, "a warp's head_dim rows start on a column block");
  uint32_t kb[TPW][NKB], vb[TPW][NVB];
  auto op_addr = [](uint32_t stage, uint32_t off, uint32_t x) -> uint32_t {
    if constexpr (!F8 && D == 128 && HPT == 32) return (off ^ x) + stage;
    else return (stage + off) ^ x;
  };
  {
    const int vh0 = dh * MT * 16 * EB / RW;           // first of them
    const int c0k = lane >> 4, c0v = F8 ? (lane >> 4) : ((lane >> 3) & 1);
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      const int r0 = 16 * (i * TG + tg) + (lane & 7);
      uint32_t rb, rk;
      row_base(r0 + ((lane >> 3) & 1) * 8, rb, rk);
#pragma unroll
      for (int h = 0; h < NKB; ++h) kb[i][h] = chunk(rb, rk, h, c0k);
      row_base(r0 + ((F8 ? (lane >> 3) : (lane >> 4)) & 1) * 8, rb, rk);
#pragma unroll
      for (int h = 0; h < NVB; ++h) vb[i][h] = chunk(rb, rk, vh0 + h, c0v);
    }
  }

  // Q^T fragments (B operand of S^T = K.Q^T): lane holds head nt*8 + lane/4,
  // dims 16kk + 2(lane%4) + {0,1} and + {8,9} -- with an E4M3 cache, in the
  // permuted order of its K operands, 16kk + 4(lane%4) + {0,1} and + {2,3}.
  // Padded heads are zero.  With an E4M3 cache the fragments are f16: q times
  // 2^qe, qe chosen so that the tile's largest |q| lies in [2^14, 2^15), which
  // keeps every bf16 value exact (down to 2^-28 of that largest, where f16 turns
  // subnormal), and 2^-qe joins the score scale.
  uint32_t qf[KT][NTW][2];
  float sl2 = p.scale_log2;
  auto q_row = [&](int nt, bool &ok) -> const uint16_t * {
    const int hl = (hg * NTW + nt) * 8 + (lane >> 2);
    ok = hl < gl;
    return p.q + b * p.q_sb + (int64_t)(h0 + (ok ? hl : 0)) * p.q_sh + (lane & 3) * (F8 ? 4 : 2);
  };
#pragma unroll
  for (int nt = 0; nt < NTW; ++nt) {
    bool ok;
    const uint16_t *qr = q_row(nt, ok);
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      qf[kk][nt][0] = ok ? __ldg(reinterpret_cast<const uint32_t *>(qr + kk * 16)) : 0u;
      qf[kk][nt][1] = ok ? __ldg(reinterpret_cast<const uint32_t *>(qr + kk * 16 + (F8 ? 2 : 8))) : 0u;
    }
  }
  if constexpr (F8) {
    float amax = 0.f;
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
      for (int kk = 0; kk < KT; ++kk)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t w = qf[kk][nt][j];
          amax = fmaxf(amax, fmaxf(fabsf(__uint_as_float(w << 16)), fabsf(__uint_as_float(w & 0xffff0000u))));
        }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    int e2 = 0;
    if (amax > 0.f && amax <= 3.0e38f) frexpf(amax, &e2);  // amax = f 2^e2, f in [0.5, 1)
    const int qe = amax > 0.f && amax <= 3.0e38f ? min(100, max(-100, 15 - e2)) : 0;
    const float qs = __int_as_float((127 + qe) << 23);
    sl2 = p.scale_log2 * __int_as_float((127 - qe) << 23);
#pragma unroll
    for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
      for (int kk = 0; kk < KT; ++kk)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const uint32_t w = qf[kk][nt][j];
          qf[kk][nt][j] = pack_f16x2(__uint_as_float(w << 16) * qs, __uint_as_float(w & 0xffff0000u) * qs);
        }
  }

  float oacc[MT][NTW][4];
  float m_run[NTW][2], l_run[NTW][2];
#pragma unroll
  for (int nt = 0; nt < NTW; ++nt) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      m_run[nt][j] = -INFINITY;
      l_run[nt][j] = 0.f;
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) oacc[mt][nt][i] = 0.f;
  }

  int st = 0;
  bool aborted = false;
#pragma unroll 1
  for (; st < nstages; ++st) {
    const int nx = st + NST - 1;
    if (warp == 0 && nx < nstages) {
      issue(idn, nx);                                 // ids fetched one stage ago
      if (nx + 1 < nstages) load_ids(idn, nx + 1);   // in flight during this stage's math
    }
    const bool landed = wait_stage(smem_addr(full + st % NST), (st / NST) & 1, p.err);

    uint8_t *sK = smem + (st % NST) * STAGE_BYTES;
    uint8_t *sV = sK + HALF;
    const uint32_t aK = smem_addr(sK), aV = aK + (uint32_t)HALF;
    const int tb = tu + st * ST;
    if (tb + ST > t1 || tb < tlo) {
      // the first and last stages: V rows outside [tlo, t1) (slots past L_b,
      // tokens before the window, rows of boxes not copied) are zeroed so that
      // their zero weights meet finite values
#pragma unroll 1
      for (int e = lane; e < TPW * 16 * CH; e += 32) {
        const int r = 16 * ((e / (16 * CH)) * TG + tg) + (e / CH) % 16, c = e % CH;
        if (tb + r >= t1 || tb + r < tlo) {
          uint32_t rb, rk;
          row_base(r, rb, rk);
          *reinterpret_cast<uint4 *>(sV + chunk(rb, rk, c / CPB, c % CPB)) = make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();  // before the slot's next TMA write
      __syncwarp();
    }
    int tbase[TPW];
    bool live = false;
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      tbase[i] = tb + 16 * (i * TG + tg);
      live = live || (tbase[i] < t1 && tbase[i] + 16 > tlo);
    }
    if (live) {  // one of the warp's tiles holds a live token
      // ---- S^T = K . Q^T over each tile's 16 tokens; k-step kk accumulates
      // into chain kk % NCH, so NCH MMA chains run side by side
      float sc[NCH][TPW][NTW][4];
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int i = 0; i < TPW; ++i)
#pragma unroll
          for (int nt = 0; nt < NTW; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) sc[c][i][nt][j] = 0.f;
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        if constexpr (F8) {
          // one ldmatrix.x4 per two k-steps: r[0]/r[1] hold codes 32kp +
          // 4(lane%4) .. +3 of tokens lane/4 and lane/4 + 8, r[2]/r[3] the next
          // 16 bytes; each pair of codes widens to f16x2 exactly
#pragma unroll
          for (int kp = 0; kp < KT / 2; ++kp) {
            uint32_t r[4];
            ldsm_x4(r, op_addr(aK, kb[i][kp * 32 / RW], kp * 32 % RW));
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const int kk = 2 * kp + hf;
              uint32_t a[4];
              e4m3x4_to_f16x2x2(r[2 * hf], a[0], a[2]);
              e4m3x4_to_f16x2x2(r[2 * hf + 1], a[1], a[3]);
#pragma unroll
              for (int nt = 0; nt < NTW; ++nt) mma_16816_f16(sc[kk % NCH][i][nt], a, qf[kk][nt][0], qf[kk][nt][1]);
            }
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < KT; ++kk) {
            uint32_t a[4];
            ldsm_x4(a, op_addr(aK, kb[i][kk * 32 / RW], kk * 32 % RW));
#pragma unroll
            for (int nt = 0; nt < NTW; ++nt) mma_16816(sc[kk % NCH][i][nt], a, qf[kk][nt][0], qf[kk][nt][1]);
          }
        }
      }

      // ---- online softmax over the warp's tiles (rows lane/4 and lane/4 + 8 of
      // each; columns 2(lane%4) + {0,1})
      uint32_t pb[TPW][NTW][2];
#pragma unroll
      for (int nt = 0; nt < NTW; ++nt) {
        float sv[TPW][4];
        bool over = false;  // a score of this lane passes its head's reference by more than the slack
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          const int ra = tbase[i] + (lane >> 2), rb8 = ra + 8;
          const bool okA = ra >= tlo && ra < t1;
          const bool okB = rb8 >= tlo && rb8 < t1;
          float acc[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[j] = sc[0][i][nt][j];
#pragma unroll
            for (int c = 1; c < NCH; ++c) acc[j] += sc[c][i][nt][j];
          }
          sv[i][0] = okA ? acc[0] * sl2 : -INFINITY;
          sv[i][1] = okA ? acc[1] * sl2 : -INFINITY;
          sv[i][2] = okB ? acc[2] * sl2 : -INFINITY;
          sv[i][3] = okB ? acc[3] * sl2 : -INFINITY;
          over = over || fmaxf(sv[i][0], sv[i][2]) > m_run[nt][0] + kRescaleSlack ||
                 fmaxf(sv[i][1], sv[i][3]) > m_run[nt][1] + kRescaleSlack;
        }
        // Lazy rescale: a head's reference max moves only when a score passes
        // it by more than kRescaleSlack (log2 units), so weights stay below
        // 2^kRescaleSlack and the O^T rescale is skipped on almost every tile.
        // Any reference point gives the same out and lse as long as l and O^T
        // share it.  The reference is uniform over the eight lanes that hold a
        // head, so each lane tests its own scores and one vote decides; the
        // tile's maximum (three shuffle rounds) is taken only when the
        // reference moves.  A tile holds a live token and the first reference is
        // -inf, so the first step always sets it.
        if (__any_sync(0xffffffffu, over)) {
          float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
          for (int i = 0; i < TPW; ++i) {
            mx0 = fmaxf(mx0, fmaxf(sv[i][0], sv[i][2]));
            mx1 = fmaxf(mx1, fmaxf(sv[i][1], sv[i][3]));
          }
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
          }
          const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
          const float al0 = fast_exp2(m_run[nt][0] - mn0), al1 = fast_exp2(m_run[nt][1] - mn1);
          m_run[nt][0] = mn0;
          m_run[nt][1] = mn1;
          l_run[nt][0] *= al0;
          l_run[nt][1] *= al1;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            oacc[mt][nt][0] *= al0;
            oacc[mt][nt][1] *= al1;
            oacc[mt][nt][2] *= al0;
            oacc[mt][nt][3] *= al1;
          }
        }
#pragma unroll
        for (int i = 0; i < TPW; ++i) {
          const float e0 = fast_exp2(sv[i][0] - m_run[nt][0]), e1 = fast_exp2(sv[i][1] - m_run[nt][1]);
          const float e2 = fast_exp2(sv[i][2] - m_run[nt][0]), e3 = fast_exp2(sv[i][3] - m_run[nt][1]);
          const uint32_t pA = F8 ? pack_f16x2(e0, e1) : pack_bf16x2(e0, e1);
          const uint32_t pB = F8 ? pack_f16x2(e2, e3) : pack_bf16x2(e2, e3);
          // The running sum takes the fp32 weights: summing the rounded ones
          // moves the LSE of a short sequence by up to 2^-9 (one weight's rounding).
          l_run[nt][0] += e0 + e2;
          l_run[nt][1] += e1 + e3;
          pb[i][nt][0] = movmatrix_t(pA);
          pb[i][nt][1] = movmatrix_t(pB);
        }
      }

      // ---- O^T += V^T . P^T over this warp's head_dim rows (rows outside
      // [tlo, t1) were zero-filled, their weights are 0)
      if constexpr (F8) {
        // one transposed ldmatrix.x4 per two m-tiles: r[0]/r[1] hold, for
        // tokens 2(lane%4) and +1 (of 0-7 / 8-15), the codes of head_dim
        // 16gm + 2(lane/4) and +1; r[2]/r[3] the same of m-tile gm + 1.  A
        // byte permute pairs the two tokens of each head_dim row.
#pragma unroll
        for (int mp = 0; mp < MT / 2; ++mp) {
#pragma unroll
          for (int i = 0; i < TPW; ++i) {
            uint32_t r[4];
            ldsm_x4_t(r, op_addr(aV, vb[i][mp * 32 / RW], mp * 32 % RW));
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const uint32_t x0 = byte_perm(r[2 * hf], 0x3120), x1 = byte_perm(r[2 * hf + 1], 0x3120);
              uint32_t a[4];
              e4m3x4_to_f16x2x2(x0, a[0], a[1]);
              e4m3x4_to_f16x2x2(x1, a[2], a[3]);
#pragma unroll
              for (int nt = 0; nt < NTW; ++nt) mma_16816_f16(oacc[2 * mp + hf][nt], a, pb[i][nt][0], pb[i][nt][1]);
            }
          }
        }
      } else {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {  // m-tile dh MT + mt of head_dim rows
#pragma unroll
          for (int i = 0; i < TPW; ++i) {
            uint32_t a[4];
            ldsm_x4_t(a, op_addr(aV, vb[i][mt * 32 / RW], mt * 32 % RW));
#pragma unroll
            for (int nt = 0; nt < NTW; ++nt) mma_16816(oacc[mt][nt], a, pb[i][nt][0], pb[i][nt][1]);
          }
        }
      }
    }
    // every warp is done with slot st % NST before it is refilled; a stage
    // whose copies never landed ends the loop for the whole CTA
    if (__syncthreads_or(!landed)) {
      aborted = true;
      break;
    }
  }
  if (aborted) {
    // leave no copy in flight: wait (bounded) for every stage issued after st
    if (tid == 0)
      for (int j = st; j < nstages && j < st + NST; ++j) wait_stage(smem_addr(full + j % NST), (j / NST) & 1, p.err);
    __syncthreads();
    return;
  }

  // ---- merge the token groups' states through shared memory (the ring is
  // free); rows padded to D+4 floats so the fragment stores are conflict free.
  // The warps of a head_dim pair hold identical (m, l); the first one stores them.
  constexpr int MROW = D + 4;
  float *sm_o = reinterpret_cast<float *>(smem);  // [TG][HPT][MROW]
  float *sm_m = sm_o + TG * HPT * MROW;            // [TG][HPT]
  float *sm_l = sm_m + TG * HPT;                   // [TG][HPT]
#pragma unroll
  for (int nt = 0; nt < NTW; ++nt) {
    const int hn = (hg * NTW + nt) * 8;  // first head of this n-tile in the head tile
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      float l = l_run[nt][j];
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
      if (dh == 0 && lane < 4) {
        sm_m[tg * HPT + hn + 2 * lane + j] = m_run[nt][j];
        sm_l[tg * HPT + hn + 2 * lane + j] = l;
      }
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      // accumulator rows lane/4 and lane/4 + 8 are head_dim rows d and d2
      const int d = (dh * MT + mt) * 16 + (F8 ? 2 : 1) * (lane >> 2);
      const int d2 = d + (F8 ? 1 : 8);
      float *o0 = sm_o + (tg * HPT + hn + (lane & 3) * 2) * MROW;
      o0[d] = oacc[mt][nt][0];
      o0[MROW + d] = oacc[mt][nt][1];
      o0[d2] = oacc[mt][nt][2];
      o0[MROW + d2] = oacc[mt][nt][3];
    }
  }
  __syncthreads();

  constexpr int D4 = D / 4;
  for (int i = tid; i < gl * D4; i += NTH) {
    const int hl = i / D4, d = (i % D4) * 4;
    float m = -INFINITY;
#pragma unroll
    for (int w = 0; w < TG; ++w) m = fmaxf(m, sm_m[w * HPT + hl]);
    float l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int w = 0; w < TG; ++w) {
      const float mw = sm_m[w * HPT + hl];
      if (mw == -INFINITY) continue;  // token group saw no token of this partition
      const float f = fast_exp2(mw - m);
      l += f * sm_l[w * HPT + hl];
      const float4 ow = *reinterpret_cast<const float4 *>(sm_o + (w * HPT + hl) * MROW + d);
      o.x += f * ow.x;
      o.y += f * ow.y;
      o.z += f * ow.z;
      o.w += f * ow.w;
    }
    const float inv = (F8 ? p.v_scale : 1.f) / l;  // out carries v_scale, lse does not
    const float lse_nat = (m + log2f(l)) * kLn2;
    const int h = h0 + hl;
    if (ns == 1) {
      float sc = inv, lse_out = lse_nat;
      if (p.sinks != nullptr) {
        // the head's sink logit joins the softmax (same page and section:
        // attention sinks): lse' = logaddexp(lse, sink), out scaled by exp(lse - lse')
        const float sg = p.sinks[h];
        lse_out = fmaxf(lse_nat, sg) + log1pf(__expf(-fabsf(lse_nat - sg)));
        sc *= __expf(lse_nat - lse_out);
      }
      uint2 packed;
      packed.x = pack_bf16x2(o.x * sc, o.y * sc);
      packed.y = pack_bf16x2(o.z * sc, o.w * sc);
      *reinterpret_cast<uint2 *>(p.out + b * p.o_sb + (int64_t)h * p.o_sh + d) = packed;
      if (d == 0 && p.lse != nullptr) p.lse[b * p.lse_sb + (int64_t)h * p.lse_sh] = lse_out;
    } else {
      const int64_t row = ((int64_t)b * p.Hq + h) * p.S + s;
      *reinterpret_cast<float4 *>(p.o_part + row * D + d) = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
      if (d == 0) p.lse_part[row] = lse_nat;
    }
  }
  if (unit_exit<D, HPT, F8, NST, ST, CPS>(p, s, full + 12) || ns == 1) return;
  if (claim_last_partition(p, b, kvh, ht, ns, flag))
    merge_partials<D, NTH>(p, b, h0, gl, s_first, ns, reinterpret_cast<float *>(smem));  // the ring is free
}

int partition_stages(int D, int hpt, bool kv_fp8) { return stages_for(D, hpt, kv_fp8); }

// ---- the unit schedule -------------------------------------------------------
//
// One CTA orders the launch's units by the number of tokens they stream,
// longest first (64 buckets of P/64 tokens; empty units last), and writes the
// permutation to p.order.  A unit's tokens are those of partition s of
// sequence b that take part: [max(s P, lo), min((s+1) P, L_b)), lo the first
// token of a sliding window.  With more units than CTA slots, the block
// scheduler dispatches the order's tail after the first wave; ordered this
// way that tail is the partial last partitions rather than full ones, which is
// what a ragged batch's time was waiting on (longest-processing-time-first
// list scheduling).  Units of one (b, s) -- its KV heads and head tiles --
// stay adjacent.  The order within a bucket follows shared-memory atomics and
// may change from call to call; which CTA runs a unit changes no result.
constexpr int kScheduleThreads = 1024;
constexpr int kScheduleBuckets = 64;

__global__ void __launch_bounds__(kScheduleThreads) schedule_kernel(const __grid_constant__ PartitionParams p) {
  __shared__ uint32_t count[kScheduleBuckets], next[kScheduleBuckets];
  const int tid = threadIdx.x;
  if (tid < kScheduleBuckets) count[tid] = 0;
  __syncthreads();
  const int capacity = p.max_blocks << p.bs_log2;
  const uint32_t per = (uint32_t)p.Hkv * p.HT;  // units of one (b, s)
  const uint32_t pairs = (uint32_t)p.B * per;    // units of one partition index
  const int npair = p.B * p.S;
  auto bucket = [&](int i) -> int {  // 0: P tokens ... kScheduleBuckets - 1: none
    const int b = i / p.S, s = i % p.S;
    int L = __ldg(p.seq_lens + b);
    L = L < 0 ? 0 : (L > capacity ? capacity : L);
    const int lo = (p.window > 0 && L > p.window) ? L - p.window : 0;
    const int t0 = s * p.P;
    const int work = min(t0 + p.P, L) - max(t0, lo);
    return work <= 0 ? kScheduleBuckets - 1
                     : (int)((int64_t)(p.P - work) * (kScheduleBuckets - 1) / p.P);
  };
  for (int i = tid; i < npair; i += kScheduleThreads) atomicAdd(&count[bucket(i)], 1u);
  __syncthreads();
  if (tid == 0) {
    uint32_t acc = 0;
    for (int k = 0; k < kScheduleBuckets; ++k) {
      next[k] = acc;
      acc += count[k];
    }
  }
  __syncthreads();
  uint32_t *order = p.order;
  for (int i = tid; i < npair; i += kScheduleThreads) {
    const uint32_t slot = atomicAdd(&next[bucket(i)], 1u);
    const int b = i / p.S, s = i % p.S;
    const uint32_t first = (uint32_t)(p.S - 1 - s) * pairs + (uint32_t)b * per;  // unit (b, s, kv head 0, tile 0)
    for (uint32_t j = 0; j < per; ++j) order[slot * per + j] = first + j;
  }
}

cudaError_t launch_schedule(const PartitionParams &p, cudaStream_t stream) {
  schedule_kernel<<<1, kScheduleThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int HPT, bool F8, bool ORDERED, int CPS>
static cudaError_t launch_o(const PartitionParams &p, int grid, cudaStream_t stream) {
  static std::atomic<uint64_t> attr_done{0};
  constexpr int NW = warps_for(D, HPT, F8);
  constexpr SmemPlan SP = smem_plan_for(D, HPT, F8, NW);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (!(attr_done.load(std::memory_order_acquire) & bit)) {
    e = cudaFuncSetAttribute(partition_kernel<D, HPT, F8, NW, ORDERED, CPS>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SP.total);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit, std::memory_order_acq_rel);
  }
  partition_kernel<D, HPT, F8, NW, ORDERED, CPS><<<grid, NW * 32, SP.total, stream>>>(p);
  return cudaGetLastError();
}

template <int D, int HPT, bool F8, int CPS>
static cudaError_t launch_c(const PartitionParams &p, int grid, cudaStream_t stream) {
  return p.order != nullptr ? launch_o<D, HPT, F8, true, CPS>(p, grid, stream)
                            : launch_o<D, HPT, F8, false, CPS>(p, grid, stream);
}

template <int D, int HPT, bool F8>
static cudaError_t launch_t(const PartitionParams &p, int grid, int ctas_per_sm, cudaStream_t stream) {
  if constexpr (has_dense_build(D, HPT, F8)) {
    if (ctas_per_sm == kDenseCtasPerSm) return launch_c<D, HPT, F8, kDenseCtasPerSm>(p, grid, stream);
  }
  constexpr int base = ctas_per_sm_for(D, HPT, F8);
  if (ctas_per_sm != base) return cudaErrorInvalidValue;
  return launch_c<D, HPT, F8, base>(p, grid, stream);
}

template <bool F8>
static cudaError_t launch_f(const PartitionParams &p, int D, int heads_per_tile, int grid, int cps, cudaStream_t s) {
  switch (D * 64 + heads_per_tile) {
    case 64 * 64 + 8: return launch_t<64, 8, F8>(p, grid, cps, s);
    case 64 * 64 + 16: return launch_t<64, 16, F8>(p, grid, cps, s);
    case 64 * 64 + 32: return launch_t<64, 32, F8>(p, grid, cps, s);
    case 128 * 64 + 8: return launch_t<128, 8, F8>(p, grid, cps, s);
    case 128 * 64 + 16: return launch_t<128, 16, F8>(p, grid, cps, s);
    case 128 * 64 + 32: return launch_t<128, 32, F8>(p, grid, cps, s);
    case 256 * 64 + 8: return launch_t<256, 8, F8>(p, grid, cps, s);
    case 256 * 64 + 16: return launch_t<256, 16, F8>(p, grid, cps, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_partition(const PartitionParams &p, int D, int heads_per_tile, bool kv_fp8, int grid,
                             int ctas_per_sm, cudaStream_t s) {
  if (heads_per_tile > max_heads_per_tile(D)) return cudaErrorInvalidValue;
  return kv_fp8 ? launch_f<true>(p, D, heads_per_tile, grid, ctas_per_sm, s)
                : launch_f<false>(p, D, heads_per_tile, grid, ctas_per_sm, s);
}

cudaError_t device_witness(int device, LaunchWitness **ptr) {
  static std::atomic<LaunchWitness *> cache[64];
  if (device < 0 || device >= 64) return cudaErrorInvalidDevice;
  LaunchWitness *v = cache[device].load(std::memory_order_acquire);
  if (v == nullptr) {
    void *addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_witness);
    if (e != cudaSuccess) return e;
    v = static_cast<LaunchWitness *>(addr);
    cache[device].store(v, std::memory_order_release);
  }
  *ptr = v;
  return cudaSuccess;
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
