// expert_mma.cuh -- the expert SwiGLU MLPs of the block (shared expert and
// routed experts: up + SwiGLU + down) streamed from HBM with TMA, multiplied
// on the tensor cores, in one persistent launch.
//
// Pages: "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and Responsibly"
// (commentary), section "Recovering time between operators": small-batch
// decode waits on weight reads; small-matrix projection kernels at batch 1-2
// and split-K at larger batches expose enough parallel work; the shared
// expert overlaps routing; weights are loaded before their consumer starts;
// dependent work should begin as soon as its inputs exist; the residual add
// belongs in the producing step's epilogue.  The pages' kernels were written
// for GB300 in CuTe DSL; this is a B200 design of the same ideas.
//
// What one launch computes, per unit (one expert's weights over at most 32
// tokens):
//   UP   h[row, :] = x[tok, :] . W13           (fp32, split-K partial sums)
//        a[row, c] = bf16(silu(h[row, c]) * h[row, I + c])  per panel, once complete
//   DOWN acc[tok, :] += w * a[row, :] . W2      (fp32 atomics)
// Shared-expert units take the tokens 32u .. 32u + 31 with weight 1 (rows of
// h_s / a_s are token indices); routed units come from the router's plan
// (rows of h / a are assignment slots b * k + j, weight = routing weight).
//
// Work list, in two segments:
//   A: UP stages of the shared expert's units;
//   B: UP stages of the routed units, DOWN stages of the shared units, DOWN
//      stages of the routed units.
// Segment A needs nothing from the router, so it runs while the router
// kernel (launched just before this one under programmatic dependent launch)
// computes the plan; a producer waits for the plan (its ready flag) only when
// its ticket reaches segment B, whose length it then reads from the plan.
// CTAs pull chunks of stages from a global ticket counter.  Segment A goes
// out in one round of a chunk per CTA; in segment B the first three quarters
// go out in chunks of T/(4G) stages (at most 64), the next 3/16 in quarter
// chunks, the rest one at a time, so the grid needs no co-residency and ends
// with a tail of about one stage.  A DOWN stage reads activation rows [row0,
// row0 + R), which one UP panel of its unit produces; it is issued once that
// panel is published (a per-panel flag holding the launch epoch, so flags
// never need clearing).  Every UP stage is handed out before any DOWN stage,
// so the CTAs that still owe UP work are running and the wait always ends (it
// is bounded all the same).  The shared expert's DOWN stages stay after the
// routed UP stages: placed right after its UP round (segment A), they waited
// for the last UP chunks of each panel with nothing else to stream, which
// measured slower at every batch size.
// The producer keeps the plan (unit list, assignment slots) and the panels it
// has seen published in shared memory: at every chunk change it would
// otherwise walk the plan with chains of dependent L2 reads, and as all CTAs
// change chunks at about the same time, those stalls line up into dips of
// the whole GPU's bandwidth.
//
// Panels.  Each matrix is cut into column panels and K-row stages of 64 KB
// of weights.  A unit with n tokens takes the panel of its token class, the
// narrower the more token tiles it has, so that a consumer warp's columns x
// token tiles -- its accumulators -- stay within 64 fp32 registers:
//   class 0: n <=  8 : 1024 local columns, 32-row stages (1 token tile)
//   class 1: n <= 16 : 1024 local columns, 32-row stages (2 token tiles)
//   class 2: n <= 32 :  512 local columns, 64-row stages (4 token tiles)
// -- 8 consumer warps in every instance, each with 32 (class 0 only) or 64
// accumulators.  Class 0 is not the wider 2048 x 16 shape its one token tile
// would allow: a hidden size of 7 x 1024 (7168) cuts into 2048-column DOWN
// panels with a half-empty last one, and a stage costs about the same ring
// time whatever its bytes (measured: the last panel's 32 KB stages landed
// 0.9x as far apart as the full ones), so 1024 columns stream the DOWN list
// in 7/8 of the stages; a piece (the split-K unit of work) also covers twice
// the rows, which halves the partial sums flushed per weight byte.
// A launch is compiled for the largest class its batch can produce (KC), so
// small batches carry no code for the wider classes.  UP panels pair gate
// columns [c0, c0 + LW/2) with up columns [I + c0, ...), so a panel holds
// both halves of its SwiGLU.
//
// Data movement.  One producer warp fills a shared-memory ring of 64 KB
// stages, guarded by mbarriers, with TMA (no multicast, L2 evict-first):
//  * tensor-map path (hidden and intermediate sizes multiples of 64): each
//    matrix has a tensor map over the 3-D view {64 columns, rows, column
//    chunks of 64}; one tiled load moves a {64, 16, 4} box (16 rows x 256
//    columns, 8 KB) with 128-byte swizzling, so a stage takes 8 loads and the
//    swizzle makes the ldmatrix reads conflict-free.  The TMA engine pays a
//    fixed cost per operation, so few large loads keep it ahead of HBM.
//  * row-copy path (other shapes): one cp.async.bulk per panel row (two for
//    UP), into rows padded by 16 bytes for the same reason.
// Plus one small copy per token of the stage's activations (x for UP, bf16 a
// for DOWN), all counted on the stage's mbarrier, and a stage header.  The
// consumer warps split the panel's columns and run mma.sync.m16n8k16 (bf16
// in, fp32 accumulate) with the tokens as the N dimension.  Partial sums of a
// piece (consecutive stages of one panel) are flushed with fp32 atomics; for
// UP the last warp to contribute to a panel (per-panel counter of
// warp-stages) applies the SwiGLU, returns its accumulators to zero and
// publishes the panel to DOWN.  The consumer loop has no CTA-wide barrier, so
// a warp whose bounded wait gives up can never leave another warp blocked.
#pragma once

#include "moe_device.cuh"

namespace moe {

constexpr int kUnitTok = kMaxUnitTokens;  // tokens of one unit, at most
constexpr int kNumClasses = 3;
// Token classes.  Every stage holds lw x rows = 32K weights (64 KB): 1024 x
// 32 for 1-8 tokens (one 8-token tile) and for 9-16 (two tiles), 512 x 64
// for 17-32 (four tiles); a consumer warp keeps eight accumulator fragments
// (32 floats) in class 0 and sixteen (64 floats) in classes 1 and 2.
__host__ __device__ constexpr int class_lw(int c) { return c == 2 ? 512 : 1024; }
__host__ __device__ constexpr int class_rows(int c) { return c == 2 ? 64 : 32; }
__host__ __device__ constexpr int class_nt(int c) { return c == 0 ? 1 : (c == 1 ? 2 : 4); }
// class of a unit with n <= kUnitTok tokens
__host__ __device__ constexpr int class_for_tokens(int n) { return n <= 8 ? 0 : (n <= 16 ? 1 : 2); }
// FP8 (e4m3) weights, stored [out, in]: a stage is 128 input rows -- one
// 128-byte line of every weight row it touches, and exactly one block of the
// 128 x 128 block scales along the input -- by 512 columns (classes 0 and 1,
// 64 KB) or 256 columns (class 2, 32 KB, so the 32 tokens' 128-row
// activations still fit the stage).  Whole lines keep DRAM and L2 reading
// each weight byte once; narrower K slices of a row (32 bytes per stage) made
// the TMA fetch every line twice.
constexpr int kFp8Rows = 128;
__host__ __device__ constexpr int class_lw_fp8(int c) { return c == 2 ? 256 : 512; }
__host__ __device__ constexpr int geo_rows(int c, bool fp8) { return fp8 ? kFp8Rows : class_rows(c); }
__host__ __device__ constexpr int geo_lw(int c, bool fp8) { return fp8 ? class_lw_fp8(c) : class_lw(c); }
// Bytes of a class's fp8 weights in a stage; the stage's row of block scales
// follows them, and the tokens' activations start 1 KB after that.
__host__ __device__ constexpr int fp8_stage_wbytes(int c) { return class_lw_fp8(c) * kFp8Rows; }
__host__ __device__ constexpr int fp8_stage_xoff(int c) { return fp8_stage_wbytes(c) + 1024; }
constexpr int kFp8XPitch = kFp8Rows * 2 + 16;  // bytes per token row of activations
__host__ __device__ constexpr int cmax(int a, int b) { return a > b ? a : b; }
// Consumer warps: eight in the bf16 instances (nine warps with the producer:
// up to 224 registers a thread, room for 64 accumulators).  Sixteen warps
// with half the columns each measured slower (batch 1 +0.6 %, batch 8
// +2.3 %, batch 64 +3.5 %): the extra warps add contention for the stage's
// shared memory more than they hide its latency; four are slower still.  The
// e4m3 instances, whose conversions make a stage twice the work, keep
// sixteen (eight measured 1.5-2 % slower there).
__host__ __device__ constexpr int consumer_warps_for(int, bool fp8 = false) { return fp8 ? 16 : 8; }
__host__ __device__ constexpr int expert_threads(int kc, bool fp8 = false) {
  return (consumer_warps_for(kc, fp8) + 1) * 32;
}
// m-tiles (16 columns) per consumer warp for class c with cw consumer warps
__host__ __device__ constexpr int class_mt(int c, int cw) { return class_lw(c) / (cw * 16); }
__host__ __device__ constexpr int geo_mt(int c, int cw, bool fp8) { return geo_lw(c, fp8) / (cw * 16); }
// accumulator fragments (of 4 floats) a consumer thread needs for classes <= KC
__host__ __device__ constexpr int class_frags(int c, int cw, bool fp8 = false) {
  return geo_mt(c, cw, fp8) * class_nt(c);
}
__host__ __device__ constexpr int acc_frags(int kc, bool fp8 = false) {
  return kc <= 0 ? class_frags(0, consumer_warps_for(kc, fp8), fp8)
                 : cmax(acc_frags(kc - 1, fp8), class_frags(kc, consumer_warps_for(kc, fp8), fp8));
}
static_assert(acc_frags(0) == 8 && acc_frags(1) == 16 && acc_frags(2) == 16, "32 or 64 accumulators a thread");
// stage buffers: weights (row pitch 2*lw + 16 on the plain-copy path) and
// the tokens' activation rows (pitch 2*rows + 16), largest over the classes
__host__ __device__ constexpr int stage_w_bytes(int c) { return class_rows(c) * (class_lw(c) * 2 + 16); }
constexpr int kStageWBytes = cmax(stage_w_bytes(0), cmax(stage_w_bytes(1), stage_w_bytes(2)));  // 66560
constexpr int kStageXBytes = kUnitTok * (class_rows(2) * 2 + 16);                                 // 4608
constexpr int kStageBytesMma = (kStageWBytes + kStageXBytes + 1023) / 1024 * 1024;               // 70 KB
static_assert(kStageBytesMma % 1024 == 0, "128-byte swizzle atoms need 1 KB aligned stages");
static_assert(fp8_stage_xoff(0) + 8 * kFp8XPitch <= kStageBytesMma &&
                  fp8_stage_xoff(1) + 16 * kFp8XPitch <= kStageBytesMma &&
                  fp8_stage_xoff(2) + 32 * kFp8XPitch <= kStageBytesMma,
              "fp8 stages: weights, scale row and the class's token rows fit one stage");
static_assert(acc_frags(0, true) == 2 && acc_frags(1, true) == 4 && acc_frags(2, true) == 4,
              "e4m3 instances: 8 or 16 accumulators a thread");
constexpr int kMaxStagesMma = 3;
constexpr int kMaxChunk = 64;  // stages per queue grab, at most
// tensor-map path: boxes of {64 columns, 16 rows, 4 column chunks}
constexpr int kChunkCols = 64;
constexpr int kBoxRows = 16;
constexpr int kBoxChunks = 4;
constexpr int kChunkTile = kBoxRows * kChunkCols * 2;  // 2048 B: one chunk of one 16-row block
constexpr int kBoxBytes = kChunkTile * kBoxChunks;     // 8192 B per load
constexpr int kTensorMapBytes = 128;
// UP panels of a unit, at most: ceil(I / 128) (fp8 class 2; bf16 class 2
// needs ceil(I / 256)); sizes the panel counters
__host__ __device__ inline int max_up_panels(int I) { return (I + class_lw_fp8(2) / 2 - 1) / (class_lw_fp8(2) / 2); }

enum : int { kKindUp = 0, kKindDown = 1, kKindEnd = 2 };
enum : int { kFirst = 1, kLast = 2 };

// Stage header, written by the producer before it arms the stage's barrier.
// row[n]: UP -> the h row of token n of the unit; DOWN -> the output row
// (token).  wt[n]: DOWN weight.  seg: 0 shared expert, 1 routed.
struct StageHdr {
  int kind, seg, unit, cls, cp, row0, nrows, flags, ntok, pstages, pad_[2];  // pstages: stages of the piece (on its last)
  int row[kUnitTok];
  float wt[kUnitTok];
};

struct MmaArgs {
  int H;             // hidden (UP rows, DOWN columns)
  int I;             // routed intermediate
  int Is;            // shared intermediate
  int E;             // routed experts (bounds the plan's expert ids)
  int top_k;         // bounds the plan's assignment slots
  int n_stages;      // ring depth
  int batch;         // tokens
  int n_su;          // shared-expert units: ceil(batch / 32), or 0 for no shared expert
  int has_routed;    // 1: routed units too (their plan comes from the previous grid)
  int max_units;     // bound on the plan's n_active
  int panel_stride;  // routed panel counters per unit (max_up_panels(I))
  int panel_stride_s;
  const __nv_bfloat16* w13_s;  // shared expert weights (routed ones come from the pointer tables)
  const __nv_bfloat16* w2_s;
  const uint8_t* maps13;     // tensor-map path: [E] 128-byte maps of the routed w13
  const uint8_t* maps2;      // [E] maps of the routed w2
  const uint8_t* maps13_s;   // shared expert maps
  const uint8_t* maps2_s;
  const Plan* plan;
  const __nv_bfloat16* x;    // [B, H]
  float* h;                  // [B*k, 2I] fp32, zero between calls
  __nv_bfloat16* a;          // [B*k, I] bf16
  float* h_s;                // [B, 2Is]
  __nv_bfloat16* a_s;        // [B, Is]
  float* acc;                // [B, H] fp32 output accumulator, zero between calls
  unsigned* panel_cnt;       // [units * panel_stride] finished warp-stages per UP panel, zero between calls
  unsigned* panel_ready;     // [units * panel_stride] = epoch + 1 once the UP panel's activations are written
  unsigned* panel_cnt_s;     // shared expert: [n_su * panel_stride_s]
  unsigned* panel_ready_s;
  unsigned* queue;           // [0] ticket counter, [1] finished CTAs (zero between calls), [2] launch epoch
  int* plan_ready;           // the plan's ready flag (set by the router), returned to zero by the last CTA out
  unsigned long long* stage_counts;  // [kNumClasses * 2]: UP, DOWN stages per token class, cumulative
  int* status;
  uint32_t spin_limit;       // probes before a bounded wait gives up
  int hold_panel;            // testing only: routed UP panel whose publication is withheld (-1: none)
  int stagger;               // segment B: stagger period of the first big chunks (0: none)
  // FP8 weights: fp32 block scales, rows of sc_pitch* floats per 128 input
  // rows (routed experts' scale arrays come in the pointer tables)
  const float* sc13_s;       // shared expert w13 scales
  const float* sc2_s;        // shared expert w2 scales
  int sc_pitch13, sc_pitch13_s, sc_pitch2;
};

// Producer's copy of the plan in shared memory: per unit the expert id,
// first assignment and token count; per assignment its slot (b * k + j, from
// which the token is b = slot / k); per unit (routed, then shared) the bit
// mask of its UP panels seen published.
constexpr int kMaxSharedUnits = kMaxBatch / kUnitTok;
constexpr int kPlanCacheBytes =
    (kMaxUnits * (2 + 2 + 1) + kMaxAssign * 2 + 3) / 4 * 4 + (kMaxUnits + kMaxSharedUnits) * 4;

__host__ __device__ inline size_t mma_smem_bytes(int n_stages) {
  // + 1 KB so the ring can start on a 1024-byte boundary (128-byte swizzle)
  return 1024 + (size_t)n_stages * kStageBytesMma + 2 * kMaxStagesMma * sizeof(uint64_t) +
         kMaxStagesMma * sizeof(StageHdr) + 16 * sizeof(int) + kPlanCacheBytes;
}

// Panels and stages per panel of one unit with class `cls`, UP or DOWN list
// (I: the unit's intermediate size).
__host__ __device__ __forceinline__ int unit_panels(int cls, bool up, int H, int I, bool fp8 = false) {
  const int lw = geo_lw(cls, fp8);
  return up ? (I + lw / 2 - 1) / (lw / 2) : (H + lw - 1) / lw;
}
__host__ __device__ __forceinline__ int unit_panel_stages(int cls, bool up, int H, int I, bool fp8 = false) {
  const int r = geo_rows(cls, fp8);
  return up ? (H + r - 1) / r : (I + r - 1) / r;
}
__host__ __device__ __forceinline__ int unit_stages(int cls, bool up, int H, int I, bool fp8 = false) {
  return unit_panels(cls, up, H, I, fp8) * unit_panel_stages(cls, up, H, I, fp8);
}

// Ticket schedule over a segment of T stages for a grid of G CTAs
// (make_sched): chunks of c_big = T / (div * G) stages (at most kMaxChunk),
// then about three chunks of c_big / 4 per CTA, then the last 2G stages one
// at a time -- the tail that balances the end is bounded in stages, not a
// fraction of the list, because every chunk ends in a flush of the
// consumers' partial sums.  make_round: one round of at most G chunks of
// max(1, T / G) stages plus the remainder.
// Staggered starts (stag = S > 1): the first G big chunks are shorter by
// tk mod S stages, so CTAs that start the segment together reach their chunk
// changes -- a flush and, for UP pieces, a fence -- at different times
// instead of all at once; the stages taken off go to the quarter band.
struct Sched {
  int T, c_big, c_mid, n_big, n_mid, T1, T2, n_tickets, G, stag;
};
// stages taken off the first m big chunks (m <= G)
__device__ __forceinline__ int sched_stagger_sum(int m, int S) {
  if (S <= 1) return 0;
  const int q = m / S, r = m - q * S;
  return q * (S * (S - 1) / 2) + r * (r - 1) / 2;
}
__device__ __forceinline__ Sched make_round(int T, int G) {
  Sched s;
  s.T = T;
  const int c = T / G > 1 ? T / G : 1;  // every CTA gets a chunk before any gets a second
  s.c_big = c;
  s.n_big = T / c;
  s.T1 = s.n_big * c;
  s.c_mid = T - s.T1 > 0 ? T - s.T1 : 1;  // the remainder, as one more chunk
  s.n_mid = T - s.T1 > 0 ? 1 : 0;
  s.T2 = T;
  s.n_tickets = s.n_big + s.n_mid;
  s.G = G;
  s.stag = 0;
  return s;
}
__device__ __forceinline__ Sched make_sched(int T, int G, int div, int stag = 0) {
  Sched s;
  s.T = T;
  s.G = G;
  int c = T / (div * G);
  c = c < 1 ? 1 : (c > kMaxChunk ? kMaxChunk : c);
  s.c_big = c;
  s.c_mid = c / 4 < 1 ? 1 : c / 4;
  s.stag = stag < c / 2 ? stag : c / 2;  // every big chunk keeps at least half its stages
  const int singles = T < 2 * G ? T : 2 * G;
  const int mid_max = 3 * G * s.c_mid;
  const int rest = T - singles;
  const int mid = rest < mid_max ? rest : mid_max;
  s.n_big = (rest - mid) / c;
  s.T1 = s.n_big * c - sched_stagger_sum(s.n_big < G ? s.n_big : G, s.stag);
  s.n_mid = (T - singles - s.T1) / s.c_mid;
  s.T2 = s.T1 + s.n_mid * s.c_mid;
  s.n_tickets = s.n_big + s.n_mid + (T - s.T2);
  return s;
}
// stages [b, e) of ticket tk (0 <= tk < n_tickets)
__device__ __forceinline__ void sched_range(const Sched& s, int tk, int& b, int& e) {
  if (tk < s.n_big) {
    b = tk * s.c_big - sched_stagger_sum(tk < s.G ? tk : s.G, s.stag);
    e = b + s.c_big - (tk < s.G && s.stag > 1 ? tk % s.stag : 0);
  } else if (tk - s.n_big < s.n_mid) {
    b = s.T1 + (tk - s.n_big) * s.c_mid;
    e = b + s.c_mid;
  } else {
    b = s.T2 + (tk - s.n_big - s.n_mid);
    e = b + 1;
  }
  if (b > s.T) b = s.T;
  if (e > s.T) e = s.T;
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                              uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// Two e4m3 values (the low and high byte of the low 16 bits of v) to f16x2
// (low byte -> low half); exact: every e4m3 value is an f16 value.
__device__ __forceinline__ uint32_t e4m3x2_lo_to_f16x2(uint32_t v) {
  uint32_t d;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(d) : "r"(v));
  return d;
}
__device__ __forceinline__ uint32_t e4m3x2_hi_to_f16x2(uint32_t v) {
  uint32_t d;
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, hi;\n\t}" : "=r"(d) : "r"(v));
  return d;
}
// bf16x2 -> f16x2 (round to nearest; exact for the activations' range)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(__uint_as_float(v & 0xffff0000u)), "f"(__uint_as_float(v << 16)));
  return d;
}

__device__ __forceinline__ void mma_f16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16_16816(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// One stage of tensor-core work for class C: this warp's MT m-tiles against
// the stage's token tiles, accumulated into acc[mt * NT + nt][0..3].
template <int C, int NF, bool TMAP, int CW>
__device__ __forceinline__ void mma_stage(float (&acc)[NF][4], uint32_t sw, uint32_t sx, int LW, int nrows,
                                          int ntiles, int warp, int lane) {
  constexpr int LWc = class_lw(C), R = class_rows(C);
  constexpr int MT = class_mt(C, CW), NT = class_nt(C), KS = R / 16;
  static_assert(MT * NT <= NF, "accumulator budget");
  constexpr int pitch = LWc * 2 + 16, xpitch = R * 2 + 16;
  constexpr int rbstride = (LWc / kChunkCols) * kChunkTile;  // tensor-map layout: one 16-row block
  const int m0 = warp * MT * 16;
  if (m0 >= LW) return;
#pragma unroll
  for (int ks = 0; ks < KS; ++ks) {
    const int k0 = ks * 16;
    if (k0 >= nrows) break;
    const bool half = (nrows - k0) < 16;  // only 8 valid rows in this k-step
    // token fragments: loaded once per k-step and kept for all m-tiles with
    // up to two tiles; four tiles (class 2) are reloaded per m-tile, which
    // measured faster than keeping them (that costs a spill)
    constexpr bool kKeepB = NT <= 2;
    uint32_t b[kKeepB ? NT : 1][2];
    auto load_b = [&](int nt, uint32_t& b0, uint32_t& b1) {
      const int l = lane & 15;
      ldsm_x2(sx + (uint32_t)(nt * 8 + (l & 7)) * xpitch + (uint32_t)(k0 + (l >> 3) * 8) * 2, b0, b1);
      if (half) b1 = 0u;
    };
    if (kKeepB) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        if (nt < ntiles) load_b(nt, b[kKeepB ? nt : 0][0], b[kKeepB ? nt : 0][1]);
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      if (m0 + mt * 16 < LW) {
        const int mi = lane >> 3, r = lane & 7;
        uint32_t a0, a1, a2, a3;
        uint32_t addr;
        if (TMAP) {
          // [16-row block][chunk][16 rows][128 B], 16-byte units swizzled by row % 8
          const int row = (mi >> 1) * 8 + r;                  // row within the k-step's block
          const int col = m0 + mt * 16 + (mi & 1) * 8;        // local column
          const int unit = (col & (kChunkCols - 1)) >> 3;
          addr = sw + (uint32_t)(ks * rbstride + (col / kChunkCols) * kChunkTile + row * 128 + ((unit ^ (row & 7)) << 4));
        } else {
          addr = sw + (uint32_t)(k0 + (mi >> 1) * 8 + r) * pitch + (uint32_t)(m0 + mt * 16 + (mi & 1) * 8) * 2;
        }
        ldsm_x4_trans(addr, a0, a1, a2, a3);
        if (half) a2 = a3 = 0u;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          if (nt < ntiles) {
            uint32_t b0, b1;
            if (kKeepB) {
              b0 = b[kKeepB ? nt : 0][0];
              b1 = b[kKeepB ? nt : 0][1];
            } else {
              load_b(nt, b0, b1);
            }
            mma_bf16_16816(acc[mt * NT + nt], a0, a1, a2, a3, b0, b1);
          }
        }
      }
    }
  }
}

// One stage of tensor-core work on e4m3 weights (class C: class_lw_fp8(C)
// columns x 128 rows), accumulated into the same fragments as mma_stage.
// The stage holds the weights as [column][128 bytes of rows] -- each column's
// rows contiguous, as the [out, in] layout stores them -- with TMA's 128-byte
// swizzle (16-byte unit u of column c sits at unit u ^ (c % 8)).  ldmatrix
// (b16, not transposed) gives a lane (g, t) of an 8 x 8 tile the four bytes
// of rows 4t .. 4t+3 of column g: converted to f16, its low pair is the A
// operand's first k pair and its high pair the second, which is the k order
// (0 1 | 8 9 ...) relabelled; the tokens' fragments are loaded in the same
// order (rows 4t .. 4t+3 as b0, b1), so each product pairs the same row of
// both.  Every e4m3 value is exact in f16 and the activations (bf16, |v| well
// inside f16's range) are converted to f16 too; each product (fp32) is
// multiplied by the warp's block scale -- a warp's columns and a stage's
// rows lie in one 128 x 128 block -- and added to the accumulators.
template <int C, int NF, int CW>
__device__ __forceinline__ void mma_stage_fp8(float (&acc)[NF][4], uint32_t sw, uint32_t sx, const float* srow,
                                              int LW, int nrows, int ntiles, bool up, int c0, int uoff, int I,
                                              int warp, int lane) {
  constexpr int MT = geo_mt(C, CW, true), NT = class_nt(C), KP = kFp8Rows / 32;
  static_assert(MT * NT <= NF, "accumulator budget");
  constexpr int xpitch = kFp8XPitch;
  const int m0 = warp * MT * 16;
  if (m0 >= LW) return;
  const int out0 = up ? (m0 < uoff ? c0 + m0 : I + c0 + (m0 - uoff)) : c0 + m0;
  const float sc = srow[out0 >> 7];
  const int g = lane >> 2, tq = lane & 3;
  const int li = lane >> 3, lr = lane & 7;
  // tokens' fragments of tile nt for the 32-row slice kp: rows 4tq .. 4tq + 3
  // of each 16-row half, converted to f16 (zero past the stage's rows)
  auto load_b = [&](int kp, int nt, uint32_t (&b)[4]) {
    const uint32_t a = sx + (uint32_t)(nt * 8 + g) * xpitch + (uint32_t)(kp * 32 + 4 * tq) * 2;
    uint32_t v0, v1, v2, v3;
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v0), "=r"(v1) : "r"(a));
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v2), "=r"(v3) : "r"(a + 32));
    const bool h0 = kp * 32 + 4 * tq < nrows, h1 = kp * 32 + 16 + 4 * tq < nrows;
    b[0] = h0 ? bf16x2_to_f16x2(v0) : 0u;
    b[1] = h0 ? bf16x2_to_f16x2(v1) : 0u;
    b[2] = h1 ? bf16x2_to_f16x2(v2) : 0u;
    b[3] = h1 ? bf16x2_to_f16x2(v3) : 0u;
  };
  // one token tile: its fragments stay in registers for all m-tiles, and the
  // stage's products are summed over its 128 rows before the one scale
  // multiply (a stage lies in one 128 x 128 block); more tiles: reloaded per
  // m-tile (keeping them all costs spills) and scaled per product
  constexpr bool kKeepB = NT == 1;
  float ts[kKeepB ? MT : 1][4];
#pragma unroll
  for (int mt = 0; mt < (kKeepB ? MT : 1); ++mt)
#pragma unroll
    for (int j = 0; j < 4; ++j) ts[mt][j] = 0.f;
  // (the slice loop stays rolled: unrolled, its hoisted addresses and
  // fragments spill in the classes with several token tiles)
#pragma unroll 1
  for (int kp = 0; kp < KP; ++kp) {
    if (kp * 32 >= nrows) break;
    uint32_t bk[4] = {0u, 0u, 0u, 0u};
    if (kKeepB) load_b(kp, 0, bk);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      if (m0 + mt * 16 < LW) {
        const int col = m0 + mt * 16 + (li & 1) * 8 + lr;  // local column of this lane's ldmatrix row
        const int unit = (2 * kp + (li >> 1)) ^ (col & 7);   // 128-byte swizzle
        uint32_t r0, r1, r2, r3;
        ldsm_x4(sw + (uint32_t)(col * 128 + unit * 16), r0, r1, r2, r3);
        if (kKeepB) {
          mma_f16_16816(ts[kKeepB ? mt : 0], e4m3x2_lo_to_f16x2(r0), e4m3x2_lo_to_f16x2(r1),
                        e4m3x2_hi_to_f16x2(r0), e4m3x2_hi_to_f16x2(r1), bk[0], bk[1]);
          mma_f16_16816(ts[kKeepB ? mt : 0], e4m3x2_lo_to_f16x2(r2), e4m3x2_lo_to_f16x2(r3),
                        e4m3x2_hi_to_f16x2(r2), e4m3x2_hi_to_f16x2(r3), bk[2], bk[3]);
        } else {
          // half by half: one half's A fragment and one tile's B pair live
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t ra = hf ? r2 : r0, rb = hf ? r3 : r1;
            const uint32_t a0 = e4m3x2_lo_to_f16x2(ra), a1 = e4m3x2_lo_to_f16x2(rb);
            const uint32_t a2 = e4m3x2_hi_to_f16x2(ra), a3 = e4m3x2_hi_to_f16x2(rb);
            const bool live = kp * 32 + hf * 16 + 4 * tq < nrows;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              if (nt < ntiles) {
                const uint32_t ad = sx + (uint32_t)(nt * 8 + g) * xpitch + (uint32_t)(kp * 32 + hf * 16 + 4 * tq) * 2;
                uint32_t v0, v1;
                asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(v0), "=r"(v1) : "r"(ad));
                float t[4] = {0.f, 0.f, 0.f, 0.f};
                mma_f16_16816(t, a0, a1, a2, a3, live ? bf16x2_to_f16x2(v0) : 0u, live ? bf16x2_to_f16x2(v1) : 0u);
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[mt * NT + nt][j] = fmaf(sc, t[j], acc[mt * NT + nt][j]);
              }
            }
          }
        }
      }
    }
  }
  if (kKeepB) {
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
      if (m0 + mt * 16 < LW)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[mt * NT][j] = fmaf(sc, ts[kKeepB ? mt : 0][j], acc[mt * NT][j]);
  }
}

// Local columns of a stage: DOWN [0, w) -> c0 + l; UP gate [0, w) -> c0 + l
// and up [uoff, uoff + w) -> I + c0 + (l - uoff); anything else is padding.
// w and uoff are multiples of 8, so four consecutive local columns map to four
// consecutive output columns.
__device__ __forceinline__ int local_to_col(int l, bool up, int c0, int w, int uoff, int I) {
  if (!up) return l < w ? c0 + l : -1;
  if (l < w) return c0 + l;
  if (l >= uoff && l < uoff + w) return I + c0 + (l - uoff);
  return -1;
}

// Flush this warp's partial sums of a piece (class C) with fp32 reductions
// into rows base + row(n) * ld, where lane n of the warp holds row(n) in my_row
// and the weight in my_wt (copied from the stage header, so the stage's slot
// can be handed back before the flush).  A lane's C fragment holds columns
// gid and gid + 8 of an m-tile for tokens 2*tig and 2*tig + 1 of an n-tile;
// each value goes out as one scalar reduction (red, no return value).  Only
// token slots that exist are visited, so a one-token piece costs MT x 2
// reductions per lane of one quad.  (Gathering runs of 4 columns into one
// lane with shuffles for vector reductions measured slower: the shuffles
// cost more issue slots than the reductions they save.)
template <int C, int NF, int CW, bool FP8 = false>
__device__ __forceinline__ void flush_piece(const float (&acc)[NF][4], float* base, size_t ld, int my_row,
                                            float my_wt, int ntok, bool up, int c0, int w, int uoff, int LW, int I,
                                            int warp, int lane) {
  constexpr int MT = geo_mt(C, CW, FP8), NT = class_nt(C);
  const int m0 = warp * MT * 16;
  if (m0 >= LW) return;
  const int gid = lane >> 2, tig = lane & 3;
  const int ntiles = (ntok + 7) >> 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    if (nt >= ntiles) break;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      if (nt * 8 + e >= ntok) break;       // no lane holds a token here (warp-uniform)
      const int n = nt * 8 + tig * 2 + e;  // this lane's token
      const int r = __shfl_sync(0xffffffffu, my_row, n);
      const float wr = __shfl_sync(0xffffffffu, my_wt, n);
      if (n < ntok) {
        float* row = base + (size_t)r * ld;
        const float wt = up ? 1.f : wr;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          if (m0 + mt * 16 >= LW) break;
          const int lo = local_to_col(m0 + mt * 16 + gid, up, c0, w, uoff, I);
          const int hi = local_to_col(m0 + mt * 16 + gid + 8, up, c0, w, uoff, I);
          if (lo >= 0) red_add(row + lo, wt * acc[mt * NT + nt][e]);
          if (hi >= 0) red_add(row + hi, wt * acc[mt * NT + nt][2 + e]);
        }
      }
    }
  }
}

// Shared-memory pieces of the expert kernels (ring, headers, flags, plan copy).
struct SmemView {
  uint8_t* stages;
  uint64_t* full;
  uint64_t* empty;
  StageHdr* hdr;
  volatile int* s_misc;  // [0]: abort flag (a bounded wait gave up), [1]: wait limit (probes),
                         // [2]: stages issued
  uint16_t* s_uexp;      // [kMaxUnits]
  uint16_t* s_ubeg;      // [kMaxUnits]
  uint16_t* s_aslot;     // [kMaxAssign]
  uint8_t* s_ucnt;       // [kMaxUnits]
  uint32_t* s_ready;     // [kMaxUnits + kMaxSharedUnits]
};

// Carve the view out of dynamic shared memory (ring on a 1 KB boundary).
__device__ __forceinline__ SmemView carve_smem(uint8_t* raw, int NS) {
  SmemView v;
  v.stages = raw + ((1024u - (smem_addr(raw) & 1023u)) & 1023u);
  v.full = reinterpret_cast<uint64_t*>(v.stages + (size_t)NS * kStageBytesMma);
  v.empty = v.full + kMaxStagesMma;
  v.hdr = reinterpret_cast<StageHdr*>(v.empty + kMaxStagesMma);
  v.s_misc = reinterpret_cast<volatile int*>(v.hdr + kMaxStagesMma);
  v.s_uexp = reinterpret_cast<uint16_t*>(const_cast<int*>(v.s_misc) + 16);
  v.s_ubeg = v.s_uexp + kMaxUnits;
  v.s_aslot = v.s_ubeg + kMaxUnits;
  v.s_ucnt = reinterpret_cast<uint8_t*>(v.s_aslot + kMaxAssign);
  v.s_ready = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(v.s_uexp) +
                                          (kMaxUnits * (2 + 2 + 1) + kMaxAssign * 2 + 3) / 4 * 4);
  return v;
}

// The last CTA out adds the launch's stages per token class to the device
// counters (evidence of which token classes ran): its copy of the plan is in
// shared memory, as every producer reads the plan before it runs out of
// tickets.  Warp 0, after the CTA's final barrier; one class at a time.
template <int KC, bool FP8>
__device__ __forceinline__ void count_stages_at_exit(const MmaArgs& args, const SmemView& sv, int lane) {
  const int H = args.H, B = args.batch;
  const int n_r = args.has_routed ? sv.s_misc[4] : 0;
#pragma unroll 1
  for (int j = 0; j < kNumClasses; ++j) {
    unsigned up_st = 0, dn_st = 0;
    for (int su = lane; su < args.n_su; su += 32) {
      if (min(class_for_tokens(min(kUnitTok, B - su * kUnitTok)), KC) == j) {
        up_st += unit_stages(j, true, H, args.Is, FP8);
        dn_st += unit_stages(j, false, H, args.Is, FP8);
      }
    }
    for (int u = lane; u < n_r; u += 32) {
      if (min(class_for_tokens((int)sv.s_ucnt[u]), KC) == j) {
        up_st += unit_stages(j, true, H, args.I, FP8);
        dn_st += unit_stages(j, false, H, args.I, FP8);
      }
    }
    up_st = __reduce_add_sync(0xffffffffu, up_st);
    dn_st = __reduce_add_sync(0xffffffffu, dn_st);
    if (lane == 0 && up_st) atomicAdd(&args.stage_counts[2 * j], (unsigned long long)up_st);
    if (lane == 0 && dn_st) atomicAdd(&args.stage_counts[2 * j + 1], (unsigned long long)dn_st);
  }
}

// The producer warp: takes tickets, walks the work list and fills the stage
// ring (weights by TMA, the stage's token activations, the stage header);
// ends by posting a kKindEnd header.  Shared by both expert kernels.
template <int KC, bool TMAP, bool FP8 = false>
__device__ __forceinline__ void producer_loop(const MmaArgs& args, const ExpertTable& tab13, const ExpertTable& tab2,
                                              const SmemView& sv, int NS, unsigned ready_mark, int lane) {
  uint8_t* stages = sv.stages;
  uint64_t* full = sv.full;
  uint64_t* empty = sv.empty;
  StageHdr* hdr = sv.hdr;
  volatile int* s_misc = sv.s_misc;
  volatile int* abort_flag = s_misc;
  uint16_t* s_uexp = sv.s_uexp;
  uint16_t* s_ubeg = sv.s_ubeg;
  uint16_t* s_aslot = sv.s_aslot;
  uint8_t* s_ucnt = sv.s_ucnt;
  uint32_t* s_ready = sv.s_ready;
  const int H = args.H;
    // ================================================================ producer
    const uint64_t pol = l2_evict_first_policy();
    const int G = gridDim.x;
    const int B = args.batch;
    // The ticket counter was returned to zero by the previous launch (see
    // the epoch above), so the first ticket is taken at once.
    int tk = 0;
    if (lane == 0) tk = (int)atomicAdd(&args.queue[0], 1u);
    auto cls_of = [&](int n) {
      const int c = class_for_tokens(n);
      return c > KC ? KC : c;  // cannot exceed: KC is the class of min(batch, 32)
    };
    auto su_tokens = [&](int su) { return min(kUnitTok, B - su * kUnitTok); };
    auto plan_tokens = [&](int u) { return (int)s_ucnt[u]; };  // valid once segment B is known
    for (int i = lane; i < kMaxUnits + kMaxSharedUnits; i += 32) s_ready[i] = 0u;
    __syncwarp();
    // the shared expert's stages are known without the router
    int S_up = 0, S_dn = 0;
    for (int su = 0; su < args.n_su; ++su) {
      const int c = cls_of(su_tokens(su));
      S_up += unit_stages(c, true, H, args.Is, FP8);
      S_dn += unit_stages(c, false, H, args.Is, FP8);
    }
    const int S_A = S_up;  // segment A: the shared UP stages
    const Sched sch_A = make_round(S_up, G);
    // segment B: the routed units, read from the plan once a ticket reaches it
    Sched sch_B = make_sched(S_dn, G, 4, args.stagger);
    bool b_known = !args.has_routed;
    int n_units_r = 0;
    auto know_b = [&]() {
      // The plan is written by the router kernel, whose last CTA sets its
      // ready flag (release) once it is complete: poll that rather than wait
      // for the router grid to complete.  Every router CTA is resident (this
      // grid was launched once all of them had started), so the flag comes;
      // the wait is bounded all the same.
      const Plan* pl = args.plan;
      int ok = 1;
      if (lane == 0) {
        uint32_t it = 0;
        while (ld_acquire_u32(reinterpret_cast<const unsigned*>(&pl->ready)) == 0u) {
          if (++it > (uint32_t)s_misc[1] || *abort_flag) {
            atomicCAS(args.status, kStatusOk, kStatusTimeout);
            *abort_flag = 1;
            ok = 0;
            break;
          }
          __nanosleep(32);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      // copy the plan to shared memory in one round of loads: every unit
      // entry the batch can produce and every assignment slot are loaded
      // together with the unit count (entries past it are never used), then
      // sanitised: an entry the router never produces is flagged and
      // replaced by one that keeps every access in bounds
      const int nas = B * args.top_k;
      const int u_cap = min(args.max_units, nas);
      int n = ok ? __ldcg(&pl->n_active) : 0;
      // (stored so that a negative or oversized value stays out of range and
      // is caught below: count 255 > kUnitTok, begin 0xffff > nas, a
      // negative expert id >= 32768 > E)
#pragma unroll 4
      for (int u = lane; u < u_cap; u += 32) {
        const int cnt = __ldcg(&pl->unit_count[u]), ex = __ldcg(&pl->unit_expert[u]),
                  bg = __ldcg(&pl->unit_begin[u]);
        s_ucnt[u] = (uint8_t)(cnt < 0 ? 255 : min(cnt, 255));
        s_uexp[u] = (uint16_t)(ex < 0 ? 0xffff : min(ex, 0xffff));
        s_ubeg[u] = (uint16_t)(bg < 0 ? 0xffff : min(bg, 0xffff));
      }
      bool bad = false;
#pragma unroll 4
      for (int i = lane; i < nas; i += 32) {
        int sl = __ldcg(&pl->assign_slot[i]);
        if (sl < 0 || sl >= nas) {
          bad = true;
          sl = 0;
        }
        s_aslot[i] = (uint16_t)sl;
      }
      if (n < 0 || n > u_cap) {
        if (lane == 0 && ok) atomicCAS(args.status, kStatusOk, kStatusPlan);
        n = 0;
      }
      n_units_r = n;
      __syncwarp();
      int T = 0;  // at most ~0.5M stages: 32-bit arithmetic
      for (int u = lane; u < n; u += 32) {
        int cnt = s_ucnt[u], ex = s_uexp[u], bg = s_ubeg[u];
        if (cnt > kUnitTok || ex >= args.E || bg + cnt > nas) {
          bad = true;
          cnt = 0;
          ex = 0;
          bg = 0;
          s_ucnt[u] = 0;
          s_uexp[u] = 0;
          s_ubeg[u] = 0;
        }
        const int c = cls_of(cnt);
        T += unit_stages(c, true, H, args.I, FP8) + unit_stages(c, false, H, args.I, FP8);
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) atomicCAS(args.status, kStatusOk, kStatusPlan);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) T += __shfl_xor_sync(0xffffffffu, T, off);
      __syncwarp();
      sch_B = make_sched(T + S_dn, G, 4, args.stagger);
      b_known = true;
      if (lane == 0) s_misc[4] = n;  // routed units, for the stage counters at exit
    };
    // Cursor over the work list: group (0 shared UP, 1 routed UP, 2 shared
    // DOWN, 3 routed DOWN), unit, and the list positions
    // [cur_base, cur_base + cur_size) of its stages.  Tickets only grow, so
    // the cursor only moves forward.
    auto g_seg = [&](int g) { return g & 1; };  // 0 shared, 1 routed
    auto g_up = [&](int g) { return g < 2; };
    int cur_g = 0, cur_unit = 0, cur_base = 0, cur_size = 0;
    auto group_units = [&](int g) { return g_seg(g) == 0 ? args.n_su : n_units_r; };
    auto unit_size = [&](int g, int u) {
      return g_seg(g) == 0 ? unit_stages(cls_of(su_tokens(u)), g_up(g), H, args.Is, FP8)
                           : unit_stages(cls_of(plan_tokens(u)), g_up(g), H, args.I, FP8);
    };
    if (args.n_su > 0) cur_size = unit_size(0, 0);
    auto advance = [&]() {
      cur_base += cur_size;
      ++cur_unit;
      while (cur_unit >= group_units(cur_g)) {
        cur_unit = 0;
        if (++cur_g > 3) {  // past the end of the list (positions never get here)
          cur_size = 1 << 30;
          return;
        }
      }
      cur_size = unit_size(cur_g, cur_unit);
    };
    // The current unit's description lives in registers -- lane j also keeps
    // its token's source row (x row for UP, activation row for DOWN), the
    // row its partial sums go to and its weight -- and is reloaded only when
    // the cursor enters a new unit: with shared memory taking almost all of
    // the SM, L1 is tiny and per-stage plan loads would go to L2 every time.
    int u_seg = -1, u_unit = -1;
    bool u_up = true;
    int u_ntok = 0, u_cls = 0, u_lw = 0, u_R = 0, u_S = 0, u_I = 0, u_src = 0, u_dst = 0;
    float u_w = 1.f;
    const __nv_bfloat16* u_W = nullptr;
    const uint8_t* u_map = nullptr;
    uint32_t q = 0;
    tk = __shfl_sync(0xffffffffu, tk, 0);
    while (true) {
      int c_beg, c_end;
      if (tk < sch_A.n_tickets) {
        sched_range(sch_A, tk, c_beg, c_end);
      } else {
        if (!b_known) know_b();
        const int tr = tk - sch_A.n_tickets;
        if (tr >= sch_B.n_tickets) break;
        sched_range(sch_B, tr, c_beg, c_end);
        c_beg += S_A;
        c_end += S_A;
      }
      if (warp_aborted(abort_flag)) break;
      int tk_next = 0;  // next ticket now: its latency overlaps this chunk
      if (lane == 0) tk_next = (int)atomicAdd(&args.queue[0], 1u);
      int piece_start = c_beg;
      bool stop = false;
      for (int t = c_beg; t < c_end; ++t, ++q) {
        while (t >= cur_base + cur_size) advance();
        const int seg = g_seg(cur_g), unit = cur_unit;  // seg: 0 shared, 1 routed
        const bool up = g_up(cur_g);
        if (unit != u_unit || up != u_up || seg != u_seg) {
          u_seg = seg;
          u_unit = unit;
          u_up = up;
          u_src = u_dst = 0;
          u_w = 1.f;
          if (seg == 0) {
            u_ntok = su_tokens(unit);
            u_I = args.Is;
            u_W = up ? args.w13_s : args.w2_s;
            if (TMAP) u_map = up ? args.maps13_s : args.maps2_s;
            if (lane < u_ntok) u_src = u_dst = unit * kUnitTok + lane;  // x/h_s (UP), a_s/out (DOWN) rows
          } else {
            const int n = s_ucnt[unit];  // sanitised copy of the plan
            const int expert = s_uexp[unit];
            const int begin = s_ubeg[unit];
            u_ntok = n;
            u_I = args.I;
            u_W = up ? tab13.p[expert] : tab2.p[expert];
            if (TMAP) u_map = (up ? args.maps13 : args.maps2) + (size_t)expert * kTensorMapBytes;
            if (lane < n) {
              const int slot = s_aslot[begin + lane];
              const int tok = slot / args.top_k;
              u_src = up ? tok : slot;  // x row (UP) / a row (DOWN)
              u_dst = up ? slot : tok;  // h row (UP) / output row (DOWN)
              if (!up) u_w = __ldcg(&args.plan->assign_w[begin + lane]);
            }
          }
          u_cls = cls_of(u_ntok);
          u_lw = geo_lw(u_cls, FP8);
          u_R = geo_rows(u_cls, FP8);
          u_S = unit_panel_stages(u_cls, up, H, u_I, FP8);
        }
        const int ntok = u_ntok, cls = u_cls, lw = u_lw, R = u_R, S = u_S, Iu = u_I;
        const int loc = t - cur_base;
        const int cp = loc / S;
        const int st = loc - cp * S;
        if (t == c_beg || st == 0) piece_start = t;
        const bool first = (t == piece_start);
        const bool last = (t == c_end - 1 || st == S - 1);
        const int row0 = st * R;
        const int nrows = min(R, (up ? H : Iu) - row0);
        // DOWN reads activation rows [row0, row0 + R): wait for the UP panel
        // that produces them (gate columns [p*lw/2, (p+1)*lw/2))
        if (!up) {
          const int need_p = row0 / (lw / 2);
          const int need_panel = unit * (seg == 0 ? args.panel_stride_s : args.panel_stride) + need_p;
          // (panels past the 32 this CTA caches a bit for are polled each time)
          uint32_t* seen = s_ready + (seg == 0 ? kMaxUnits + unit : unit);
          if (need_p >= 32 || !((*seen >> need_p) & 1u)) {
            const unsigned* pr = (seg == 0 ? args.panel_ready_s : args.panel_ready) + need_panel;
            int ok = 1;
            if (lane == 0) {
              uint32_t it = 0;
              while (ld_acquire_u32(pr) != ready_mark) {
                if (++it > (uint32_t)s_misc[1] || *abort_flag) {
                  atomicCAS(args.status, kStatusOk, kStatusTimeout);
                  *abort_flag = 1;
                  ok = 0;
                  break;
                }
                __nanosleep(64);
              }
              // the activations were written by other CTAs through the generic
              // proxy; order them before this CTA's TMA (async proxy) reads
              asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
              stop = true;
              break;
            }
            if (lane == 0 && need_p < 32) *seen |= 1u << need_p;
            __syncwarp();
          }
        }
        const int slot = q % NS;
        const uint32_t ph = (q / NS) & 1u;
        const bool free_slot =
            mbar_wait_abortable_warp(&empty[slot], ph ^ 1u, args.status, abort_flag);
        if (!free_slot || warp_aborted(abort_flag)) {
          stop = true;
          break;
        }
        const int c0 = cp * (up ? lw / 2 : lw);
        const int w = min(up ? lw / 2 : lw, (up ? Iu : H) - c0);  // columns per half (UP) or panel (DOWN)
        const uint32_t wbytes = (uint32_t)w * 2;
        const uint32_t pitch = (uint32_t)lw * 2 + 16, xpitch = FP8 ? (uint32_t)kFp8XPitch : (uint32_t)R * 2 + 16;
        // tensor-map path: loads = halves x 16-row blocks x groups of 4 chunks
        const int t_ncg = (w / kChunkCols + kBoxChunks - 1) / kBoxChunks;
        const int t_nrb = R / kBoxRows;
        // FP8: loads = halves x 128-column boxes (each 128 rows x 128 bytes),
        // plus the stage's row of block scales (pitch floats per 128 weight rows)
        const int f_nb = (w + 127) / 128;
        const int f_pitch = up ? (seg == 0 ? args.sc_pitch13_s : args.sc_pitch13) : args.sc_pitch2;
        const int t_nops = FP8 ? (up ? 2 : 1) * f_nb : (up ? 2 : 1) * t_nrb * t_ncg;
        const uint32_t wtotal = FP8 ? (uint32_t)t_nops * (128u * kFp8Rows) + (uint32_t)f_pitch * 4u
                                    : (TMAP ? (uint32_t)t_nops * kBoxBytes : (uint32_t)nrows * (up ? 2u : 1u) * wbytes);
        const uint32_t bytes = wtotal + (uint32_t)ntok * nrows * 2;
        uint8_t* sw = stages + (size_t)slot * kStageBytesMma;
        uint8_t* sx = sw + (FP8 ? fp8_stage_xoff(cls) : kStageWBytes);
        StageHdr& hd = hdr[slot];
        if (lane < ntok) {
          hd.row[lane] = u_dst;
          hd.wt[lane] = u_w;
        }
        if (lane == 0) {
          hd.kind = up ? kKindUp : kKindDown;
          hd.seg = seg;
          hd.unit = unit;
          hd.cls = cls;
          hd.cp = cp;
          hd.row0 = row0;
          hd.nrows = nrows;
          hd.flags = (first ? kFirst : 0) | (last ? kLast : 0);
          hd.ntok = ntok;
          hd.pstages = t - piece_start + 1;
        }
        __syncwarp();  // every lane's header writes precede lane 0's (releasing) arrive
        if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
        __syncwarp();
        // activations of this lane's token: x row (UP) or a row (DOWN)
        const void* act = up ? (const void*)(args.x + (size_t)u_src * H + row0)
                             : (const void*)((seg == 0 ? args.a_s : args.a) + (size_t)u_src * Iu + row0);
        if constexpr (FP8) {
          // [column][128 bytes of rows] with 128-byte swizzle, UP's up half
          // from local column lw / 2 (the weights are [out, in]); the input
          // coordinate row0 is a multiple of 128 bytes
          for (int o = lane; o < t_nops; o += 32) {
            const int hh = o / f_nb, mb = o - hh * f_nb;
            uint8_t* dst = sw + (size_t)(hh * (lw / 2) + mb * 128) * kFp8Rows;
            const int m = (up ? (hh ? Iu + c0 : c0) : c0) + mb * 128;
            tma_load_2d(dst, u_map, row0, m, &full[slot], pol);
          }
          if (lane == 31)  // u_W holds the matrix's scale array here
            bulk_copy_g2s(sw + fp8_stage_wbytes(cls), reinterpret_cast<const float*>(u_W) + (size_t)(row0 >> 7) * f_pitch,
                          (uint32_t)f_pitch * 4u, &full[slot], pol);
        } else if (TMAP) {
          const int per_half = t_nrb * t_ncg;
          const int rbstride = (lw / kChunkCols) * kChunkTile;
          const int nch_half = (up ? lw / 2 : lw) / kChunkCols;
          for (int o = lane; o < t_nops; o += 32) {
            const int hh = o / per_half, rem = o - hh * per_half;
            const int rb = rem / t_ncg, cg = rem - rb * t_ncg;
            uint8_t* dst = sw + (size_t)rb * rbstride + (size_t)(hh * nch_half + cg * kBoxChunks) * kChunkTile;
            const int col0 = up ? (hh ? Iu + c0 : c0) : c0;
            tma_load_3d(dst, u_map, 0, row0 + rb * kBoxRows, col0 / kChunkCols + cg * kBoxChunks, &full[slot], pol);
          }
        } else if (up) {
          for (int r = lane; r < nrows; r += 32) {
            const __nv_bfloat16* src = u_W + (size_t)(row0 + r) * (2 * Iu) + c0;
            uint8_t* d = sw + (size_t)r * pitch;
            bulk_copy_g2s(d, src, wbytes, &full[slot], pol);
            bulk_copy_g2s(d + wbytes, src + Iu, wbytes, &full[slot], pol);
          }
        } else {
          for (int r = lane; r < nrows; r += 32)
            bulk_copy_g2s(sw + (size_t)r * pitch, u_W + (size_t)(row0 + r) * H + c0, wbytes, &full[slot], pol);
        }
        if (lane < ntok) bulk_copy_g2s_plain(sx + (size_t)lane * xpitch, act, (uint32_t)nrows * 2, &full[slot]);
        if (lane == 0) {
          s_misc[2] = (int)(q + 1);
        }
      }
      if (stop) break;
      tk = __shfl_sync(0xffffffffu, tk_next, 0);
    }
    // the router grid ended long ago: wait for it formally, so nothing after
    // this grid on the stream can overlap it
    cudaGridDependencySynchronize();
    // tell the consumers there is no more work.  Only into a slot the
    // consumers have handed back: if that wait gave up, a stage may still
    // own the slot (its header in use, its barrier's phase not complete),
    // and an arrival there would fall outside the barrier's phase count --
    // after an abort the consumers stop on their own, as their waits give up
    // once the abort flag is set
    const int slot = q % NS;
    const uint32_t ph = (q / NS) & 1u;
    if (mbar_wait_abortable_warp(&empty[slot], ph ^ 1u, args.status, abort_flag) && lane == 0) {
      hdr[slot].kind = kKindEnd;
      mbar_arrive(&full[slot]);
    }
    __syncwarp();
}

template <int KC, bool TMAP, bool FP8 = false>
__global__ void __launch_bounds__(expert_threads(KC, FP8), 1)
    expert_mlp_kernel(const __grid_constant__ MmaArgs args, const __grid_constant__ ExpertTable tab13,
                      const __grid_constant__ ExpertTable tab2) {
  extern __shared__ __align__(1024) uint8_t mma_smem[];
  const int NS = args.n_stages;
  const SmemView sv = carve_smem(mma_smem, NS);
  uint8_t* stages = sv.stages;
  uint64_t* full = sv.full;
  uint64_t* empty = sv.empty;
  StageHdr* hdr = sv.hdr;
  volatile int* s_misc = sv.s_misc;

  constexpr int CW = consumer_warps_for(KC, FP8);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_producer = (warp == CW);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], CW);
    }
    for (int i = 0; i < 16; ++i) s_misc[i] = 0;
    s_misc[1] = (int)min(args.spin_limit, 0x7fffffffu);
    mbar_fence_init();
  }
  __syncthreads();

  const int H = args.H;
  volatile int* abort_flag = s_misc;
  // Launch epoch: advanced by the last CTA of the previous launch on this
  // workspace, which finished before the previous grid (the router) passed
  // its own dependency wait; every CTA of this launch reads the same value.
  const unsigned ready_mark = __ldcg(&args.queue[2]) + 1u;

  if (is_producer) {
    producer_loop<KC, TMAP, FP8>(args, tab13, tab2, sv, NS, ready_mark, lane);
  } else {
    // =============================================================== consumers
    // (they read nothing the router writes: the stage headers carry it)
    constexpr int NF = acc_frags(KC, FP8);
    float acc[NF][4];
    uint32_t q = 0;
    while (true) {
      const int slot = q % NS;
      const uint32_t ph = (q / NS) & 1u;
      // (warp-uniform: the stage's ldmatrix / mma.sync need all 32 lanes)
      const bool landed = mbar_wait_abortable_warp(&full[slot], ph, args.status, abort_flag);
      if (!landed) break;
      // the header stays valid until this warp releases the slot (below,
      // once the stage's tensor-core work is done); every lane reads the same
      // word, written before the phase the warp observed, so the branch is
      // uniform
      const StageHdr& hd = hdr[slot];
      if (hd.kind == kKindEnd) break;
      const bool up = hd.kind == kKindUp;
      const bool sh = hd.seg == 0;
      const int Iu = sh ? args.Is : args.I;
      const int lw = geo_lw(hd.cls, FP8);
      const int c0 = hd.cp * (up ? lw / 2 : lw);
      const int w = min(up ? lw / 2 : lw, (up ? Iu : H) - c0);
      // local layout of the stage: UP gate [0, w), up [uoff, uoff + w); DOWN [0, w)
      const int uoff = up ? (TMAP ? lw / 2 : w) : 0;
      const int LW = up ? uoff + w : w;
      const int ntiles = (hd.ntok + 7) >> 3;
      if (hd.flags & kFirst) {
#pragma unroll
        for (int i = 0; i < NF; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
      }
      const uint32_t sw = smem_addr(stages + (size_t)slot * kStageBytesMma);
      const uint32_t sx = sw + (FP8 ? fp8_stage_xoff(hd.cls) : kStageWBytes);
      if constexpr (FP8) {
        const float* srow =
            reinterpret_cast<const float*>(stages + (size_t)slot * kStageBytesMma + fp8_stage_wbytes(hd.cls));
        if (hd.cls == 0)
          mma_stage_fp8<0, NF, CW>(acc, sw, sx, srow, LW, hd.nrows, ntiles, up, c0, uoff, Iu, warp, lane);
        else if constexpr (KC >= 1) {
          if (hd.cls == 1)
            mma_stage_fp8<1, NF, CW>(acc, sw, sx, srow, LW, hd.nrows, ntiles, up, c0, uoff, Iu, warp, lane);
          else if constexpr (KC >= 2)
            mma_stage_fp8<2, NF, CW>(acc, sw, sx, srow, LW, hd.nrows, ntiles, up, c0, uoff, Iu, warp, lane);
        }
      } else {
        if (hd.cls == 0)
          mma_stage<0, NF, TMAP, CW>(acc, sw, sx, LW, hd.nrows, ntiles, warp, lane);
        else if constexpr (KC >= 1) {
          if (hd.cls == 1)
            mma_stage<1, NF, TMAP, CW>(acc, sw, sx, LW, hd.nrows, ntiles, warp, lane);
          else if constexpr (KC >= 2)
            mma_stage<2, NF, TMAP, CW>(acc, sw, sx, LW, hd.nrows, ntiles, warp, lane);
        }
      }
      const bool piece_end = (hd.flags & kLast) != 0;
      // What the flush and the SwiGLU fix-up need from the header goes to
      // registers (lane n keeps token n's row and weight), so the slot can be
      // handed back to the producer before the flush: its atomics and fence
      // then overlap the next stages' loads instead of stalling the ring.
      const int ntok = hd.ntok, cls = hd.cls, cp = hd.cp, unit = hd.unit, pstages = hd.pstages;
      const int my_row = lane < ntok ? hd.row[lane] : 0;
      const float my_wt = lane < ntok ? hd.wt[lane] : 0.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);  // release the stage (data and header)
      ++q;
      if (piece_end) {
        // ------------------------------------------- flush the piece's sums
        float* fbase = up ? (sh ? args.h_s : args.h) : args.acc;
        const size_t ld = up ? 2 * (size_t)Iu : (size_t)H;
        if (!warp_aborted(abort_flag)) {
          if (cls == 0)
            flush_piece<0, NF, CW, FP8>(acc, fbase, ld, my_row, my_wt, ntok, up, c0, w, uoff, LW, Iu, warp, lane);
          else if constexpr (KC >= 1) {
            if (cls == 1)
              flush_piece<1, NF, CW, FP8>(acc, fbase, ld, my_row, my_wt, ntok, up, c0, w, uoff, LW, Iu, warp, lane);
            else if constexpr (KC >= 2)
              flush_piece<2, NF, CW, FP8>(acc, fbase, ld, my_row, my_wt, ntok, up, c0, w, uoff, LW, Iu, warp, lane);
          }
        }
        if (up) {
          // ---------------- last warp to finish a panel applies the SwiGLU.
          // Every consumer warp counts its own stages of the piece, so the
          // panel is complete when its counter reaches (stages * CW); no
          // barrier across warps is needed.
          __threadfence();
          __syncwarp();
          unsigned* pcnt = sh ? args.panel_cnt_s : args.panel_cnt;
          unsigned* pready = sh ? args.panel_ready_s : args.panel_ready;
          const int panel = unit * (sh ? args.panel_stride_s : args.panel_stride) + cp;
          const unsigned target = (unsigned)unit_panel_stages(cls, true, H, Iu, FP8) * CW;
          int last = 0;
          if (lane == 0 && !*abort_flag) {
            const unsigned steps = (unsigned)pstages;
            const unsigned old = atomicAdd(&pcnt[panel], steps);
            last = (old + steps == target) ? 1 : 0;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            __threadfence();
            float* hb = sh ? args.h_s : args.h;
            __nv_bfloat16* ab = sh ? args.a_s : args.a;
            const int w4 = w / 4;
            const int total = ntok * w4;
            for (int i0 = 0; i0 < total; i0 += 32) {  // warp-uniform trip count (shuffles inside)
              const int i = i0 + lane;
              const int n = i < total ? i / w4 : 0;
              const int r = __shfl_sync(0xffffffffu, my_row, n);
              if (i >= total) continue;
              const int c = c0 + 4 * (i - n * w4);
              float* hg = hb + (size_t)r * (2 * Iu) + c;
              const float4 g = __ldcg(reinterpret_cast<const float4*>(hg));
              const float4 u = __ldcg(reinterpret_cast<const float4*>(hg + Iu));
              const __nv_bfloat162 lo = __floats2bfloat162_rn(silu_f32(g.x) * u.x, silu_f32(g.y) * u.y);
              const __nv_bfloat162 hi = __floats2bfloat162_rn(silu_f32(g.z) * u.z, silu_f32(g.w) * u.w);
              uint2 pk;
              pk.x = *reinterpret_cast<const uint32_t*>(&lo);
              pk.y = *reinterpret_cast<const uint32_t*>(&hi);
              *reinterpret_cast<uint2*>(ab + (size_t)r * Iu + c) = pk;
              __stcg(reinterpret_cast<float4*>(hg), make_float4(0.f, 0.f, 0.f, 0.f));
              __stcg(reinterpret_cast<float4*>(hg + Iu), make_float4(0.f, 0.f, 0.f, 0.f));
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) {
              pcnt[panel] = 0u;
              if (sh || panel != args.hold_panel) atomicExch(&pready[panel], ready_mark);  // publish after the fence
            }
          }
        }
      }
    }
  }

  // ------------------------------------------------------------------ exit
  __syncthreads();
  if (*abort_flag && tid == 0) {
    // copies still in flight land in this CTA's shared memory: wait for the
    // last NS stages issued (the ring holds no more) before the CTA exits,
    // with the default limit (a copy in flight always lands; the runtime
    // limit may be short)
    const int issued = s_misc[2];
    for (int qq = max(0, issued - NS); qq < issued; ++qq)
      mbar_wait_bounded(&full[qq % NS], (uint32_t)(qq / NS) & 1u, args.status);
  }
  if (tid == 0) {
    // the last CTA out returns the counters to zero and advances the epoch
    __threadfence();
    const unsigned done = atomicAdd(&args.queue[1], 1u);
    s_misc[5] = done == gridDim.x - 1 ? 1 : 0;
    if (done == gridDim.x - 1) {
      __threadfence();
      args.queue[0] = 0u;
      args.queue[1] = 0u;
      args.queue[2] = args.queue[2] + 1u;
      if (args.has_routed) *args.plan_ready = 0;
    }
  }
  __syncthreads();
  if (warp == 0 && s_misc[5] && !*abort_flag) count_stages_at_exit<KC, FP8>(args, sv, lane);
}

}  // namespace moe
