// expert_mma.cuh -- grouped expert SwiGLU MLPs (up + SwiGLU + down) streamed
// from HBM with TMA, multiplied on the tensor cores, in one persistent launch.
//
// Pages: "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and Responsibly"
// (commentary), section "Recovering time between operators": small-batch
// decode waits on weight reads; small-matrix projection kernels at batch 1-2
// and split-K at larger batches expose enough parallel work; weights are
// loaded before their consumer starts, and dependent work should begin as
// soon as its inputs exist.  The pages' kernels were written for GB300 in
// CuTe DSL; this is a B200 design of the same ideas.
//
// What one launch computes (routed: every active expert of the plan; DENSE:
// the shared expert over all tokens, weight 1):
//   UP   h[slot, :] = x[tok, :] . W13[e]           (fp32, split-K partial sums)
//        a[slot, c] = bf16(silu(h[slot, c]) * h[slot, I + c])  per panel, once complete
//   DOWN acc[tok, :] += w_slot * a[slot, :] . W2[e] (fp32 atomics)
//
// Panels.  Each matrix is cut into column panels and K-row stages.  A
// consumer thread keeps at most 128 fp32 accumulators, so panel columns x
// token tiles is bounded: a unit (expert) with n tokens uses the widest panel
// its token count allows --
//   class 0: n <=  8 : 2048 local columns, 16-row stages (1 token tile, 64 accumulators)
//   class 1: n <= 16 : 2048 local columns, 16-row stages (2 token tiles)
//   class 2: n <= 32 : 1024 local columns, 32-row stages (4 token tiles)
//   class 3: n <= 64 :  512 local columns, 64-row stages (8 token tiles)
// -- every stage is 64 KB of weights.  A launch is compiled for the largest
// class its batch can produce (KC), so batches of <= 8 tokens run code that
// holds only 64 accumulators.  Wide panels matter because the TMA
// engine pays per copy: a stage is one bulk copy per panel row (two for UP,
// whose panels pair gate columns [c0, c0+LW/2) with up columns [I+c0, ...),
// so a panel holds both halves of its SwiGLU), and rows of 2-4 KB stream at
// full HBM rate where 0.5-1 KB rows do not.
//
// Work list.  [UP stages of every unit, then DOWN stages of every unit]; CTAs
// pull chunks from a global ticket counter.  Ticket i maps to a fixed range:
// the first three quarters of the list go out in chunks of T/(4G) stages (at
// most 64), the rest one stage at a time, so the grid needs no co-residency
// and ends with a tail of about one stage.  A DOWN stage reads rows
// [row0, row0 + R) of the unit's activations, which one UP panel produces;
// it is issued once that panel is published (a per-panel flag holding the
// launch epoch, so flags never need clearing).  Every UP stage was handed out
// before any DOWN stage, so the CTAs that still owe UP work are running and
// the wait always ends (it is bounded all the same).
//
// Data movement.  One producer warp fills a shared-memory ring of 64 KB
// stages, guarded by mbarriers, with TMA (no multicast, L2 evict-first):
//  * tensor-map path (hidden and intermediate sizes multiples of 64): each
//    expert matrix has a tensor map over the 3-D view {64 columns, rows,
//    column chunks of 64}; one tiled load moves a {64, 16, 4} box (16 rows x
//    256 columns, 8 KB) with 128-byte swizzling, so a stage takes 8 loads and
//    the swizzle makes the ldmatrix reads conflict-free.  The TMA engine pays
//    a fixed cost per operation, so few large loads keep it ahead of HBM.
//  * row-copy path (other shapes): one cp.async.bulk per panel row (two for
//    UP), into rows padded by 16 bytes for the same reason.
// Plus one small copy per token of the stage's activations (x for UP, bf16 a
// for DOWN), all counted on the stage's mbarrier, and a stage header.  Eight consumer warps split
// the panel's columns and run mma.sync.m16n8k16 (bf16 in, fp32 accumulate)
// with the tokens as the N dimension, so the tensor cores do the arithmetic
// and the consumers stay far ahead of HBM.  Partial sums of a piece
// (consecutive stages of one panel) are flushed with fp32 atomics; for UP the
// last warp to contribute to a panel (per-panel counter of warp-stages)
// applies the SwiGLU, returns its accumulators to zero and publishes the
// panel to DOWN.  The consumer loop has no CTA-wide barrier, so a warp whose
// bounded wait gives up can never leave another warp blocked.
//
// Ordering under programmatic dependent launch: the plan, activations and
// workspace are read only after the grid-dependency wait.
#pragma once

#include "moe_device.cuh"

namespace moe {

constexpr int kMaxTok = 64;
constexpr int kNumClasses = 4;
__host__ __device__ constexpr int class_lw(int c) { return c <= 1 ? 2048 : (c == 2 ? 1024 : 512); }
__host__ __device__ constexpr int class_rows(int c) { return c <= 1 ? 16 : (c == 2 ? 32 : 64); }
__host__ __device__ constexpr int class_nt(int c) { return c == 0 ? 1 : (c == 1 ? 2 : (c == 2 ? 4 : 8)); }
__host__ __device__ constexpr int class_for_tokens(int n) { return n <= 8 ? 0 : (n <= 16 ? 1 : (n <= 32 ? 2 : 3)); }
// Consumer warps of the instance compiled for classes <= kc: sixteen when a
// thread needs only 32 accumulators (more warps hide more latency), eight
// otherwise -- nine warps per CTA leave each thread 168 registers, enough for
// 128 accumulators, where seventeen warps cap it at 96.
__host__ __device__ constexpr int consumer_warps_for(int kc) { return kc == 0 ? 16 : 8; }
__host__ __device__ constexpr int expert_threads(int kc) { return (consumer_warps_for(kc) + 1) * 32; }
// m-tiles (16 columns) per consumer warp for class c with cw consumer warps
__host__ __device__ constexpr int class_mt(int c, int cw) { return class_lw(c) / (cw * 16); }
// accumulator fragments (of 4 floats) a consumer thread needs for classes <= KC
__host__ __device__ constexpr int acc_frags(int kc) {
  return kc == 0 ? class_mt(0, consumer_warps_for(0)) * class_nt(0)
                 : class_mt(1, consumer_warps_for(kc)) * class_nt(1);
}
constexpr int kStageWBytes = 65536 + 64 * 16;              // rows * (2*LW + 16), largest over classes
constexpr int kStageXBytes = kMaxTok * (64 * 2 + 16);      // tokens * (2*rows + 16), largest
constexpr int kStageBytesMma = kStageWBytes + kStageXBytes;  // 75776
constexpr int kMaxStagesMma = 3;
constexpr int kMaxChunk = 64;  // stages per queue grab, at most
// tensor-map path: boxes of {64 columns, 16 rows, 4 column chunks}
constexpr int kChunkCols = 64;
constexpr int kBoxRows = 16;
constexpr int kBoxChunks = 4;
constexpr int kChunkTile = kBoxRows * kChunkCols * 2;          // 2048 B: one chunk of one 16-row block
constexpr int kBoxBytes = kChunkTile * kBoxChunks;               // 8192 B per load
constexpr int kTensorMapBytes = 128;
// UP panels of a unit, at most: ceil(I / 256) (class 3); sizes the panel counters
__host__ __device__ inline int max_up_panels(int I) { return (I + class_lw(3) / 2 - 1) / (class_lw(3) / 2); }

enum : int { kKindUp = 0, kKindDown = 1, kKindEnd = 2 };
enum : int { kFirst = 1, kLast = 2 };

// Stage header, written by the producer before it arms the stage's barrier.
// row[n]: UP -> the h/a row (assignment slot) of token n of the unit;
//         DOWN -> the output row (token).  wt[n]: DOWN routing weight.
struct StageHdr {
  int kind, unit, cls, cp, row0, nrows, flags, ntok, begin, pstages;  // pstages: stages of the piece (on its last)
  int row[kMaxTok];
  float wt[kMaxTok];
};

struct MmaArgs {
  int H;             // hidden (UP rows, DOWN columns)
  int I;             // intermediate (UP columns per half, DOWN rows)
  int n_stages;      // ring depth
  int batch;         // tokens (DENSE)
  int max_units;     // bound on the plan's n_active
  int panel_stride;  // panel counters per unit (max_up_panels(I))
  const __nv_bfloat16* w13;  // DENSE weights; routed experts come from the pointer tables
  const __nv_bfloat16* w2;
  const uint8_t* maps13;     // tensor-map path: [units] 128-byte maps of w13 (DENSE: one)
  const uint8_t* maps2;      // tensor-map path: maps of w2
  const Plan* plan;          // nullptr for DENSE
  const __nv_bfloat16* x;    // [B, H]
  float* h;                  // [slots, 2I] fp32, zero between calls
  __nv_bfloat16* a;          // [slots, I] bf16
  float* acc;                // [B, H] fp32 output accumulator
  unsigned* panel_cnt;       // [units * panel_stride] finished warp-stages per UP panel, zero between calls
  unsigned* panel_ready;     // [units * panel_stride] = epoch + 1 once the UP panel's activations are written
  unsigned* queue;           // [0] ticket counter, [1] finished CTAs (zero between calls), [2] launch epoch
  int* status;
};

__host__ __device__ inline size_t mma_smem_bytes(int n_stages) {
  // + 1 KB so the ring can start on a 1024-byte boundary (128-byte swizzle)
  return 1024 + (size_t)n_stages * kStageBytesMma + 2 * kMaxStagesMma * sizeof(uint64_t) +
         kMaxStagesMma * sizeof(StageHdr) + 16 * sizeof(int);
}

// Panels and stages per panel of one unit with class `cls`, UP or DOWN list.
__device__ __forceinline__ int unit_panels(int cls, bool up, int H, int I) {
  const int lw = class_lw(cls);
  return up ? (I + lw / 2 - 1) / (lw / 2) : (H + lw - 1) / lw;
}
__device__ __forceinline__ int unit_panel_stages(int cls, bool up, int H, int I) {
  const int r = class_rows(cls);
  return up ? (H + r - 1) / r : (I + r - 1) / r;
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
    // token fragments: kept for all tiles when there are few of them, loaded
    // per m-tile otherwise (keeps the 64 accumulators in registers)
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

// Flush this warp's partial sums of a piece (class C) with fp32 atomics.
// Local columns: DOWN [0, w) -> c0 + l; UP gate [0, w) -> c0 + l and up
// [uoff, uoff + w) -> I + c0 + (l - uoff); anything else is padding.  w and
// uoff are multiples of 8, so four consecutive local columns map to four
// consecutive output columns.
__device__ __forceinline__ int local_to_col(int l, bool up, int c0, int w, int uoff, int I) {
  if (!up) return l < w ? c0 + l : -1;
  if (l < w) return c0 + l;
  if (l >= uoff && l < uoff + w) return I + c0 + (l - uoff);
  return -1;
}

// Flush this warp's partial sums of a piece (class C) with fp32 atomics.  An
// m-tile's C fragment spreads 16 columns of a token over 8 lanes; shuffles
// gather each run of 4 columns into one lane, so every 16 bytes take one
// vector atomic instead of four scalar ones.
template <int C, int NF, int CW>
__device__ __forceinline__ void flush_piece(const float (&acc)[NF][4], const MmaArgs& args, const StageHdr& hd,
                                            bool up, int c0, int w, int uoff, int LW, int warp, int lane) {
  constexpr int MT = class_mt(C, CW), NT = class_nt(C);
  const int m0 = warp * MT * 16;
  if (m0 >= LW) return;
  const int gid = lane >> 2, tig = lane & 3;
  const int I = args.I, H = args.H;
  const int ntiles = (hd.ntok + 7) >> 3;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    if (nt >= ntiles) break;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int n = nt * 8 + tig * 2 + e;  // this lane's token (same for its tig group)
      const bool valid = n < hd.ntok;
      float* row = nullptr;
      float wt = 1.f;
      if (valid) {
        const int r = hd.row[n];
        wt = up ? 1.f : hd.wt[n];
        row = up ? args.h + (size_t)r * (2 * I) : args.acc + (size_t)r * H;
      }
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        if (m0 + mt * 16 >= LW) break;
        const float v_lo = acc[mt * NT + nt][e];      // column gid
        const float v_hi = acc[mt * NT + nt][2 + e];  // column gid + 8
        // lane with gid < 4 collects columns 4*gid .. 4*gid + 3 of its token
        float o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int c = 4 * (gid & 3) + j;
          const int src = ((c & 7) << 2) | tig;
          const float a = __shfl_sync(0xffffffffu, v_lo, src);
          const float b = __shfl_sync(0xffffffffu, v_hi, src);
          o[j] = c < 8 ? a : b;
        }
        if (valid && gid < 4) {
          const int col = local_to_col(m0 + mt * 16 + 4 * gid, up, c0, w, uoff, I);
          if (col >= 0)
            atomicAdd(reinterpret_cast<float4*>(row + col), make_float4(wt * o[0], wt * o[1], wt * o[2], wt * o[3]));
        }
      }
    }
  }
}

template <bool DENSE, int KC, bool TMAP>
__global__ void __launch_bounds__(expert_threads(KC), 1)
    expert_mlp_kernel(const __grid_constant__ MmaArgs args, const __grid_constant__ ExpertTable tab13,
                      const __grid_constant__ ExpertTable tab2) {
  extern __shared__ __align__(1024) uint8_t mma_smem[];
  const int NS = args.n_stages;
  // the ring starts on a 1024-byte boundary (128-byte swizzle atoms)
  uint8_t* stages = mma_smem + ((1024u - (smem_addr(mma_smem) & 1023u)) & 1023u);
  uint64_t* full = reinterpret_cast<uint64_t*>(stages + (size_t)NS * kStageBytesMma);
  uint64_t* empty = full + kMaxStagesMma;
  StageHdr* hdr = reinterpret_cast<StageHdr*>(empty + kMaxStagesMma);
  volatile int* s_misc = reinterpret_cast<volatile int*>(hdr + kMaxStagesMma);
  // s_misc[0]: abort flag (a bounded wait gave up), [2]: stages issued

  constexpr int CW = consumer_warps_for(KC);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_producer = (warp == CW);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], CW);
    }
    s_misc[0] = 0;
    s_misc[2] = 0;
    mbar_fence_init();
  }
  __syncthreads();

  const int H = args.H, I = args.I;
  volatile int* abort_flag = s_misc;
  const Plan* plan = args.plan;
  // Launch epoch: advanced by the last CTA of the previous launch (an earlier
  // grid on this stream), so every CTA of this launch reads the same value.

  if (is_producer) {
    // ================================================================ producer
    const uint64_t pol = l2_evict_first_policy();
    // The first ticket only touches this kernel's own counter (returned to
    // zero by the previous launch of this kernel, which finished before the
    // router started), so take it before the wait: its round trip overlaps
    // the router's tail.  It is turned into a range only after the wait.
    int tk = 0;
    if (lane == 0) tk = (int)atomicAdd(&args.queue[0], 1u);
    cudaGridDependencySynchronize();  // the plan and the activations come from earlier kernels
    const unsigned ready_mark = __ldcg(&args.queue[2]) + 1u;
    int n_units = 1;
    if (!DENSE) {
      n_units = plan->n_active;
      if (n_units < 0 || n_units > args.max_units) {
        if (lane == 0) atomicCAS(args.status, kStatusOk, kStatusPlan);
        n_units = 0;
      }
    }
    auto unit_tokens = [&](int u) {
      const int n = DENSE ? args.batch : plan->unit_count[u];
      return n > kMaxTok ? kMaxTok : n;  // cannot exceed: batch <= 64
    };
    auto unit_class = [&](int n) {
      const int c = class_for_tokens(n);
      return c > KC ? KC : c;  // cannot exceed: KC is the class of the batch size
    };
    auto unit_stages = [&](int u, bool up) {
      const int c = unit_class(unit_tokens(u));
      return unit_panels(c, up, H, I) * unit_panel_stages(c, up, H, I);
    };
    int T_up = 0, T_dn = 0;  // at most ~1.5M stages: 32-bit arithmetic
    for (int u = lane; u < n_units; u += 32) {
      T_up += unit_stages(u, true);
      T_dn += unit_stages(u, false);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      T_up += __shfl_xor_sync(0xffffffffu, T_up, off);
      T_dn += __shfl_xor_sync(0xffffffffu, T_dn, off);
    }
    const int T_all = T_up + T_dn;
    const int G = gridDim.x;
    // ticket -> range: 3/4 of the list in chunks of c_big, then 3/16 in
    // chunks of c_big / 4, then single stages
    int c_big = T_all / (4 * G);
    c_big = c_big < 1 ? 1 : (c_big > kMaxChunk ? kMaxChunk : c_big);
    const int c_mid = c_big / 4 < 1 ? 1 : c_big / 4;
    const int n_big = (T_all / 4 * 3) / c_big;
    const int T1 = n_big * c_big;
    const int n_mid = ((T_all - T1) / 4 * 3) / c_mid;
    const int T2 = T1 + n_mid * c_mid;
    auto chunk_of = [&](int tk, int& b, int& e) {
      if (tk < n_big) {
        b = tk * c_big;
        e = b + c_big;
      } else if (tk - n_big < n_mid) {
        b = T1 + (tk - n_big) * c_mid;
        e = b + c_mid;
      } else {
        b = T2 + (tk - n_big - n_mid);
        e = b + 1;
      }
      if (b > T_all) b = T_all;
      if (e > T_all) e = T_all;
    };
    // cursor over the work list (tickets only grow, so it only moves forward).
    // The current unit's description lives in registers -- lane j also keeps
    // the token (UP) or slot (DOWN) of the unit's tokens j and j + 32 -- and is
    // reloaded only when the cursor enters a new unit: with shared memory
    // taking almost all of the SM, L1 is tiny and per-stage plan loads would
    // go to L2 every time.
    bool cur_up = true;
    int cur_unit = 0;
    int cur_base = 0, cur_size = n_units > 0 ? unit_stages(0, true) : 0;
    int u_loaded = -1;
    bool u_loaded_up = true;
    int u_ntok = 0, u_cls = 0, u_lw = 0, u_R = 0, u_S = 0, u_begin = 0, u_row0 = 0, u_row1 = 0;
    int u_out0 = 0, u_out1 = 0;  // flush rows of tokens lane, lane + 32
    float u_w0 = 1.f, u_w1 = 1.f;
    const __nv_bfloat16* u_W = nullptr;
    const uint8_t* u_map = nullptr;
    uint32_t q = 0;
    int ready_panel = -1;  // last (unit, UP panel) seen published
    tk = __shfl_sync(0xffffffffu, tk, 0);
    while (true) {
      int c_beg, c_end;
      chunk_of(tk, c_beg, c_end);
      if (c_beg >= T_all || *abort_flag) break;
      int tk_next = 0;  // next ticket now: its latency overlaps this chunk
      if (lane == 0) tk_next = (int)atomicAdd(&args.queue[0], 1u);
      int piece_start = c_beg;
      bool stop = false;
      for (int t = c_beg; t < c_end; ++t, ++q) {
        while (t >= cur_base + cur_size) {
          cur_base += cur_size;
          if (++cur_unit == n_units) {
            cur_unit = 0;
            cur_up = false;
          }
          cur_size = unit_stages(cur_unit, cur_up);
        }
        const bool up = cur_up;
        const int unit = cur_unit;
        if (unit != u_loaded || up != u_loaded_up) {
          u_loaded = unit;
          u_loaded_up = up;
          u_ntok = unit_tokens(unit);
          u_cls = unit_class(u_ntok);
          u_lw = class_lw(u_cls);
          u_R = class_rows(u_cls);
          u_S = unit_panel_stages(u_cls, up, H, I);
          const int expert = DENSE ? 0 : plan->unit_expert[unit];
          u_begin = DENSE ? 0 : plan->unit_begin[unit];
          u_W = up ? (DENSE ? args.w13 : tab13.p[expert]) : (DENSE ? args.w2 : tab2.p[expert]);
          if (TMAP) u_map = (up ? args.maps13 : args.maps2) + (size_t)(DENSE ? 0 : expert) * kTensorMapBytes;
          // per token: the row its activations are read from (x row for UP,
          // a row for DOWN) and the row its partial sums go to (h row for UP,
          // output row for DOWN) with the routing weight
          u_row0 = u_row1 = u_out0 = u_out1 = 0;
          u_w0 = u_w1 = 1.f;
          if (lane < u_ntok) {
            const int tk0 = DENSE ? lane : plan->assign_tok[u_begin + lane];
            const int sl0 = DENSE ? lane : plan->assign_slot[u_begin + lane];
            u_row0 = up ? tk0 : sl0;
            u_out0 = up ? sl0 : tk0;
            if (!DENSE && !up) u_w0 = plan->assign_w[u_begin + lane];
          }
          if (lane + 32 < u_ntok) {
            const int tk1 = DENSE ? lane + 32 : plan->assign_tok[u_begin + lane + 32];
            const int sl1 = DENSE ? lane + 32 : plan->assign_slot[u_begin + lane + 32];
            u_row1 = up ? tk1 : sl1;
            u_out1 = up ? sl1 : tk1;
            if (!DENSE && !up) u_w1 = plan->assign_w[u_begin + lane + 32];
          }
        }
        const int ntok = u_ntok, cls = u_cls, lw = u_lw, R = u_R, S = u_S, begin = u_begin;
        const int loc = t - cur_base;
        const int cp = loc / S;
        const int st = loc - cp * S;
        if (t == c_beg || st == 0) piece_start = t;
        const bool first = (t == piece_start);
        const bool last = (t == c_end - 1 || st == S - 1);
        const int row0 = st * R;
        const int nrows = min(R, (up ? H : I) - row0);
        // DOWN reads activation rows [row0, row0 + R): wait for the UP panel
        // that produces them (gate columns [p*lw/2, (p+1)*lw/2))
        const int need_panel = up ? -1 : unit * args.panel_stride + row0 / (lw / 2);
        if (!up && need_panel != ready_panel) {
          int ok = 1;
          if (lane == 0) {
            uint32_t it = 0;
            while (ld_acquire_u32(&args.panel_ready[need_panel]) != ready_mark) {
              if (++it > kSpinLimit || *abort_flag) {
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
          ready_panel = need_panel;
        }
        const int slot = q % NS;
        const uint32_t ph = (q / NS) & 1u;
        bool go = mbar_wait_abortable(&empty[slot], ph ^ 1u, args.status, abort_flag) && !*abort_flag;
        go = __all_sync(0xffffffffu, go);
        if (!go) {
          stop = true;
          break;
        }
        const int c0 = cp * (up ? lw / 2 : lw);
        const int w = min(up ? lw / 2 : lw, (up ? I : H) - c0);  // columns per half (UP) or panel (DOWN)
        const uint32_t wbytes = (uint32_t)w * 2;
        const uint32_t pitch = (uint32_t)lw * 2 + 16, xpitch = (uint32_t)R * 2 + 16;
        // tensor-map path: loads = halves x 16-row blocks x groups of 4 chunks
        const int t_ncg = (w / kChunkCols + kBoxChunks - 1) / kBoxChunks;
        const int t_nrb = R / kBoxRows;
        const int t_nops = (up ? 2 : 1) * t_nrb * t_ncg;
        const uint32_t wtotal = TMAP ? (uint32_t)t_nops * kBoxBytes : (uint32_t)nrows * (up ? 2u : 1u) * wbytes;
        const uint32_t bytes = wtotal + (uint32_t)ntok * nrows * 2;
        uint8_t* sw = stages + (size_t)slot * kStageBytesMma;
        uint8_t* sx = sw + kStageWBytes;
        StageHdr& hd = hdr[slot];
        if (lane < ntok) {
          hd.row[lane] = u_out0;
          hd.wt[lane] = u_w0;
        }
        if (lane + 32 < ntok) {
          hd.row[lane + 32] = u_out1;
          hd.wt[lane + 32] = u_w1;
        }
        if (lane == 0) {
          hd.kind = up ? kKindUp : kKindDown;
          hd.unit = unit;
          hd.cls = cls;
          hd.cp = cp;
          hd.row0 = row0;
          hd.nrows = nrows;
          hd.flags = (first ? kFirst : 0) | (last ? kLast : 0);
          hd.ntok = ntok;
          hd.begin = begin;
          hd.pstages = t - piece_start + 1;
        }
        __syncwarp();  // every lane's header writes precede lane 0's (releasing) arrive
        if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
        __syncwarp();
        const __nv_bfloat16* W = u_W;
        if (TMAP) {
          const int per_half = t_nrb * t_ncg;
          const int rbstride = (lw / kChunkCols) * kChunkTile;
          const int nch_half = (up ? lw / 2 : lw) / kChunkCols;
          for (int o = lane; o < t_nops; o += 32) {
            const int hh = o / per_half, rem = o - hh * per_half;
            const int rb = rem / t_ncg, cg = rem - rb * t_ncg;
            uint8_t* dst = sw + (size_t)rb * rbstride + (size_t)(hh * nch_half + cg * kBoxChunks) * kChunkTile;
            const int col0 = up ? (hh ? I + c0 : c0) : c0;
            tma_load_3d(dst, u_map, 0, row0 + rb * kBoxRows, col0 / kChunkCols + cg * kBoxChunks, &full[slot], pol);
          }
        }
        if (TMAP) {
          // activations only (the weights went above)
          if (lane < ntok)
            bulk_copy_g2s_plain(sx + (size_t)lane * xpitch, (up ? (const void*)(args.x + (size_t)u_row0 * H + row0)
                                                                : (const void*)(args.a + (size_t)u_row0 * I + row0)),
                                (uint32_t)nrows * 2, &full[slot]);
          if (lane + 32 < ntok)
            bulk_copy_g2s_plain(sx + (size_t)(lane + 32) * xpitch,
                                (up ? (const void*)(args.x + (size_t)u_row1 * H + row0)
                                    : (const void*)(args.a + (size_t)u_row1 * I + row0)),
                                (uint32_t)nrows * 2, &full[slot]);
        } else if (up) {
          for (int r = lane; r < nrows; r += 32) {
            const __nv_bfloat16* src = W + (size_t)(row0 + r) * (2 * I) + c0;
            uint8_t* d = sw + (size_t)r * pitch;
            bulk_copy_g2s(d, src, wbytes, &full[slot], pol);
            bulk_copy_g2s(d + wbytes, src + I, wbytes, &full[slot], pol);
          }
          if (lane < ntok)
            bulk_copy_g2s_plain(sx + (size_t)lane * xpitch, args.x + (size_t)u_row0 * H + row0, (uint32_t)nrows * 2,
                                &full[slot]);
          if (lane + 32 < ntok)
            bulk_copy_g2s_plain(sx + (size_t)(lane + 32) * xpitch, args.x + (size_t)u_row1 * H + row0,
                                (uint32_t)nrows * 2, &full[slot]);
        } else {
          for (int r = lane; r < nrows; r += 32)
            bulk_copy_g2s(sw + (size_t)r * pitch, W + (size_t)(row0 + r) * H + c0, wbytes, &full[slot], pol);
          if (lane < ntok)
            bulk_copy_g2s_plain(sx + (size_t)lane * xpitch, args.a + (size_t)u_row0 * I + row0, (uint32_t)nrows * 2,
                                &full[slot]);
          if (lane + 32 < ntok)
            bulk_copy_g2s_plain(sx + (size_t)(lane + 32) * xpitch, args.a + (size_t)u_row1 * I + row0,
                                (uint32_t)nrows * 2, &full[slot]);
        }
        if (lane == 0) s_misc[2] = (int)(q + 1);
      }
      if (stop) break;
      tk = __shfl_sync(0xffffffffu, tk_next, 0);
    }
    // tell the consumers there is no more work (after an abort they stop on
    // their own: their waits give up once the abort flag is set)
    const int slot = q % NS;
    const uint32_t ph = (q / NS) & 1u;
    mbar_wait_abortable(&empty[slot], ph ^ 1u, args.status, abort_flag);
    if (lane == 0) {
      hdr[slot].kind = kKindEnd;
      mbar_arrive(&full[slot]);
    }
  } else {
    // =============================================================== consumers
    cudaGridDependencySynchronize();
    const unsigned ready_mark = __ldcg(&args.queue[2]) + 1u;
    constexpr int NF = acc_frags(KC);
    float acc[NF][4];
    uint32_t q = 0;
    while (true) {
      const int slot = q % NS;
      const uint32_t ph = (q / NS) & 1u;
      const bool landed = mbar_wait_abortable(&full[slot], ph, args.status, abort_flag);
      // the header stays valid until this warp releases the slot (below,
      // after any flush that reads its token rows)
      const StageHdr& hd = hdr[slot];
      if (!landed || hd.kind == kKindEnd) break;
      const bool up = hd.kind == kKindUp;
      const int lw = class_lw(hd.cls);
      const int c0 = hd.cp * (up ? lw / 2 : lw);
      const int w = min(up ? lw / 2 : lw, (up ? I : H) - c0);
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
      const uint32_t sx = sw + kStageWBytes;
      if (hd.cls == 0)
        mma_stage<0, NF, TMAP, CW>(acc, sw, sx, LW, hd.nrows, ntiles, warp, lane);
      else if constexpr (KC >= 1) {
        if (hd.cls == 1)
          mma_stage<1, NF, TMAP, CW>(acc, sw, sx, LW, hd.nrows, ntiles, warp, lane);
        else if constexpr (KC >= 2) {
          if (hd.cls == 2)
            mma_stage<2, NF, TMAP, CW>(acc, sw, sx, LW, hd.nrows, ntiles, warp, lane);
          else if constexpr (KC >= 3)
            mma_stage<3, NF, TMAP, CW>(acc, sw, sx, LW, hd.nrows, ntiles, warp, lane);
        }
      }
      if (hd.flags & kLast) {
        // ------------------------------------------- flush the piece's sums
        if (!*abort_flag) {
          if (hd.cls == 0)
            flush_piece<0, NF, CW>(acc, args, hd, up, c0, w, uoff, LW, warp, lane);
          else if constexpr (KC >= 1) {
            if (hd.cls == 1)
              flush_piece<1, NF, CW>(acc, args, hd, up, c0, w, uoff, LW, warp, lane);
            else if constexpr (KC >= 2) {
              if (hd.cls == 2)
                flush_piece<2, NF, CW>(acc, args, hd, up, c0, w, uoff, LW, warp, lane);
              else if constexpr (KC >= 3)
                flush_piece<3, NF, CW>(acc, args, hd, up, c0, w, uoff, LW, warp, lane);
            }
          }
        }
        if (up) {
          // ---------------- last warp to finish a panel applies the SwiGLU.
          // Every consumer warp counts its own stages of the piece, so the
          // panel is complete when its counter reaches (stages * CW); no
          // barrier across warps is needed.
          __threadfence();
          __syncwarp();
          const int panel = hd.unit * args.panel_stride + hd.cp;
          const unsigned target = (unsigned)unit_panel_stages(hd.cls, true, H, I) * CW;
          int last = 0;
          if (lane == 0 && !*abort_flag) {
            const unsigned steps = (unsigned)hd.pstages;
            const unsigned old = atomicAdd(&args.panel_cnt[panel], steps);
            last = (old + steps == target) ? 1 : 0;
          }
          last = __shfl_sync(0xffffffffu, last, 0);
          if (last) {
            __threadfence();
            const int w4 = w / 4;
            const int total = hd.ntok * w4;
            for (int i = lane; i < total; i += 32) {
              const int n = i / w4;
              const int c = c0 + 4 * (i - n * w4);
              const int slot_id = hd.row[n];
              float* hg = args.h + (size_t)slot_id * (2 * I) + c;
              const float4 g = __ldcg(reinterpret_cast<const float4*>(hg));
              const float4 u = __ldcg(reinterpret_cast<const float4*>(hg + I));
              const __nv_bfloat162 lo = __floats2bfloat162_rn(silu_f32(g.x) * u.x, silu_f32(g.y) * u.y);
              const __nv_bfloat162 hi = __floats2bfloat162_rn(silu_f32(g.z) * u.z, silu_f32(g.w) * u.w);
              uint2 pk;
              pk.x = *reinterpret_cast<const uint32_t*>(&lo);
              pk.y = *reinterpret_cast<const uint32_t*>(&hi);
              *reinterpret_cast<uint2*>(args.a + (size_t)slot_id * I + c) = pk;
              __stcg(reinterpret_cast<float4*>(hg), make_float4(0.f, 0.f, 0.f, 0.f));
              __stcg(reinterpret_cast<float4*>(hg + I), make_float4(0.f, 0.f, 0.f, 0.f));
            }
            __threadfence();
            __syncwarp();
            if (lane == 0) {
              args.panel_cnt[panel] = 0u;
              atomicExch(&args.panel_ready[panel], ready_mark);  // publish after the fence above
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);  // release the stage (data and header)
      ++q;
    }
  }

  // ------------------------------------------------------------------ exit
  __syncthreads();
  if (*abort_flag && tid == 0) {
    const int issued = s_misc[2];
    for (int qq = max(0, issued - NS); qq < issued; ++qq)
      mbar_wait_bounded(&full[qq % NS], (uint32_t)(qq / NS) & 1u, args.status);
  }
  if (tid == 0) {
    // the last CTA out returns the counters to zero and advances the epoch
    __threadfence();
    const unsigned done = atomicAdd(&args.queue[1], 1u);
    if (done == gridDim.x - 1) {
      __threadfence();
      args.queue[0] = 0u;
      args.queue[1] = 0u;
      args.queue[2] = args.queue[2] + 1u;
    }
  }
}

}  // namespace moe
