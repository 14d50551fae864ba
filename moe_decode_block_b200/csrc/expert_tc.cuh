// expert_tc.cuh -- the expert kernel on the 5th-generation tensor cores:
// tcgen05.mma with the accumulators in tensor memory (TMEM).
//
// Same work list, stage ring and producer as expert_mlp_kernel (see
// expert_mma.cuh); what changes is how a stage is multiplied.  There the 8-16
// consumer warps ran mma.sync with the partial sums in registers, so every
// stage cost each warp its tensor-core work plus a flush of its registers at
// the end of a piece, and a stage's slot stayed taken until the slowest warp
// was done.  Here:
//   * one MMA warp stages the tokens' activations in the canonical K-major
//     layout and one thread issues the stage's tcgen05.mma instructions
//     (M = 128 weight columns, N = the unit's tokens rounded up to 16 or 32,
//     K = 16 rows), accumulating in TMEM; tcgen05.commit hands the stage's slot back
//     to the producer as soon as the tensor cores have read it;
//   * four epilogue warps drain a finished piece from TMEM (tcgen05.ld: TMEM
//     lane = weight column, so a warp's 32 lanes are 32 consecutive output
//     columns and its reductions coalesce), while the next piece accumulates
//     in the other half of TMEM (two accumulator buffers of 256 columns).
// The weights are the A operand, read straight from the TMA stage: the
// tensor-map boxes (64 columns x 16 rows with 128-byte swizzle) are the
// canonical MN-major 128-byte-swizzled layout (64-column blocks 2 KB apart,
// 8-row groups 1 KB apart).  Tokens are the B operand.
#pragma once

#include "expert_mma.cuh"

namespace moe {

constexpr int kTcThreads = 6 * 32;      // producer, MMA, 4 epilogue warps
constexpr int kTmemCols = 512;          // two accumulator buffers of 256 columns
constexpr int kTmemBufCols = 256;
constexpr int kTcBBytes = kUnitTok * class_rows(2) * 2;  // B operand: 32 tokens x 64 rows bf16 (largest class)

// Shared memory of expert_tc_kernel: the expert_mlp_kernel layout, then the
// B-operand buffers, two piece descriptors, the accumulator barriers and the
// TMEM base address.
__host__ __device__ inline size_t tc_extra_bytes() {
  return 128 + kMaxStagesMma * (size_t)kTcBBytes + 2 * sizeof(StageHdr) + 8 * sizeof(uint64_t) + 16;
}
__host__ __device__ inline size_t tc_smem_bytes(int n_stages) { return mma_smem_bytes(n_stages) + tc_extra_bytes(); }

// ---- PTX wrappers (sm_100a) ------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] x B[smem desc], kind::f16, one CTA.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  const uint32_t mask0 = 0, mask1 = 0, mask2 = 0, mask3 = 0;  // no output lane disabled
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(mask0), "r"(mask1), "r"(mask2), "r"(mask3)
      : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

// 32 consecutive TMEM columns of this warp's 32 lanes (one lane per thread),
// then wait for the load (the registers are defined only after the wait).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptors (tcgen05): start address, leading and
// stride byte offsets (all >> 4), descriptor version 1, layout type.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
constexpr uint32_t kLayoutNone = 0;
constexpr uint32_t kLayoutSw128 = 2;

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, A (the
// weights) MN-major, B (the tokens) K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t tc_idesc(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

__global__ void __launch_bounds__(kTcThreads, 1)
    expert_tc_kernel(const __grid_constant__ MmaArgs args, const __grid_constant__ ExpertTable tab13,
                     const __grid_constant__ ExpertTable tab2) {
  extern __shared__ __align__(1024) uint8_t mma_smem[];
  const int NS = args.n_stages;
  const SmemView sv = carve_smem(mma_smem, NS);
  uint8_t* stages = sv.stages;
  uint64_t* full = sv.full;
  uint64_t* empty = sv.empty;
  StageHdr* hdr = sv.hdr;
  volatile int* s_misc = sv.s_misc;
  // tc extras after the plan copy
  uint8_t* extra = reinterpret_cast<uint8_t*>(sv.s_ready + kMaxUnits + kMaxSharedUnits);
  extra += (128u - (smem_addr(extra) & 127u)) & 127u;
  uint8_t* sB = extra;                                                        // [NS][kTcBBytes]
  StageHdr* pdesc = reinterpret_cast<StageHdr*>(sB + kMaxStagesMma * kTcBBytes);  // [2]
  uint64_t* acc_full = reinterpret_cast<uint64_t*>(pdesc + 2);                // [2]: commit + descriptor
  uint64_t* acc_empty = acc_full + 2;                                         // [2]: 4 epilogue warps
  uint64_t* mma_done = acc_empty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(mma_done + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);  // tcgen05.commit of the stage's MMAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 2);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(mma_done, 1);
    for (int i = 0; i < 16; ++i) s_misc[i] = 0;
    s_misc[1] = (int)min(args.spin_limit, 0x7fffffffu);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  const int H = args.H;
  volatile int* abort_flag = s_misc;
  const unsigned ready_mark = __ldcg(&args.queue[2]) + 1u;

  if (warp == 0) {
    // ============================================================ producer
    producer_loop<2, true>(args, tab13, tab2, sv, NS, ready_mark, lane);
  } else if (warp == 1) {
    // ================================================================= MMA
    uint32_t q = 0, piece = 0;
    // Tell the epilogue warps there is no more work -- once they are done
    // with the descriptor of the piece that last used buffer b.  If that wait
    // gives up, nothing is posted (the buffer's barrier may still have a
    // phase in flight, and its descriptor may be in use): the epilogue warps
    // stop on the abort flag instead.
    auto post_end = [&](int b) {
      if (mbar_wait_abortable_warp(&acc_empty[b], ((piece >> 1) & 1u) ^ 1u, args.status, abort_flag)) {
        if (lane == 0) pdesc[b].kind = kKindEnd;
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&acc_full[b]);
          mbar_arrive(&acc_full[b]);
        }
      }
      __syncwarp();
    };
    while (true) {
      const int slot = q % NS;
      const uint32_t ph = (q / NS) & 1u;
      // (warp-uniform: everything below is warp-collective)
      const bool landed = mbar_wait_abortable_warp(&full[slot], ph, args.status, abort_flag);
      const int b = piece & 1;
      if (!landed) {
        post_end(b);
        break;
      }
      const StageHdr& hd = hdr[slot];
      if (__shfl_sync(0xffffffffu, hd.kind, 0) == kKindEnd) {
        post_end(b);
        break;
      }
      const bool up = hd.kind == kKindUp;
      const int Iu = hd.seg == 0 ? args.Is : args.I;
      const int cls = hd.cls, ntok = hd.ntok, flags = hd.flags, nrows = hd.nrows;
      const int lw = class_lw(cls), R = class_rows(cls);
      const int c0 = hd.cp * (up ? lw / 2 : lw);
      const int w = min(up ? lw / 2 : lw, (up ? Iu : H) - c0);
      const int uoff = up ? lw / 2 : 0;
      const int N = ntok <= 16 ? 16 : 32;  // M = 128 takes N in multiples of 16
      const int nslots = lw / 128;
      if (cls < 0 || cls > 2 || ntok < 0 || ntok > kUnitTok || nrows < 0 || nrows > R || nslots * N > kTmemBufCols) {
        // a header the producer never writes: stop before touching TMEM
        if (lane == 0) {
          atomicCAS(args.status, kStatusOk, kStatusPlan);
          *abort_flag = 1;
        }
        __syncwarp();
        post_end(b);
        break;
      }
      if (flags & kFirst) {
        // the accumulator buffer must have been drained by the epilogue
        const uint32_t use = piece >> 1;
        if (!mbar_wait_abortable_warp(&acc_empty[b], (use & 1u) ^ 1u, args.status, abort_flag))
          break;  // the abort flag is set: the epilogue warps stop on it
        tc_fence_after();
      }
      // B operand: the stage's token rows (x or a) in the canonical K-major
      // layout without swizzle -- [8-token group][8-row core][8 tokens][16 B]
      // -- with zeros for missing tokens and rows
      const uint32_t xpitch = (uint32_t)R * 2 + 16;
      const uint8_t* sx = stages + (size_t)slot * kStageBytesMma + kStageWBytes;
      uint8_t* bb = sB + (size_t)slot * kTcBBytes;
      const int kc = R / 8;
      for (int it = lane; it < N * kc; it += 32) {
        const int n = it / kc, c = it - n * kc;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (n < ntok && c * 8 < nrows) val = *reinterpret_cast<const uint4*>(sx + (size_t)n * xpitch + c * 16);
        *reinterpret_cast<uint4*>(bb + (size_t)(n >> 3) * (kc * 128) + c * 128 + (n & 7) * 16) = val;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (flags & kLast) {
        // the piece's descriptor for the epilogue, copied from the stage header
        // now: once the commit below hands the slot back, the producer may
        // overwrite the header (the buffer's previous piece was drained before
        // its first stage, so the descriptor slot is free)
        StageHdr& pd = pdesc[b];
        if (lane == 0) {
          pd.kind = hd.kind;
          pd.seg = hd.seg;
          pd.unit = hd.unit;
          pd.cls = cls;
          pd.cp = hd.cp;
          pd.row0 = hd.row0;
          pd.nrows = nrows;
          pd.flags = flags;
          pd.ntok = ntok;
          pd.pstages = hd.pstages;
        }
        if (lane < ntok) {
          pd.row[lane] = hd.row[lane];
          pd.wt[lane] = hd.wt[lane];
        }
      }
      __syncwarp();
      if (lane == 0) {
        tc_fence_after();
        const uint32_t idesc = tc_idesc(N);
        const uint32_t sw = smem_addr(stages + (size_t)slot * kStageBytesMma);
        const uint32_t sbb = smem_addr(bb);
        const uint32_t rbstride = (uint32_t)(lw / kChunkCols) * kChunkTile;
        const uint32_t dbase = tmem + (uint32_t)b * kTmemBufCols;
        for (int s = 0; s < R / 16; ++s) {
          if (s * 16 >= nrows) break;
          const uint64_t bdesc = smem_desc(sbb + (uint32_t)s * 256u, 128u, (uint32_t)kc * 128u, kLayoutNone);
          for (int j = 0; j < nslots; ++j) {
            const int l0 = j * 128;
            const bool valid = up ? (l0 < w || (l0 >= uoff && l0 < uoff + w)) : (l0 < w);
            if (!valid) continue;
            const uint64_t adesc = smem_desc(sw + (uint32_t)s * rbstride + (uint32_t)(2 * j) * kChunkTile,
                                             (uint32_t)kChunkTile, 1024u, kLayoutSw128);
            tc_mma(dbase + (uint32_t)(j * N), adesc, bdesc, idesc, ((flags & kFirst) && s == 0) ? 0u : 1u);
          }
        }
        tc_commit(&empty[slot]);  // the slot is free once these MMAs have read it
      }
      __syncwarp();
      if (flags & kLast) {
        // hand the piece to the epilogue: MMA completion (commit) + the
        // descriptor written above (plain arrive, releasing those writes)
        if (lane == 0) {
          tc_commit(&acc_full[b]);
          mbar_arrive(&acc_full[b]);
        }
        ++piece;
      }
      ++q;
    }
    // every MMA issued has completed before TMEM is released
    if (lane == 0) {
      tc_commit(mma_done);
      mbar_wait_bounded(mma_done, 0u, args.status);
    }
    __syncwarp();
  } else {
    // ============================================================ epilogue
    const int quarter = warp & 3;  // TMEM lanes [32 * quarter, +32) = columns of each 128-wide block
    uint32_t piece = 0;
    while (true) {
      const int b = piece & 1;
      const uint32_t use = piece >> 1;
      // (warp-uniform: tcgen05.ld below is .sync.aligned)
      const bool ok = mbar_wait_abortable_warp(&acc_full[b], use & 1u, args.status, abort_flag);
      tc_fence_after();
      if (!ok) break;
      const StageHdr& pd = pdesc[b];
      if (__shfl_sync(0xffffffffu, pd.kind, 0) == kKindEnd) break;
      const bool up = pd.kind == kKindUp;
      const bool sh = pd.seg == 0;
      const int Iu = sh ? args.Is : args.I;
      const int cls = pd.cls, ntok = pd.ntok, cp = pd.cp, unit = pd.unit, pstages = pd.pstages;
      const int lw = class_lw(cls);
      const int c0 = cp * (up ? lw / 2 : lw);
      const int w = min(up ? lw / 2 : lw, (up ? Iu : H) - c0);
      const int uoff = up ? lw / 2 : 0;
      const int N = ntok <= 16 ? 16 : 32;  // M = 128 takes N in multiples of 16
      const int nslots = lw / 128;
      if (cls < 0 || cls > 2 || ntok < 0 || ntok > kUnitTok || nslots * N > kTmemBufCols) {
        // never written by the MMA warp: keep every TMEM access in range
        if (lane == 0) {
          atomicCAS(args.status, kStatusOk, kStatusPlan);
          *abort_flag = 1;
        }
        break;
      }
      const int my_row = lane < ntok ? pd.row[lane] : 0;
      const float my_wt = lane < ntok ? pd.wt[lane] : 0.f;
      float* fbase = up ? (sh ? args.h_s : args.h) : args.acc;
      const size_t ld = up ? 2 * (size_t)Iu : (size_t)H;
      const uint32_t dbase = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)b * kTmemBufCols;
      const int total = nslots * N;
      for (int cc = 0; cc < total; cc += 32) {
        float v[32];
        tmem_ld32(dbase + (uint32_t)cc, v);
        if (cc + 32 >= total) {
          // the buffer is free for the MMA warp once the last columns are read
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        if (warp_aborted(abort_flag)) continue;
        // column cc + i holds token (cc + i) % N of 128-column block (cc + i) / N
        for (int t = 0; t < N && t < ntok; ++t) {
          const int r = __shfl_sync(0xffffffffu, my_row, t);
          const float wr = __shfl_sync(0xffffffffu, my_wt, t);
          float* row = fbase + (size_t)r * ld;
          const float wt = up ? 1.f : wr;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            if ((cc + i) % N != t) continue;
            const int j = (cc + i) / N;
            const int col = local_to_col(j * 128 + 32 * quarter + lane, up, c0, w, uoff, Iu);
            if (col >= 0) red_add(row + col, wt * v[i]);
          }
        }
      }
      ++piece;
      if (up && !warp_aborted(abort_flag)) {
        // ---------------- last warp to finish a panel applies the SwiGLU
        __threadfence();
        __syncwarp();
        unsigned* pcnt = sh ? args.panel_cnt_s : args.panel_cnt;
        unsigned* pready = sh ? args.panel_ready_s : args.panel_ready;
        const int panel = unit * (sh ? args.panel_stride_s : args.panel_stride) + cp;
        const unsigned target = (unsigned)unit_panel_stages(cls, true, H, Iu) * 4u;
        int last = 0;
        if (lane == 0) {
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
          const int tot = ntok * w4;
          for (int i0 = 0; i0 < tot; i0 += 32) {  // warp-uniform trip count (shuffles inside)
            const int i = i0 + lane;
            const int n = i < tot ? i / w4 : 0;
            const int r = __shfl_sync(0xffffffffu, my_row, n);
            if (i >= tot) continue;
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

  // ------------------------------------------------------------------ exit
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (*abort_flag && tid == 0) {
    // copies still in flight land in this CTA's shared memory (default limit)
    const int issued = s_misc[2];
    for (int qq = max(0, issued - NS); qq < issued; ++qq)
      mbar_wait_bounded(&full[qq % NS], (uint32_t)(qq / NS) & 1u, args.status);
  }
  if (tid == 0) {
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
  if (warp == 0 && s_misc[5] && !*abort_flag) count_stages_at_exit<2, false>(args, sv, lane);
}

}  // namespace moe
