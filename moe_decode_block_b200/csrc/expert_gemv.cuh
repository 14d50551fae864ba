// expert_gemv.cuh -- grouped expert projections, streamed from HBM with TMA.
//
// Pages: "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and Responsibly"
// (commentary), section "Recovering time between operators": small-batch
// decode is weight-read bound, served by small-matrix projection kernels at
// batch 1-2 and split-K at larger batches to expose parallel work; weights
// are loaded before their consumer needs them.  The pages' kernels were
// written for GB300 in CuTe DSL; this is a B200 design of the same idea.
//
// One kernel template serves four launches of a forward:
//   UP   (routed or shared): h[slot, :] += x[tok, rows] . W13[e][rows, panel]
//        and, once every row of a panel is in, a[slot, c] = silu(g) * u
//   DOWN (routed or shared): acc[tok, :] += w_slot * a[slot, rows] . W2[e][rows, panel]
//
// Work decomposition (split-K over a flattened space).  Each unit (an active
// expert, or the shared expert) has n_cp column panels of at most 4096 local
// columns and K rows cut into 64-row steps.  The units' (panel, step) pairs
// are laid end to end and the G CTAs take equal contiguous ranges, so every
// CTA streams the same number of weight bytes whatever the routing (weights
// dominate the traffic).  A CTA keeps fp32 partial sums for one
// (panel, token group) in registers and reduces them into global fp32
// buffers with vector atomics at the end of its piece.  For UP a per-panel
// counter of finished steps elects the last contributor, which applies the
// SwiGLU (gate column c pairs with up column I + c, both in the same panel)
// and returns the accumulators to zero for the next call.
//
// Data movement.  One producer warp issues cp.async.bulk (TMA, no multicast)
// copies of 32 KB stages of the panel rows into an n-stage shared-memory
// ring guarded by mbarriers; 16 consumer warps each own one 16-byte column
// vector (8 bf16 columns) of the panel and accumulate up to TG tokens per
// pass.  Weight copies carry an L2 evict-first hint.
//
// Ordering under programmatic dependent launch: a kernel only reads weights
// before cudaGridDependencySynchronize(); activations, the plan and the
// workspace are read after it.  The shared-expert producer (whose partition
// does not depend on routing) starts streaming weights before the wait.
#pragma once

#include "moe_device.cuh"

namespace moe {

struct GemvArgs {
  const __nv_bfloat16* dense_w;  // shared expert matrix (DENSE); routed: from the ExpertTable
  int K;            // rows of each matrix (H for UP, I for DOWN)
  int N;            // row length in elements (2I for UP, H for DOWN)
  int I;            // UP: gate/up split (= N/2); DOWN: unused
  int panel_w;      // UP: gate columns per panel; DOWN: columns per panel
  int n_cp;         // column panels per unit
  int stage_rows;   // rows per pipeline stage (power of two dividing kStepRows)
  int n_stages;     // pipeline depth (<= kMaxStages)
  int batch;        // tokens (DENSE)
  int max_units;    // upper bound on the plan's n_active (n_experts)
  const Plan* plan;                // routed plan (nullptr for DENSE)
  const __nv_bfloat16* x;          // UP: block input [B, H]
  const float* a_in;               // DOWN: activations [slots, K]
  float* h;                        // UP: fp32 accumulators [slots, 2I], zero between calls
  float* a_out;                    // UP: activations out [slots, I]
  unsigned* counters;              // UP: per-panel finished-step counters, zero between calls
  float* acc;                      // DOWN: fp32 output accumulator [B, H]
  int* status;
};

__host__ __device__ inline size_t gemv_smem_bytes(int n_stages, int TG) {
  return (size_t)n_stages * kStageBytes + 2 * kMaxStages * sizeof(uint64_t) +
         (size_t)kStepRows * TG * sizeof(float) + 16 * sizeof(int);
}

template <int TG, bool DENSE, bool UP>
__global__ void __launch_bounds__(kGemvThreads, 1)
    expert_gemv_kernel(const __grid_constant__ GemvArgs args, const __grid_constant__ ExpertTable tab) {
  extern __shared__ __align__(1024) uint8_t gemv_smem[];
  uint8_t* smem = gemv_smem;
  const int NS = args.n_stages;
  uint8_t* stages = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)NS * kStageBytes);
  uint64_t* empty = full + kMaxStages;
  float* xs = reinterpret_cast<float*>(empty + kMaxStages);  // [kStepRows][TG]
  volatile int* s_misc = reinterpret_cast<volatile int*>(xs + kStepRows * TG);
  // s_misc[0]: abort flag (a bounded wait gave up), s_misc[1]: "this CTA
  // finishes the panel", s_misc[2]: stages issued by the producer

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool is_producer = (warp == kConsumerWarps);

  if (tid == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], kConsumerWarps);
    }
    s_misc[0] = 0;
    s_misc[1] = 0;
    s_misc[2] = 0;
    mbar_fence_init();
  }
  __syncthreads();

  // Weights only before the dependency wait (the shared-expert producer);
  // everything else waits for the previous grid's results to be visible.
  if (!(DENSE && is_producer)) cudaGridDependencySynchronize();
  cudaTriggerProgrammaticLaunchCompletion();

  const Plan* plan = args.plan;
  int n_units = 1;
  if (!DENSE) {
    n_units = plan->n_active;
    if (n_units < 0 || n_units > args.max_units) {
      if (tid == 0) atomicCAS(args.status, kStatusOk, kStatusPlan);
      n_units = 0;
    }
  }
  const int K = args.K, N = args.N, n_cp = args.n_cp, R = args.stage_rows;
  const int S = (K + kStepRows - 1) / kStepRows;
  const long long T = (long long)n_units * n_cp * S;
  const long long t0 = T * blockIdx.x / gridDim.x;
  const long long t1 = T * (blockIdx.x + 1) / gridDim.x;
  const int cols_total = UP ? args.I : N;

  uint32_t q = 0;  // running stage counter (same sequence in producer and consumers)
  volatile int* abort_flag = s_misc;

  float acc[TG][8];

  for (long long t = t0; t < t1;) {
    const int panel = (int)(t / S);
    const int s_beg = (int)(t - (long long)panel * S);
    const long long s_lim = (long long)s_beg + (t1 - t);
    const int s_end = (int)(s_lim < S ? s_lim : (long long)S);
    t += s_end - s_beg;
    const int unit = panel / n_cp, cp = panel - unit * n_cp;
    int expert = 0, begin = 0, ntok = args.batch;
    if (!DENSE) {
      expert = plan->unit_expert[unit];
      begin = plan->unit_begin[unit];
      ntok = plan->unit_count[unit];
    }
    const __nv_bfloat16* W = DENSE ? args.dense_w : tab.p[expert];
    const int c0 = cp * args.panel_w;
    const int w = min(args.panel_w, cols_total - c0);
    const int LW = UP ? 2 * w : w;     // local row width in elements
    const bool full_rows = (LW == N);  // panel rows are whole contiguous rows
    const int n_groups = (ntok + TG - 1) / TG;

    for (int g = 0; g < n_groups; ++g) {
      const int nj = min(TG, ntok - g * TG);
      if (!is_producer) {
#pragma unroll
        for (int j = 0; j < TG; ++j)
#pragma unroll
          for (int c = 0; c < 8; ++c) acc[j][c] = 0.f;
      }
      for (int s = s_beg; s < s_end; ++s) {
        const int r_beg = s * kStepRows, r_end = min(K, r_beg + kStepRows);
        if (is_producer) {
          // ---------------------------------------------------- producer
          const uint64_t pol = l2_evict_first_policy();
          for (int r0 = r_beg; r0 < r_end; r0 += R, ++q) {
            const int nr = min(R, r_end - r0);
            const int slot = q % NS;
            const uint32_t ph = (q / NS) & 1u;
            bool go = mbar_wait_abortable(&empty[slot], ph ^ 1u, args.status, abort_flag) && !*abort_flag;
            go = __all_sync(0xffffffffu, go);
            if (!go) continue;  // aborted: issue nothing more
            const uint32_t bytes = (uint32_t)nr * LW * 2;
            uint8_t* dst = stages + (size_t)slot * kStageBytes;
            if (lane == 0) mbar_arrive_expect_tx(&full[slot], bytes);
            __syncwarp();
            if (full_rows) {
              if (lane == 0) bulk_copy_g2s(dst, W + (size_t)r0 * N, bytes, &full[slot], pol);
            } else {
              for (int r = lane; r < nr; r += 32) {
                const __nv_bfloat16* src = W + (size_t)(r0 + r) * N + c0;
                uint8_t* d = dst + (size_t)r * LW * 2;
                bulk_copy_g2s(d, src, (uint32_t)w * 2, &full[slot], pol);
                if (UP) bulk_copy_g2s(d + (size_t)w * 2, src + args.I, (uint32_t)w * 2, &full[slot], pol);
              }
            }
            if (lane == 0) s_misc[2] = (int)(q + 1);
          }
        } else {
          // ---------------------------------------------------- consumers
          consumer_sync();  // previous chunk's xs reads are done
          const int nvals = (r_end - r_beg) * TG;
          for (int i = tid; i < nvals; i += kConsumerThreads) {
            const int rr = i / TG, j = i - rr * TG;
            float v = 0.f;
            if (j < nj) {
              const int idx = g * TG + j;
              if (UP) {
                const int tok = DENSE ? idx : plan->assign_tok[begin + idx];
                v = __bfloat162float(args.x[(size_t)tok * K + r_beg + rr]);
              } else {
                const int slot_id = DENSE ? idx : plan->assign_slot[begin + idx];
                v = args.a_in[(size_t)slot_id * K + r_beg + rr];
              }
            }
            xs[i] = v;
          }
          consumer_sync();
          const bool active = tid * 8 < LW;
          for (int r0 = r_beg; r0 < r_end; r0 += R, ++q) {
            const int nr = min(R, r_end - r0);
            const int slot = q % NS;
            const uint32_t ph = (q / NS) & 1u;
            const bool landed = mbar_wait_abortable(&full[slot], ph, args.status, abort_flag);
            if (active && landed) {
              const uint8_t* st = stages + (size_t)slot * kStageBytes + (size_t)tid * 16;
              const float* xr = xs + (r0 - r_beg) * TG;
#pragma unroll 4
              for (int r = 0; r < nr; ++r) {
                const uint4 wv = *reinterpret_cast<const uint4*>(st + (size_t)r * LW * 2);
                float wf[8];
                bf16x2_to_f32(wv.x, wf[0], wf[1]);
                bf16x2_to_f32(wv.y, wf[2], wf[3]);
                bf16x2_to_f32(wv.z, wf[4], wf[5]);
                bf16x2_to_f32(wv.w, wf[6], wf[7]);
#pragma unroll
                for (int j = 0; j < TG; ++j) {
                  if (j < nj) {
                    const float xv = xr[r * TG + j];
#pragma unroll
                    for (int c = 0; c < 8; ++c) acc[j][c] = fmaf(xv, wf[c], acc[j][c]);
                  }
                }
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[slot]);
          }
        }
      }
      // ------------------------------------------- epilogue of (piece, group)
      if (!is_producer && !*abort_flag && tid * 8 < LW) {
        const int l = tid * 8;
        if (UP) {
          const int col = (l < w) ? c0 + l : args.I + c0 + (l - w);
#pragma unroll
          for (int j = 0; j < TG; ++j) {
            if (j < nj) {
              const int idx = g * TG + j;
              const int slot_id = DENSE ? idx : plan->assign_slot[begin + idx];
              float* dst = args.h + (size_t)slot_id * N + col;
              atomicAdd(reinterpret_cast<float4*>(dst), make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]));
              atomicAdd(reinterpret_cast<float4*>(dst + 4), make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]));
            }
          }
        } else {
          const int col = c0 + l;
#pragma unroll
          for (int j = 0; j < TG; ++j) {
            if (j < nj) {
              const int idx = g * TG + j;
              const int tok = DENSE ? idx : plan->assign_tok[begin + idx];
              const float wt = DENSE ? 1.f : plan->assign_w[begin + idx];
              float* dst = args.acc + (size_t)tok * N + col;
              atomicAdd(reinterpret_cast<float4*>(dst),
                        make_float4(wt * acc[j][0], wt * acc[j][1], wt * acc[j][2], wt * acc[j][3]));
              atomicAdd(reinterpret_cast<float4*>(dst + 4),
                        make_float4(wt * acc[j][4], wt * acc[j][5], wt * acc[j][6], wt * acc[j][7]));
            }
          }
        }
      }
    }

    // ----------------------------------- UP: last contributor applies SwiGLU
    if (UP && !is_producer) {
      __threadfence();
      consumer_sync();
      if (tid == 0) {
        int last = 0;
        if (!*abort_flag) {
          const unsigned steps = (unsigned)(s_end - s_beg);
          const unsigned old = atomicAdd(&args.counters[panel], steps);
          last = (old + steps == (unsigned)S) ? 1 : 0;
        }
        s_misc[1] = last;
      }
      consumer_sync();
      if (s_misc[1]) {
        __threadfence();
        const int w4 = w / 4;
        const int total = ntok * w4;
        for (int i = tid; i < total; i += kConsumerThreads) {
          const int idx = i / w4;
          const int c = c0 + 4 * (i - idx * w4);
          const int slot_id = DENSE ? idx : plan->assign_slot[begin + idx];
          float* hg = args.h + (size_t)slot_id * N + c;
          float* hu = hg + args.I;
          const float4 gv = __ldcg(reinterpret_cast<const float4*>(hg));
          const float4 uv = __ldcg(reinterpret_cast<const float4*>(hu));
          float4 av;
          av.x = silu_f32(gv.x) * uv.x;
          av.y = silu_f32(gv.y) * uv.y;
          av.z = silu_f32(gv.z) * uv.z;
          av.w = silu_f32(gv.w) * uv.w;
          *reinterpret_cast<float4*>(args.a_out + (size_t)slot_id * args.I + c) = av;
          __stcg(reinterpret_cast<float4*>(hg), make_float4(0.f, 0.f, 0.f, 0.f));
          __stcg(reinterpret_cast<float4*>(hu), make_float4(0.f, 0.f, 0.f, 0.f));
        }
        if (tid == 0) args.counters[panel] = 0u;
      }
      consumer_sync();  // s_misc[1] is rewritten by the next panel
    }
  }

  // After an aborted wait, let copies already in flight land before the
  // CTA's shared memory goes away (bounded as well).
  __syncthreads();
  if (*abort_flag && tid == 0) {
    const int issued = s_misc[2];
    for (int qq = max(0, issued - NS); qq < issued; ++qq)
      mbar_wait_bounded(&full[qq % NS], (uint32_t)(qq / NS) & 1u, args.status);
  }
}

// out[t, c] = bf16_rne(x[t, c] + acc[t, c]); acc returns to zero.
__global__ void __launch_bounds__(256) combine_residual_kernel(const __nv_bfloat16* __restrict__ x,
                                                               float* __restrict__ acc,
                                                               __nv_bfloat16* __restrict__ out, int n_vec8) {
  cudaGridDependencySynchronize();
  cudaTriggerProgrammaticLaunchCompletion();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_vec8) return;
  const uint4 xv = reinterpret_cast<const uint4*>(x)[i];
  float4* ap = reinterpret_cast<float4*>(acc) + 2 * (size_t)i;
  const float4 a0 = ap[0], a1 = ap[1];
  float xf[8];
  bf16x2_to_f32(xv.x, xf[0], xf[1]);
  bf16x2_to_f32(xv.y, xf[2], xf[3]);
  bf16x2_to_f32(xv.z, xf[4], xf[5]);
  bf16x2_to_f32(xv.w, xf[6], xf[7]);
  const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  uint32_t o[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(xf[2 * c] + av[2 * c], xf[2 * c + 1] + av[2 * c + 1]);
    o[c] = *reinterpret_cast<const uint32_t*>(&p);
  }
  reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  ap[0] = make_float4(0.f, 0.f, 0.f, 0.f);
  ap[1] = make_float4(0.f, 0.f, 0.f, 0.f);
}

}  // namespace moe
