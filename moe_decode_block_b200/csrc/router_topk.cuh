// router_topk.cuh -- router scores, softmax, top-k, renormalisation and
// token->expert bucketing in one kernel.
//
// Pages: "Hyper Optimizing Kimi K3 in vLLM: Moving Fast and Responsibly"
// (commentary), section "Recovering time between operators": MoE preparation
// computes the router scores for every token; the pages give no formula, the
// reading used here is softmax over all experts, top-k by logit (descending,
// ties to the smaller id) and renormalisation of the selected probabilities.
//
// Structure (one launch, G CTAs):
//   * CTA c owns hidden rows [c*H/G, (c+1)*H/G) of router_w [H, E].  Its slab
//     is staged in shared memory with TMA bulk copies issued *before* the
//     grid-dependency wait (router_w is a static weight, so reading it early
//     under programmatic dependent launch is safe); x is read only after it.
//   * Each thread owns a pair of expert columns and accumulates the partial
//     logits of every token over the slab in fp32; partials are reduced into
//     a global fp32 [B, E] buffer with vector reductions (red, no return).
//   * The last CTA to finish (ticket counter) reads the logits, adds the
//     optional bias, selects the top k per token with warp argmax rounds,
//     computes the renormalised weights, writes topk_ids/topk_w, builds the
//     bucketed plan (experts ascending, assignments sorted by token) and
//     returns the logits buffer and the ticket to zero for the next call.
#pragma once

#include "moe_device.cuh"

namespace moe {

struct RouterArgs {
  const __nv_bfloat16* x;       // [B, H]
  const __nv_bfloat16* router_w;  // [H, E]
  const float* bias;            // [E] or nullptr
  int B, H, E, k;
  int G;                        // grid size
  int chunk_rows;               // rows of router_w staged per bulk copy
  float* logits;                // [B, E] fp32 accumulators, zero between calls
  unsigned* ticket;             // zero between calls
  Plan* plan;
  int32_t* topk_ids;            // [B, k]
  float* topk_w;                // [B, k]
  int* status;
};

// Tokens padded to a multiple of 8 (x is staged token-contiguous per row).
__host__ __device__ inline int router_bpad(int B) { return (B + 7) / 8 * 8; }

// Shared memory needed by router_topk_kernel for these sizes.
__host__ __device__ inline size_t router_smem_bytes(int B, int E, int chunk_rows) {
  size_t gemv = (size_t)chunk_rows * E * 2 + (size_t)router_bpad(B) * chunk_rows * 4;
  size_t topk = (size_t)kMaxAssign * 8 + (size_t)E * 16 + 64;
  gemv = (gemv + 15) / 16 * 16;
  return gemv > topk ? gemv : topk;
}

// Warp-wide argmax with ties to the smaller index.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    float v2 = __shfl_xor_sync(0xffffffffu, v, off);
    int i2 = __shfl_xor_sync(0xffffffffu, i, off);
    if (v2 > v || (v2 == v && i2 < i)) {
      v = v2;
      i = i2;
    }
  }
}

// Exclusive scan of one int per thread over the block (kRouterThreads).
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    int o = __shfl_up_sync(0xffffffffu, inc, off);
    if (lane >= off) inc += o;
  }
  if (lane == 31) warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int t = lane < kRouterThreads / 32 ? warp_tot[lane] : 0;
    int ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int o = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += o;
    }
    if (lane < kRouterThreads / 32) warp_tot[lane] = ti - t;  // exclusive warp offsets
    if (lane == kRouterThreads / 32 - 1) warp_tot[kRouterThreads / 32] = ti;
  }
  __syncthreads();
  const int r = warp_tot[warp] + inc - v;
  total = warp_tot[kRouterThreads / 32];
  __syncthreads();
  return r;
}

// NV: logits per lane a warp holds in registers during top-k (E <= 32 * NV).
template <int NV>
__global__ void __launch_bounds__(kRouterThreads, 1) router_topk_kernel(const __grid_constant__ RouterArgs a) {
  extern __shared__ __align__(1024) uint8_t router_smem[];
  uint8_t* smem = router_smem;
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_last;
  __shared__ int s_warp[kRouterThreads / 32 + 1];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E, B = a.B, H = a.H, k = a.k;
  const int h0 = (int)((long long)H * blockIdx.x / a.G);
  const int h1 = (int)((long long)H * (blockIdx.x + 1) / a.G);
  __nv_bfloat16* rs = reinterpret_cast<__nv_bfloat16*>(smem);
  float* xs = reinterpret_cast<float*>(smem + (((size_t)a.chunk_rows * E * 2 + 15) / 16 * 16));
  const uint64_t pol = l2_evict_first_policy();

  // Stage the first chunk of router_w before waiting on the previous grid.
  if (tid == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
    const int nr = min(a.chunk_rows, h1 - h0);
    if (nr > 0) {
      const uint32_t bytes = (uint32_t)nr * E * 2;
      mbar_arrive_expect_tx(&bar, bytes);
      bulk_copy_g2s(rs, a.router_w + (size_t)h0 * E, bytes, &bar, pol);
    }
  }
  __syncthreads();

  cudaGridDependencySynchronize();
  cudaTriggerProgrammaticLaunchCompletion();

  uint32_t phase = 0;
  const int npairs = E / 2;
  const int bp = router_bpad(B);
  for (int r0 = h0; r0 < h1; r0 += a.chunk_rows) {
    const int nr = min(a.chunk_rows, h1 - r0);
    // x staged as [row][token] (tokens padded to 8 with zeros), so a row's
    // 8-token group is two 16-byte shared loads
    for (int i = tid; i < bp * nr; i += kRouterThreads) {
      const int r = i / bp, t = i - r * bp;
      xs[i] = t < B ? __bfloat162float(a.x[(size_t)t * H + r0 + r]) : 0.f;
    }
    mbar_wait_bounded(&bar, phase, a.status);
    phase ^= 1;
    __syncthreads();
    for (int p = tid; p < npairs; p += kRouterThreads) {
      for (int t0 = 0; t0 < B; t0 += 8) {
        float acc[8][2];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = 0.f;
        const int nt = min(8, B - t0);
#pragma unroll 4
        for (int r = 0; r < nr; ++r) {
          float w0, w1;
          bf16x2_to_f32(reinterpret_cast<const uint32_t*>(rs + (size_t)r * E)[p], w0, w1);
          const float4 xa = *reinterpret_cast<const float4*>(xs + (size_t)r * bp + t0);
          const float4 xb = *reinterpret_cast<const float4*>(xs + (size_t)r * bp + t0 + 4);
          const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            acc[j][0] = fmaf(xv[j], w0, acc[j][0]);
            acc[j][1] = fmaf(xv[j], w1, acc[j][1]);
          }
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < nt)
            red_add_v2(a.logits + (size_t)(t0 + j) * E + 2 * p, acc[j][0], acc[j][1]);
      }
    }
    __syncthreads();
    const int r1 = r0 + a.chunk_rows;
    if (r1 < h1 && tid == 0) {
      const uint32_t bytes = (uint32_t)min(a.chunk_rows, h1 - r1) * E * 2;
      mbar_arrive_expect_tx(&bar, bytes);
      bulk_copy_g2s(rs, a.router_w + (size_t)r1 * E, bytes, &bar, pol);
    }
  }

  // ---- last CTA: top-k, weights, bucketing -------------------------------
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(a.ticket, 1u) == (unsigned)(a.G - 1));
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  int* s_ids = reinterpret_cast<int*>(smem);            // [B*k]
  float* s_w = reinterpret_cast<float*>(s_ids + kMaxAssign);  // [B*k]
  int* s_cnt = reinterpret_cast<int*>(s_w + kMaxAssign);  // [E]
  int* s_off = s_cnt + E;                                 // [E]
  int* s_act = s_off + E;                                 // [E] active index or -1

  const int nv = (E + 31) / 32;
  for (int t = warp; t < B; t += kRouterThreads / 32) {
    float* lg = a.logits + (size_t)t * E;
    float v[NV];
    uint32_t taken = 0;
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int e = lane + 32 * i;
      v[i] = -INFINITY;
      if (i < nv && e < E) {
        v[i] = __ldcg(lg + e) + (a.bias ? a.bias[e] : 0.f);
        __stcg(lg + e, 0.f);
      }
    }
    // each lane keeps its best untaken (value, id); only the lane that owned
    // a round's winner has to look again
    auto local_best = [&](float& bv, int& bi) {
      bv = -INFINITY;
      bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        // e ascends with i, so strict '>' keeps the smaller id on equal logits
        if (i < nv && e < E && !((taken >> i) & 1u) && (bi == 0x7fffffff || v[i] > bv)) {
          bv = v[i];
          bi = e;
        }
      }
    };
    float lbv;
    int lbi;
    local_best(lbv, lbi);
    int my_id = -1;
    float my_v = -INFINITY;
    for (int j = 0; j < k; ++j) {
      float bv = lbv;
      int bi = lbi;
      warp_argmax(bv, bi);
      if (bi < 0 || bi >= E) {  // cannot happen for k <= E; keep the plan valid
        atomicCAS(a.status, kStatusOk, kStatusPlan);
        bi = j;
      }
      if (lane == j) {
        my_id = bi;
        my_v = bv;
      }
      if ((bi & 31) == lane) {
        taken |= 1u << (bi >> 5);
        local_best(lbv, lbi);
      }
    }
    // renormalised weights: p_j / sum_S p = exp(l_j - l_max) / sum_S exp(l_i - l_max)
    const float lmax = __shfl_sync(0xffffffffu, my_v, 0);
    const float ex = (lane < k) ? expf(my_v - lmax) : 0.f;
    float sum = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (lane < k) {
      const float wj = ex / sum;
      a.topk_ids[(size_t)t * k + lane] = my_id;
      a.topk_w[(size_t)t * k + lane] = wj;
      s_ids[t * k + lane] = my_id;
      s_w[t * k + lane] = wj;
    }
  }
  for (int e = tid; e < E; e += kRouterThreads) s_cnt[e] = 0;
  __syncthreads();
  const int nas = B * k;
  for (int i = tid; i < nas; i += kRouterThreads) atomicAdd(&s_cnt[s_ids[i]], 1);
  __syncthreads();

  // Exclusive scans of counts and of units per expert over E (<= 1024 =
  // 4/thread); an expert with c tokens gets ceil(c / kMaxUnitTokens) units.
  int c4[4], f4[4], csum = 0, fsum = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid * 4 + i;
    c4[i] = e < E ? s_cnt[e] : 0;
    f4[i] = (c4[i] + kMaxUnitTokens - 1) / kMaxUnitTokens;
    csum += c4[i];
    fsum += f4[i];
  }
  int ctot, ftot;
  int cbase = block_exclusive_scan(csum, s_warp, ctot);
  int fbase = block_exclusive_scan(fsum, s_warp, ftot);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = tid * 4 + i;
    if (e < E) {
      s_off[e] = cbase;
      s_act[e] = f4[i] ? fbase : -1;
      for (int j = 0; j < f4[i]; ++j) {
        a.plan->unit_expert[fbase + j] = e;
        a.plan->unit_begin[fbase + j] = cbase + j * kMaxUnitTokens;
        a.plan->unit_count[fbase + j] = min(kMaxUnitTokens, c4[i] - j * kMaxUnitTokens);
      }
    }
    cbase += c4[i];
    fbase += f4[i];
  }
  if (tid == 0) {
    a.plan->n_active = ftot;
    if (ctot != nas) atomicCAS(a.status, kStatusOk, kStatusPlan);
  }

  __syncthreads();
  // Assignment (t, j) goes to offset[e] + #{t' < t : e in ids[t']} (ids of one
  // token are distinct, so this orders each expert's assignments by token).
  for (int i = tid; i < nas; i += kRouterThreads) {
    const int t = i / k, e = s_ids[i];
    int rank = 0;
    for (int i2 = 0; i2 < t * k; ++i2) rank += (s_ids[i2] == e);
    const int pos = s_off[e] + rank;
    a.plan->assign_tok[pos] = t;
    a.plan->assign_slot[pos] = i;
    a.plan->assign_w[pos] = s_w[i];
  }
  if (tid == 0) *a.ticket = 0u;
}

}  // namespace moe
