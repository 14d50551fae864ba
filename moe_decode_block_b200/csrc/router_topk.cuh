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
//   * A work item is a pair of expert columns and a group of 8 tokens; a
//     thread accumulates the item's partial logits over the slab in fp32, and
//     partials are reduced into a global fp32 [B, E] buffer with vector
//     reductions (red, no return).
//   * The last CTA to finish (ticket counter) stages the logits in shared
//     memory (one batched load per group of tokens), adds the optional bias,
//     selects the top k per token with warp argmax rounds, computes the
//     renormalised weights, writes topk_ids/topk_w, builds the bucketed plan
//     (experts ascending, assignments sorted by token) and returns the ticket
//     to zero for the next call.
//   * Zeroing the logits for the next call is spread over all CTAs: with two
//     buffers used alternately (parity of a launch counter), each CTA clears
//     a slice of the buffer the next launch will use while it runs its GEMV.
//     The last CTA runs while the expert kernel already streams weights at
//     full HBM bandwidth, so every global access it makes queues behind that
//     traffic: it reads the logits once and writes only the results.
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
  float* logits;                // fp32 accumulators [B, E]; see logits_stride
  int logits_stride;            // 0: one buffer, zero between calls (the last CTA re-zeroes it);
                                // > 0: two buffers logits and logits + stride (>= B * E floats,
                                // a multiple of 4), used by launch parity, the unused one zero
  unsigned* epoch;              // launch counter choosing the buffer (logits_stride > 0)
  unsigned* ticket;             // zero between calls
  Plan* plan;
  int32_t* topk_ids;            // [B, k]
  float* topk_w;                // [B, k]
  int* status;
  uint32_t spin_limit;          // probes before the slab wait gives up
};

// Tokens padded to a multiple of 8 (x is staged token-contiguous per row).
__host__ __device__ inline int router_bpad(int B) { return (B + 7) / 8 * 8; }

// Tokens whose logits the last CTA stages in shared memory at once.
__host__ __device__ inline int router_stage_tokens(int B, int E) {
  const int tb = 16384 / E;  // 64 KB of fp32 logits
  return B < tb ? B : (tb < 1 ? 1 : tb);
}

// Shared memory needed by router_topk_kernel for these sizes.
__host__ __device__ inline size_t router_smem_bytes(int B, int E, int chunk_rows) {
  size_t gemv = (size_t)chunk_rows * E * 2 + (size_t)router_bpad(B) * chunk_rows * 4;
  size_t topk = (size_t)kMaxAssign * 8 + (size_t)E * 16 + 64 + ((size_t)router_stage_tokens(B, E) + 1) * E * 4;
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

// (value, id) order of the selection: larger logit first, equal logits to the
// smaller expert id.
__device__ __forceinline__ bool ranks_before(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// Top-8 of one token's logits by one warp: lg (shared memory) holds the E
// logits, bias the per-expert bias; every lane ends with the 8 best
// (value, id) pairs sorted in selection order.  Each lane first keeps its own
// best 8 (experts lane + 32 i) in a sorted list (insertion), then five
// butterfly levels merge lists between lanes l and l ^ off: the element-wise
// better of list A and reversed list B is a bitonic sequence holding the 8
// best of both, which a 3-stage bitonic network sorts.  The loops over
// experts and levels are kept rolled: this runs once per call in one CTA
// while the expert kernel saturates the memory system, so a long straight
// line of code would pay for instruction fetches.
__device__ __forceinline__ void warp_top8(const float* lg, const float* bias, int E, int lane, float (&tv)[8],
                                          int (&ti)[8]) {
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    tv[r] = -INFINITY;
    ti[r] = 0x7fffffff;  // after every real expert on ties
  }
#pragma unroll 1
  for (int e = lane; e < E; e += 32) {
    float cv = lg[e] + bias[e];
    int ci = e;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const bool sw = ranks_before(cv, ci, tv[r], ti[r]);
      const float sv = tv[r];
      const int si = ti[r];
      tv[r] = sw ? cv : sv;
      ti[r] = sw ? ci : si;
      cv = sw ? sv : cv;
      ci = sw ? si : ci;
    }
  }
#pragma unroll 1
  for (int off = 1; off < 32; off <<= 1) {
    float pv[8];
    int pi[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      pv[r] = __shfl_xor_sync(0xffffffffu, tv[r], off);
      pi[r] = __shfl_xor_sync(0xffffffffu, ti[r], off);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const bool sw = ranks_before(pv[7 - r], pi[7 - r], tv[r], ti[r]);
      tv[r] = sw ? pv[7 - r] : tv[r];
      ti[r] = sw ? pi[7 - r] : ti[r];
    }
#pragma unroll
    for (int d = 4; d > 0; d >>= 1) {
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if ((r & d) == 0) {
          const bool sw = ranks_before(tv[r + d], ti[r + d], tv[r], ti[r]);
          const float a0 = tv[r], a1 = tv[r + d];
          const int i0 = ti[r], i1 = ti[r + d];
          tv[r] = sw ? a1 : a0;
          ti[r] = sw ? i1 : i0;
          tv[r + d] = sw ? a0 : a1;
          ti[r + d] = sw ? i0 : i1;
        }
      }
    }
  }
}

// Exclusive scan of one int per thread over the block (NT threads).
template <int NT>
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
    int t = lane < NT / 32 ? warp_tot[lane] : 0;
    int ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int o = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += o;
    }
    if (lane < NT / 32) warp_tot[lane] = ti - t;  // exclusive warp offsets
    if (lane == NT / 32 - 1) warp_tot[NT / 32] = ti;
  }
  __syncthreads();
  const int r = warp_tot[warp] + inc - v;
  total = warp_tot[NT / 32];
  __syncthreads();
  return r;
}

// NV: logits per lane a warp holds in registers during top-k (E <= 32 * NV).
// Threads: 512 up to 512 experts -- sixteen warps share the last CTA's
// per-token top-k and the GEMV's (expert pair, token group) items -- and 256
// above, where a lane's 32 logits need more than the 128 registers a
// 512-thread block leaves.
__host__ __device__ constexpr int router_threads(int nv) { return nv <= 16 ? 512 : 256; }

template <int NV>
__global__ void __launch_bounds__(router_threads(NV), 1) router_topk_kernel(const __grid_constant__ RouterArgs a) {
  constexpr int NT = router_threads(NV);
  extern __shared__ __align__(1024) uint8_t router_smem[];
  uint8_t* smem = router_smem;
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_last;
  __shared__ int s_warp[NT / 32 + 1];

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

  // this launch's logits buffer; clear this CTA's slice of the other one
  float* lg_buf = a.logits;
  if (a.logits_stride > 0) {
    const unsigned par = __ldcg(a.epoch) & 1u;
    lg_buf = a.logits + (size_t)par * a.logits_stride;
    float4* other = reinterpret_cast<float4*>(a.logits + (size_t)(par ^ 1u) * a.logits_stride);
    const int n4 = a.logits_stride / 4;
    const int c0 = (int)((long long)n4 * blockIdx.x / a.G), c1 = (int)((long long)n4 * (blockIdx.x + 1) / a.G);
    for (int i = c0 + tid; i < c1; i += NT) __stcg(other + i, make_float4(0.f, 0.f, 0.f, 0.f));
  }

  uint32_t phase = 0;
  bool copy_failed = false;  // block-uniform
  const int npairs = E / 2;
  const int bp = router_bpad(B);
  for (int r0 = h0; r0 < h1; r0 += a.chunk_rows) {
    const int nr = min(a.chunk_rows, h1 - r0);
    // x staged as [row][token] (tokens padded to 8 with zeros), so a row's
    // 8-token group is two 16-byte shared loads
    for (int i = tid; i < bp * nr; i += NT) {
      const int r = i / bp, t = i - r * bp;
      xs[i] = t < B ? __bfloat162float(a.x[(size_t)t * H + r0 + r]) : 0.f;
    }
    // the whole block agrees on the outcome: after a failed wait no thread
    // reads the slab and no further copy is issued into it (the status word
    // says the logits are incomplete; the plan below stays well formed)
    if (!__syncthreads_and(mbar_wait_bounded(&bar, phase, a.status, a.spin_limit))) {
      copy_failed = true;
      break;
    }
    phase ^= 1;
    // items: (expert pair, group of 8 tokens); a warp's lanes take
    // consecutive pairs of one group
    const int n_items = npairs * ((B + 7) / 8);
    for (int it = tid; it < n_items; it += NT) {
      {
        const int t0 = (it / npairs) * 8, p = it - (it / npairs) * npairs;
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
            red_add_v2(lg_buf + (size_t)(t0 + j) * E + 2 * p, acc[j][0], acc[j][1]);
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

  // a copy whose wait gave up may still land in the slab: wait for it (with
  // the default limit) before this CTA can exit
  if (copy_failed && tid == 0) mbar_wait_bounded(&bar, phase, a.status);

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

  float* s_bias = reinterpret_cast<float*>(s_act + E);  // [E] (16-byte aligned: E % 8 == 0)
  float* s_lg = s_bias + E;                                 // [TB, E]
  for (int e = tid; e < E; e += NT) s_bias[e] = a.bias ? a.bias[e] : 0.f;
  const int nv = (E + 31) / 32;
  const int TB = router_stage_tokens(B, E);
  constexpr int NWARP = NT / 32;
  // one token whose logits all fit one per thread: the threshold top-k below
  const bool one_token = B == 1 && E <= NT && k <= 8 && nv >= k;
  // lanes j < k of a warp hold token t's selection in order: the ids, their
  // renormalised weights p_j / sum_S p = exp(l_j - l_max) / sum_S exp(l_i - l_max)
  auto finish_token = [&](int t, int my_id, float my_v) {
    if (lane < k && (my_id < 0 || my_id >= E)) {  // cannot happen for k <= E; keep the plan valid
      atomicCAS(a.status, kStatusOk, kStatusPlan);
      my_id = lane;
    }
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
  };
  for (int tb0 = 0; tb0 < B; tb0 += TB) {
    const int ntb = min(TB, B - tb0);
    {
      // one batched load of ntb rows of logits (8 float4 in flight per thread)
      float4* src = reinterpret_cast<float4*>(lg_buf + (size_t)tb0 * E);
      float4* dst = reinterpret_cast<float4*>(s_lg);
      const int n4 = ntb * E / 4;
      for (int i0 = 0; i0 < n4; i0 += 8 * NT) {
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * NT + tid;
          if (i < n4) v[u] = __ldcg(src + i);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int i = i0 + u * NT + tid;
          if (i < n4) {
            dst[i] = v[u];
            if (a.logits_stride == 0) __stcg(src + i, make_float4(0.f, 0.f, 0.f, 0.f));
          }
        }
      }
    }
    __syncthreads();
  if (one_token) {
    // One token, one logit per thread.  The k-th largest of the warps' maxima
    // is a threshold no member of the top k lies below (k real values reach
    // it); the values at or above it -- a handful -- are collected and one
    // warp sorts them by (value desc, id asc).  A few dependent steps across
    // the whole CTA instead of one warp's long merge chain on the path the
    // expert kernel waits for.  More than 32 candidates (ties on a large
    // scale): the one-warp merge below.
    float* w_max = s_w + kMaxAssign - 64;  // [NWARP + 1]: the warps' maxima, then the threshold
    int* n_cand = s_ids + kMaxAssign - 64;
    float* cand_v = s_w + kMaxAssign / 2;  // [32]
    int* cand_i = s_ids + kMaxAssign / 2;
    const float v = tid < E ? s_lg[tid] + s_bias[tid] : -INFINITY;
    float m = v;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) w_max[warp] = m;
    if (tid == 0) *n_cand = 0;
    __syncthreads();
    if (warp == 0) {
      float mv = lane < NWARP ? w_max[lane] : -INFINITY;
      // bitonic sort, descending
#pragma unroll
      for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, mv, stride);
          const bool keep_max = ((lane & stride) == 0) == ((lane & size) == 0);
          mv = keep_max ? fmaxf(mv, ov) : fminf(mv, ov);
        }
      }
      if (lane == k - 1) w_max[NWARP] = mv;
    }
    __syncthreads();
    const float thr = w_max[NWARP];
    if (tid < E && v >= thr) {
      const int p = atomicAdd(n_cand, 1);
      if (p < 32) {
        cand_v[p] = v;
        cand_i[p] = tid;
      }
    }
    __syncthreads();
    if (warp == 0) {
      const int nc = *n_cand;
      int my_id = -1;
      float my_v = -INFINITY;
      if (nc <= 32) {
        float cv = lane < nc ? cand_v[lane] : -INFINITY;
        int ci = lane < nc ? cand_i[lane] : 0x7fffffff;
        // bitonic sort, best first: larger value, then the smaller id
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
          for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, cv, stride);
            const int oi = __shfl_xor_sync(0xffffffffu, ci, stride);
            const bool other_better = ranks_before(ov, oi, cv, ci);
            const bool keep_better = ((lane & stride) == 0) == ((lane & size) == 0);
            if (keep_better == other_better) {
              cv = ov;
              ci = oi;
            }
          }
        }
        if (lane < k) {
          my_id = ci;
          my_v = cv;
        }
      } else {
        float tv[8];
        int ti[8];
        warp_top8(s_lg, s_bias, E, lane, tv, ti);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          if (r == lane && r < k) {
            my_id = ti[r];
            my_v = tv[r];
          }
        }
      }
      finish_token(tb0, my_id, my_v);
    }
  } else
  for (int t = tb0 + warp; t < tb0 + ntb; t += NT / 32) {
    const float* lg = s_lg + (size_t)(t - tb0) * E;
    float v[NV];
    uint32_t taken = 0;
    const bool rounds = k > 8;
    if (rounds) {
#pragma unroll
      for (int i = 0; i < NV; ++i) {
        const int e = lane + 32 * i;
        v[i] = -INFINITY;
        if (i < nv && e < E) v[i] = lg[e] + s_bias[e];
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
    int my_id = -1;
    float my_v = -INFINITY;
    if (!rounds) {
      float tv[8];
      int ti[8];
      warp_top8(lg, s_bias, E, lane, tv, ti);
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (r == lane && r < k) {
          my_id = ti[r];
          my_v = tv[r];
        }
      }
    } else {
    float lbv;
    int lbi;
    local_best(lbv, lbi);
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
    }
    finish_token(t, my_id, my_v);
  }
    __syncthreads();  // the staging buffer is reused by the next group of tokens
  }
  for (int e = tid; e < E; e += NT) s_cnt[e] = 0;
  __syncthreads();
  const int nas = B * k;
  for (int i = tid; i < nas; i += NT) atomicAdd(&s_cnt[s_ids[i]], 1);
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
  int cbase = block_exclusive_scan<NT>(csum, s_warp, ctot);
  int fbase = block_exclusive_scan<NT>(fsum, s_warp, ftot);
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
  // Assignment (t, j) goes to offset[e] + #{t' < t : e in ids[t']}: one warp
  // walks the tokens in order, lane j placing slot j, with a per-expert fill
  // counter (the ids of one token are distinct, so no two lanes of a step
  // share a counter); each expert's assignments end up ordered by token.
  for (int e = tid; e < E; e += NT) s_cnt[e] = 0;
  __syncthreads();
  if (warp == 0) {
    for (int t = 0; t < B; ++t) {
      if (lane < k) {
        const int i = t * k + lane, e = s_ids[i];
        const int pos = s_off[e] + s_cnt[e];
        s_cnt[e] = s_cnt[e] + 1;
        if (pos < nas) {
          a.plan->assign_slot[pos] = i;
          a.plan->assign_w[pos] = s_w[i];
        }
      }
      __syncwarp();
    }
  }
  // publish: every thread's plan writes, then the flag the expert kernel's
  // producers poll (sooner than this grid's completion)
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(&a.plan->ready), "r"(1u) : "memory");
    *a.ticket = 0u;
    if (a.logits_stride > 0) *a.epoch = *a.epoch + 1u;  // every CTA read it before taking its ticket
  }
}

}  // namespace moe
