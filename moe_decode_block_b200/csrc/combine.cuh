// combine.cuh -- weighted combine + residual epilogue of the MoE block.
//
// The routed experts (each scaled by its renormalised routing weight) and the
// shared expert (weight 1) have already been summed into one fp32 buffer by
// the expert kernels' atomics; this kernel adds the block input x (the
// residual) and rounds once to bf16 (pages: "Hyper Optimizing Kimi K3 in
// vLLM", section "Recovering time between operators": residual processing is
// fused with the producing step's epilogue).  It also returns the buffer to
// zero for the next forward.
#pragma once

#include "expert_mma.cuh"
#include "moe_device.cuh"

namespace moe {

// What the combine kernel needs to count, per token class, the weight
// stages the expert kernels streamed (from the plan they consumed).
struct StageCountArgs {
  const Plan* plan;                  // the routed units (nullptr: no routed pass)
  unsigned long long* counts;        // [kNumClasses * 2]: UP, DOWN per class, cumulative
  int n_su, batch, H, I, Is, kc, max_units, fp8;
};

// out[t, c] = bf16_rne(x[t, c] + acc[t, c]); acc returns to zero.  Warp 0 of
// CTA 0 also adds the stages of this forward's units to the per-class
// counters (device-side evidence of which token classes ran), off the
// expert kernels' paths.
__global__ void __launch_bounds__(256) combine_residual_kernel(const __nv_bfloat16* __restrict__ x,
                                                               float* __restrict__ acc,
                                                               __nv_bfloat16* __restrict__ out, int n_vec8,
                                                               const __grid_constant__ StageCountArgs sc) {
  cudaGridDependencySynchronize();
  cudaTriggerProgrammaticLaunchCompletion();
  if (blockIdx.x == 0 && threadIdx.x < 32) {
    const int lane = threadIdx.x;
    unsigned long long c[2 * kNumClasses] = {};
    auto add = [&](int n, int I) {
      const int cls = min(class_for_tokens(n), sc.kc);
      const unsigned long long u = (unsigned long long)unit_stages(cls, true, sc.H, I, sc.fp8 != 0);
      const unsigned long long d = (unsigned long long)unit_stages(cls, false, sc.H, I, sc.fp8 != 0);
#pragma unroll
      for (int j = 0; j < kNumClasses; ++j) {
        c[2 * j] += cls == j ? u : 0ull;
        c[2 * j + 1] += cls == j ? d : 0ull;
      }
    };
    for (int su = lane; su < sc.n_su; su += 32) add(min(kMaxUnitTokens, sc.batch - su * kMaxUnitTokens), sc.Is);
    if (sc.plan) {
      const int n = min(max(__ldcg(&sc.plan->n_active), 0), sc.max_units);
      for (int u = lane; u < n; u += 32) add(min(max(__ldcg(&sc.plan->unit_count[u]), 0), kMaxUnitTokens), sc.I);
    }
#pragma unroll
    for (int j = 0; j < 2 * kNumClasses; ++j) {
      const unsigned long long v = __reduce_add_sync(0xffffffffu, (unsigned)c[j]);
      if (lane == 0 && v) atomicAdd(&sc.counts[j], v);
    }
  }
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
