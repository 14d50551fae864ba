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

// MOE_FLAG_PARTIAL_SUM: out[t, c] = acc[t, c] (fp32, no residual, no
// rounding) for a tensor-parallel rank's share of the block; acc returns to
// zero.
__global__ void __launch_bounds__(256) partial_sum_kernel(float* __restrict__ acc, float* __restrict__ out,
                                                          int n_vec4) {
  cudaGridDependencySynchronize();
  cudaTriggerProgrammaticLaunchCompletion();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_vec4) return;
  float4* ap = reinterpret_cast<float4*>(acc) + i;
  reinterpret_cast<float4*>(out)[i] = *ap;
  *ap = make_float4(0.f, 0.f, 0.f, 0.f);
}

// The ranks' partial sums, by value (device pointers; peer memory allowed).
constexpr int kMaxReduceParts = 16;
struct PartialPtrs {
  const float* p[kMaxReduceParts];
};

// out[t, c] = bf16_rne(x[t, c] + (partials[0][t, c] + partials[1][t, c] +
// ...)), the ranks' sums added in rank order so every rank gets the same
// bits; 8 columns per thread (one 16-byte load of x, two of each partial).
__global__ void __launch_bounds__(256) reduce_residual_kernel(const __grid_constant__ PartialPtrs pp, int n_parts,
                                                              const __nv_bfloat16* x, __nv_bfloat16* out,
                                                              int n_vec8) {
  // (x and out may be the same buffer: each thread reads its x before it
  // writes the same elements of out)
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n_vec8) return;
  float s[8];
  {
    const float4* p0 = reinterpret_cast<const float4*>(pp.p[0]) + 2 * (size_t)i;
    const float4 a0 = __ldcg(p0), a1 = __ldcg(p0 + 1);
    s[0] = a0.x; s[1] = a0.y; s[2] = a0.z; s[3] = a0.w;
    s[4] = a1.x; s[5] = a1.y; s[6] = a1.z; s[7] = a1.w;
  }
  for (int r = 1; r < n_parts; ++r) {
    const float4* pr = reinterpret_cast<const float4*>(pp.p[r]) + 2 * (size_t)i;
    const float4 a0 = __ldcg(pr), a1 = __ldcg(pr + 1);
    s[0] += a0.x; s[1] += a0.y; s[2] += a0.z; s[3] += a0.w;
    s[4] += a1.x; s[5] += a1.y; s[6] += a1.z; s[7] += a1.w;
  }
  const uint4 xv = reinterpret_cast<const uint4*>(x)[i];
  float xf[8];
  bf16x2_to_f32(xv.x, xf[0], xf[1]);
  bf16x2_to_f32(xv.y, xf[2], xf[3]);
  bf16x2_to_f32(xv.z, xf[4], xf[5]);
  bf16x2_to_f32(xv.w, xf[6], xf[7]);
  uint32_t o[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(xf[2 * c] + s[2 * c], xf[2 * c + 1] + s[2 * c + 1]);
    o[c] = *reinterpret_cast<const uint32_t*>(&v);
  }
  reinterpret_cast<uint4*>(out)[i] = make_uint4(o[0], o[1], o[2], o[3]);
}

}  // namespace moe
