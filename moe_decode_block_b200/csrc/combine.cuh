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

}  // namespace moe
