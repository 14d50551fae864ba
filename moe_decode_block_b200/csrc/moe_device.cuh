// moe_device.cuh -- device-side building blocks shared by the MoE decode
// kernels: constants, the routing plan written by the router kernel, and
// thin wrappers over the sm_90+/sm_100 PTX used for TMA bulk staging
// (cp.async.bulk + mbarrier), L2 prefetch and bounded waits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxExperts = 1024;
constexpr int kMaxTopK = 32;
constexpr int kMaxBatch = 64;
constexpr int kMaxAssign = kMaxBatch * kMaxTopK;
// A unit is one pass of the expert kernels over one expert's weights; an
// expert routed more than kMaxUnitTokens tokens is split into several units.
constexpr int kMaxUnitTokens = 32;
constexpr int kMaxUnits = kMaxExperts + kMaxAssign / kMaxUnitTokens;

// Device status word values (the host maps them to MOE_ERR_*).
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = 1;
constexpr int kStatusPlan = 2;

// Default bounded-wait limit (probes): try_wait already suspends in hardware
// for a while per probe, so this bounds a stuck wait to well under a minute.
// Launches take the limit they use as an argument (a handle can shorten it).
constexpr uint32_t kSpinLimit = 1u << 24;

// Routing plan: written by the last router CTA, read by the expert kernels.
// Units follow the active experts in ascending id order (an expert with more
// than kMaxUnitTokens tokens gets several consecutive units); the
// assignments of unit u are [unit_begin[u], unit_begin[u] + unit_count[u]),
// sorted by token.  `ready` is set (release store) once the rest is written;
// the expert kernel polls it instead of waiting for the router grid to
// complete, and its last CTA returns it to zero.
struct Plan {
  int n_active;  // number of units
  int ready;
  int pad_[2];
  int unit_expert[kMaxUnits];
  int unit_begin[kMaxUnits];
  int unit_count[kMaxUnits];
  int assign_slot[kMaxAssign];  // b * top_k + j: token b = slot / top_k, row of the per-assignment buffers
  float assign_w[kMaxAssign];   // renormalised routing weight
};

// Per-expert weight pointers, passed by value as a __grid_constant__
// parameter (8 KB) so no per-call host->device copy is needed.
struct ExpertTable {
  const __nv_bfloat16* p[kMaxExperts];
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait for the phase of `bar` with the given parity; gives up after `limit`
// probes, records kStatusTimeout in *status and returns false.  The result
// is per thread.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, int* status,
                                                  uint32_t limit = kSpinLimit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  atomicCAS(status, kStatusOk, kStatusTimeout);
  return false;
}

// Same, for waits inside a CTA that shares control words in shared memory:
// ctl[0] is the CTA's abort flag, ctl[1] the wait limit in probes.  Once any
// thread of the CTA has given up, the others stop waiting within ~1k probes,
// so a failed copy never turns into a hang.  Both words are read only every
// 1024 probes (the limit has that granularity), so the common path holds no
// register for them.  The result is per thread: lanes of one warp can
// disagree (one sees the phase complete, another the flag), so a warp that
// branches on it must first agree (mbar_wait_abortable_warp).
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t* bar, uint32_t parity, int* status,
                                                    volatile int* ctl) {
  for (uint32_t i = 0; i < kSpinLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 1023u) == 1023u) {
      if (ctl[0]) return false;
      if (i >= (uint32_t)ctl[1]) break;
    }
  }
  atomicCAS(status, kStatusOk, kStatusTimeout);
  ctl[0] = 1;
  return false;
}

// Warp-uniform form: every lane waits (so each lane's later shared-memory
// reads are ordered after the phase it observed), then the warp agrees --
// true only if every lane saw the phase complete.  What follows such a wait
// is warp-collective (ldmatrix / mma.sync / tcgen05.ld .sync.aligned,
// shuffles, __syncwarp), and a warp-collective instruction reached by only
// some lanes of a warp is undefined (on sm_100 it can raise an illegal
// instruction), so every branch on a wait result or on the abort flag is
// taken by whole warps.  Must be called by all 32 lanes.
__device__ __forceinline__ bool mbar_wait_abortable_warp(uint64_t* bar, uint32_t parity, int* status,
                                                         volatile int* ctl) {
  const bool ok = mbar_wait_abortable(bar, parity, status, ctl);
  return __all_sync(0xffffffffu, ok);
}

// The CTA's abort flag, read once and agreed by the whole warp (all 32 lanes
// must call it).
__device__ __forceinline__ bool warp_aborted(volatile int* abort_flag) {
  return __any_sync(0xffffffffu, *abort_flag != 0);
}

// L2 policy for weight streams: each weight byte is read once per forward,
// so mark it evict-first and leave L2 to the small activation buffers.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// TMA bulk copy global -> shared (no multicast), completion counted on `bar`.
// dst, src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Same without a cache hint (activations: small and re-read by many CTAs).
__device__ __forceinline__ void bulk_copy_g2s_plain(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// TMA tiled load of a 3-D box described by a tensor map in global memory
// (no multicast), completion counted on `bar`.  dst must be 1024-byte
// aligned when the map uses 128-byte swizzling.
__device__ __forceinline__ void tma_load_3d(void* dst, const void* map, int c0, int c1, int c2, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// TMA tiled load of a 2-D box (no multicast), completion counted on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int c0, int c1, uint64_t* bar,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_addr(bar)), "l"(policy)
      : "memory");
}

// Fire-and-forget fp32 adds to global memory (no value comes back, so a warp
// issuing many of them never waits on their round trips).  Vector forms need
// the address aligned to the vector size.
__device__ __forceinline__ void red_add(float* p, float a) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}
__device__ __forceinline__ void red_add_v2(float* p, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(a), "f"(b) : "memory");
}

__device__ __forceinline__ void bf16x2_to_f32(uint32_t v, float& lo, float& hi) {
  lo = __uint_as_float(v << 16);
  hi = __uint_as_float(v & 0xffff0000u);
}

__device__ __forceinline__ float silu_f32(float z) { return z / (1.0f + expf(-z)); }

}  // namespace moe
