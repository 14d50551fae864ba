// moe_decode.cu -- host side of the C ABI declared in include/moe_decode.h.
//
// Two execution plans (pages: "Hyper Optimizing Kimi K3 in vLLM", section
// "Recovering time between operators": the shared expert overlaps routing,
// weights are fetched before their consumer starts, the residual add is
// fused into the producing epilogue, fewer launches per layer):
//   default (three kernels, stream_main only):
//     router+top-k+plan; the persistent expert kernel, which streams the
//     shared expert's up projection before its grid-dependency wait (so it
//     overlaps the router) and then the routed experts and the shared
//     expert's down projection; combine + residual.
//   MOE_FLAG_TWO_STREAM (four kernels, the pages' layout):
//     stream_main: router, routed experts, [join] combine
//     stream_aux : shared expert, forked with an event after the router
// Consecutive kernels on one stream use programmatic dependent launch so the
// next kernel's CTAs start (and fetch static weights) while the previous one
// drains.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "moe_decode.h"
#include "combine.cuh"
#include "expert_mma.cuh"
#include "expert_tc.cuh"
#include "moe_device.cuh"
#include "router_topk.cuh"

namespace {

using moe::ExpertTable;
using moe::MmaArgs;
using moe::Plan;
using moe::RouterArgs;

thread_local int g_last_cuda_error = 0;

// Workspace: [0, state_end) is the per-forward state (returned to zero by
// every forward, re-zeroed after a failure); the tensor maps and the
// device-side stage counters follow, outside that range, so re-zeroing the
// state never destroys them.
struct WorkspaceLayout {
  size_t status, ticket, router_epoch, logits, plan, h, a, panel_cnt, panel_ready, queue, h_s, a_s, panel_cnt_s, panel_ready_s,
      queue_s, acc, x_stage, out_stage, ids_stage, w_stage, state_end, maps, stage_counts, total;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Block scales of e4m3 expert weights (moe_decode_forward_fp8).
struct Fp8Scales {
  const void* const* w13s;  // host array of E device pointers
  const void* const* w2s;
  const void* sw13s;        // shared expert
  const void* sw2s;
};

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

bool shapes_valid(const moe_decode_shapes* s) {
  if (!s) return false;
  auto in = [](int v, int lo, int hi) { return v >= lo && v <= hi; };
  if (!in(s->hidden, 8, 16384) || s->hidden % 8) return false;
  if (!in(s->n_experts, 8, moe::kMaxExperts) || s->n_experts % 8) return false;
  if (!in(s->top_k, 1, moe::kMaxTopK) || s->top_k > s->n_experts) return false;
  if (!in(s->inter, 8, 16384) || s->inter % 8) return false;
  if (s->n_shared != 0 && s->n_shared != 1) return false;
  if (s->n_shared == 1 && (!in(s->shared_inter, 8, 16384) || s->shared_inter % 8)) return false;
  if (!in(s->max_batch, 1, moe::kMaxBatch)) return false;
  if ((s->flags & ~(MOE_FLAG_TWO_STREAM | MOE_FLAG_TCGEN05 | MOE_FLAG_TEST_HOLD_PANEL | MOE_FLAG_FP8_WEIGHTS |
                    MOE_FLAG_PARTIAL_SUM)) != 0)
    return false;
  if (s->flags & MOE_FLAG_FP8_WEIGHTS) {
    // e4m3 weights: whole 128 x 128 scale blocks, on the mma.sync kernel
    if (s->hidden % 128 || s->inter % 128 || (s->n_shared && s->shared_inter % 128)) return false;
    if (s->flags & MOE_FLAG_TCGEN05) return false;
  }
  return true;
}

// Units of a routed pass: one per active expert, plus the extra units of
// experts routed more than kMaxUnitTokens tokens.
size_t max_units(const moe_decode_shapes* s) {
  return (size_t)s->n_experts + ((size_t)s->max_batch * s->top_k) / moe::kMaxUnitTokens;
}

// Units of the shared expert for a batch (each holds at most kMaxUnitTokens).
inline int shared_units(const moe_decode_shapes& s, int batch) {
  return s.n_shared ? (batch + moe::kMaxUnitTokens - 1) / moe::kMaxUnitTokens : 0;
}

WorkspaceLayout layout_for(const moe_decode_shapes* s) {
  WorkspaceLayout L{};
  const size_t A = 256;
  const size_t B = (size_t)s->max_batch, E = (size_t)s->n_experts, k = (size_t)s->top_k;
  const size_t H = (size_t)s->hidden, I = (size_t)s->inter;
  const size_t Is = s->n_shared ? (size_t)s->shared_inter : 0;
  const int ncp = moe::max_up_panels(s->inter);
  const int ncp_s = s->n_shared ? moe::max_up_panels(s->shared_inter) : 0;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, A);
    return o;
  };
  L.status = take(sizeof(int));
  L.ticket = take(sizeof(unsigned));
  L.router_epoch = take(sizeof(unsigned));
  L.logits = take(2 * B * E * 4);  // two buffers, used alternately by the router
  L.plan = take(sizeof(Plan));
  L.h = take(B * k * 2 * I * 4);
  L.a = take(B * k * I * 2);
  const size_t U = max_units(s);
  L.panel_cnt = take(U * (size_t)ncp * 4);
  L.panel_ready = take(U * (size_t)ncp * 4);
  L.queue = take(4 * 4);
  L.h_s = take(B * 2 * Is * 4);
  L.a_s = take(B * Is * 2);
  const size_t su = (size_t)shared_units(*s, s->max_batch);
  L.panel_cnt_s = take(su * ncp_s * 4 + 4);
  L.panel_ready_s = take(su * ncp_s * 4 + 4);
  L.queue_s = take(4 * 4);
  L.acc = take(B * H * 4);
  L.x_stage = take(B * H * 2);
  L.out_stage = take(B * H * 2);
  L.ids_stage = take(B * k * 4);
  L.w_stage = take(B * k * 4);
  L.state_end = off;
  L.maps = take((2 * E + 2) * (size_t)moe::kTensorMapBytes);  // tensor maps: w13[E], w2[E], shared w13, w2
  L.stage_counts = take(2 * moe::kNumClasses * sizeof(unsigned long long));
  L.total = off;
  return L;
}

int env_int(const char* name, int dflt, int lo, int hi) {
  const char* v = std::getenv(name);
  if (!v || !*v) return dflt;
  int x = std::atoi(v);
  return x < lo ? lo : (x > hi ? hi : x);
}

int fail_cuda(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return MOE_ERR_CUDA;
}

template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t st, bool pdl,
                   Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3((unsigned)block);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

using MlpKernel = void (*)(MmaArgs, ExpertTable, ExpertTable);

// The expert kernel compiled for the largest token class `kc` (0..2) a
// launch can see, on the tensor-map or the row-copy path.
template <bool TMAP>
MlpKernel pick_mlp_t(int kc) {
  switch (kc) {
    case 0: return moe::expert_mlp_kernel<0, TMAP>;
    case 1: return moe::expert_mlp_kernel<1, TMAP>;
    default: return moe::expert_mlp_kernel<2, TMAP>;
  }
}
MlpKernel pick_mlp(int kc, bool tmap) { return tmap ? pick_mlp_t<true>(kc) : pick_mlp_t<false>(kc); }
// The expert kernel on e4m3 weights (tensor-map path only).
MlpKernel pick_mlp_fp8(int kc) {
  switch (kc) {
    case 0: return moe::expert_mlp_kernel<0, true, true>;
    case 1: return moe::expert_mlp_kernel<1, true, true>;
    default: return moe::expert_mlp_kernel<2, true, true>;
  }
}

// Token class the expert kernel is compiled for at this batch: units hold
// at most kMaxUnitTokens tokens.
inline int kernel_class(int batch) {
  return moe::class_for_tokens(batch < moe::kMaxUnitTokens ? batch : moe::kMaxUnitTokens);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library is needed).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

// Tensor map of a row-major bf16 [rows, cols] matrix seen as the 3-D tensor
// {64 columns, rows, cols / 64 chunks} (strides: one row, 128 bytes), with
// {64, 16, 4} boxes and 128-byte swizzling (see expert_mma.cuh).
bool encode_matrix_map(uint8_t* out, const void* base, int rows, int cols) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc || cols % moe::kChunkCols) return false;
  CUtensorMap m;
  cuuint64_t dims[3] = {(cuuint64_t)moe::kChunkCols, (cuuint64_t)rows, (cuuint64_t)(cols / moe::kChunkCols)};
  cuuint64_t strides[2] = {(cuuint64_t)cols * 2, (cuuint64_t)moe::kChunkCols * 2};
  cuuint32_t box[3] = {(cuuint32_t)moe::kChunkCols, (cuuint32_t)moe::kBoxRows, (cuuint32_t)moe::kBoxChunks};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  static_assert(sizeof(CUtensorMap) == moe::kTensorMapBytes, "tensor map size");
  std::memcpy(out, &m, sizeof m);
  return true;
}

// Tensor map of an e4m3 matrix [rows, cols] stored row-major ([out, in]: a
// row holds one output's weights over the inputs), seen as the 2-D tensor
// {cols, rows} with {128, 128} boxes (128 bytes of inputs x 128 outputs) and
// 128-byte swizzling (see mma_stage_fp8).
bool encode_fp8_map(uint8_t* out, const void* base, int rows, int cols) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc || cols % 16) return false;
  CUtensorMap m;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols};
  // one load: 128 input bytes (one line) of 128 output rows, 128-byte swizzle
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  std::memcpy(out, &m, sizeof m);
  return true;
}

// Floats per row of an e4m3 matrix's block scales: one per 128 outputs,
// padded to a multiple of 4 (16-byte rows).
inline int scale_pitch(int outs) { return ((outs + 127) / 128 + 3) / 4 * 4; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// Address at which the current device can write the host buffer `p` (pinned
// host memory mapped into the device's address space), or nullptr when it
// has none (pageable memory) or is not aligned to `align` bytes.  Asked anew
// on every call: a buffer can be unpinned and its address reused.
void* host_buffer_device_view(void* p, uintptr_t align) {
  if ((reinterpret_cast<uintptr_t>(p) & (align - 1)) != 0) return nullptr;
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

}  // namespace

struct moe_decode_ctx {
  moe_decode_shapes s{};
  int device = 0;
  int num_sms = 0;
  int n_stages = 3;     // stage ring depth of expert_mlp_kernel
  int n_stages_tc = 2;  // of expert_tc_kernel (its B-operand buffers take room)
  int grid_routed = 0, grid_shared = 0, grid_router_max = 0;
  bool grid_routed_auto = true;
  int router_chunk_rows = 0;
  int stagger = 8;             // expert kernel: stagger period of the first segment-B chunks
  WorkspaceLayout L{};
  uint8_t* ws = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  // end of the last forward enqueued outside graph capture (what
  // get_status / get_stats / destroy wait for); captured_last: the last
  // forward was captured, so its work is on a stream the handle never sees
  cudaEvent_t ev_done = nullptr;
  bool done_recorded = false, captured_last = false;
  uint32_t spin_limit = moe::kSpinLimit;
  bool dirty = false;
  moe_decode_stats stats{};
  ExpertTable* tab13 = nullptr;  // host staging of the pointer tables (kernel parameters)
  ExpertTable* tab2 = nullptr;
  bool timing = false;
  cudaEvent_t tev[MOE_TIMING_EVENTS] = {};
  ExpertTable* tab_none = nullptr;  // zero table passed to the shared-expert launch
  // tensor-map path: maps encoded for the pointer tables of the last forward
  bool use_tmap = false;
  bool use_tc = false;  // tcgen05 expert kernel (tensor-map path only)
  uint8_t* maps_host = nullptr;  // pinned staging, (2E + 2) maps
  std::vector<const void*> map_ptrs;  // w13[E], w2[E], shared w13, shared w2 the maps describe
  bool maps_uploaded = false;
  cudaEvent_t ev_maps = nullptr;
  // moe_decode_forward_host with pinned, mapped host buffers: the copy of x
  // and the forward captured once into a graph and replayed while the
  // arguments stay the same (host_key)
  bool host_graph_on = true;
  cudaGraphExec_t host_exec = nullptr;
  std::vector<const void*> host_key;
  int host_key_batch = -1, host_graph_kernels = 0;

  template <typename T>
  T* at(size_t off) const {
    return reinterpret_cast<T*>(ws + off);
  }
};

namespace {

int router_grid(const moe_decode_ctx* h, int /*batch*/) {
  return h->grid_router_max < 1 ? 1 : h->grid_router_max;
}

// Router kernel holding E <= 32 * NV logits per lane during top-k.
using RouterKernel = void (*)(RouterArgs);
RouterKernel pick_router(int n_experts) {
  if (n_experts <= 128) return moe::router_topk_kernel<4>;
  if (n_experts <= 256) return moe::router_topk_kernel<8>;
  if (n_experts <= 512) return moe::router_topk_kernel<16>;
  return moe::router_topk_kernel<32>;
}
// Threads of the router kernel pick_router returns.
int router_threads_for(int n_experts) {
  return moe::router_threads(n_experts <= 128 ? 4 : (n_experts <= 256 ? 8 : (n_experts <= 512 ? 16 : 32)));
}

// CTAs for the shared expert when it runs beside the routed experts: its
// share of the forward's weight bytes (routed share estimated for uniform
// routing, E * (1 - (1 - k/E)^B) distinct experts), weighted up for the wider
// token classes, whose stages take the consumers longer per byte (empirical
// factors; only this two-stream plan uses them).  The routed kernel gets the
// remaining SMs, so the two grids never wait for each other's SMs.
int shared_grid(const moe_decode_ctx* h, int batch) {
  if (h->grid_shared > 0) return h->grid_shared;
  const moe_decode_shapes& s = h->s;
  const double E = s.n_experts, k = s.top_k;
  const double distinct = E * (1.0 - std::pow(1.0 - k / E, (double)batch));
  const double routed = distinct * 3.0 * s.hidden * s.inter;
  const int cls = kernel_class(batch);
  const double slow = cls <= 1 ? 1.3 : 3.0;
  const double shared = shared_units(s, batch) * 3.0 * s.hidden * s.shared_inter * slow;
  int g = (int)std::ceil(h->num_sms * shared / (shared + routed));
  const int cap = h->num_sms / 2;
  g = g < 1 ? 1 : (g > cap ? cap : g);
  return g;
}

// A kernel's dynamic shared-memory limit is a property of the function, not
// of a handle: raise it to what this handle needs, never lower it (another
// handle, made for a larger batch, may rely on the higher limit).
template <typename K>
cudaError_t raise_smem_limit(K kern, int bytes) {
  cudaFuncAttributes fa{};
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if (fa.maxDynamicSharedSizeBytes >= bytes) return cudaSuccess;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

int set_kernel_attrs(const moe_decode_ctx* h) {
  const int smem = (int)moe::mma_smem_bytes(h->n_stages);
  cudaError_t e;
  for (int kc = 0; kc < moe::kNumClasses; ++kc) {
    for (int tm = 0; tm < 2; ++tm) {
      if ((e = raise_smem_limit(pick_mlp(kc, tm), smem)) != cudaSuccess) return fail_cuda(e);
    }
  }
  for (int kc = 0; kc < moe::kNumClasses; ++kc)
    if ((e = raise_smem_limit(pick_mlp_fp8(kc), smem)) != cudaSuccess) return fail_cuda(e);
  if ((e = raise_smem_limit(moe::expert_tc_kernel, (int)moe::tc_smem_bytes(h->n_stages_tc))) != cudaSuccess)
    return fail_cuda(e);
  const int rsmem = (int)moe::router_smem_bytes(h->s.max_batch, h->s.n_experts, h->router_chunk_rows);
  if ((e = raise_smem_limit(pick_router(h->s.n_experts), rsmem)) != cudaSuccess) return fail_cuda(e);
  return MOE_OK;
}

// Tensor-map path: (re)encode the maps whose matrices moved since the last
// forward and copy the table to the workspace, in stream order.  Weight
// pointers normally stay fixed, so this usually does nothing.
int refresh_maps(moe_decode_ctx* h, const void* const* w13, const void* const* w2, const void* sw13,
                 const void* sw2, cudaStream_t sm) {
  const moe_decode_shapes& s = h->s;
  const int E = s.n_experts;
  const size_t nm = 2 * (size_t)E + 2, mb = moe::kTensorMapBytes;
  const void** ptrs = h->map_ptrs.data();
  uint8_t* stage = h->maps_host;
  bool changed = !h->maps_uploaded;
  for (int e = 0; e < E && !changed; ++e) changed = (ptrs[e] != w13[e] || ptrs[E + e] != w2[e]);
  if (s.n_shared && !changed) changed = (ptrs[2 * E] != sw13 || ptrs[2 * E + 1] != sw2);
  if (!changed) return MOE_OK;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(sm, &cap);
  // the staging buffer may still feed the previous upload
  if (h->maps_uploaded && cap == cudaStreamCaptureStatusNone) cudaEventSynchronize(h->ev_maps);
  const bool fp8 = (s.flags & MOE_FLAG_FP8_WEIGHTS) != 0;
  // bf16: w13 [H, 2I], w2 [I, H]; e4m3: w13 [2I, H], w2 [H, I]
  auto enc = [&](uint8_t* o, const void* p, int rows_bf16, int cols_bf16) {
    return fp8 ? encode_fp8_map(o, p, cols_bf16, rows_bf16) : encode_matrix_map(o, p, rows_bf16, cols_bf16);
  };
  for (int e = 0; e < E; ++e) {
    if (!enc(stage + e * mb, w13[e], s.hidden, 2 * s.inter)) return MOE_ERR_INVALID_ARG;
    if (!enc(stage + (E + e) * mb, w2[e], s.inter, s.hidden)) return MOE_ERR_INVALID_ARG;
    ptrs[e] = w13[e];
    ptrs[E + e] = w2[e];
  }
  if (s.n_shared) {
    if (!enc(stage + 2 * E * mb, sw13, s.hidden, 2 * s.shared_inter)) return MOE_ERR_INVALID_ARG;
    if (!enc(stage + (2 * E + 1) * mb, sw2, s.shared_inter, s.hidden)) return MOE_ERR_INVALID_ARG;
    ptrs[2 * E] = sw13;
    ptrs[2 * E + 1] = sw2;
  }
  cudaError_t e = cudaMemcpyAsync(h->ws + h->L.maps, stage, nm * mb, cudaMemcpyHostToDevice, sm);
  if (e != cudaSuccess) return fail_cuda(e);
  if (cap == cudaStreamCaptureStatusNone && (e = cudaEventRecord(h->ev_maps, sm)) != cudaSuccess)
    return fail_cuda(e);
  h->maps_uploaded = true;
  return MOE_OK;
}

// Enqueue the whole forward (device pointers only).
int enqueue_forward(moe_decode_ctx* h, const void* x, const void* router_w, const void* const* w13,
                    const void* const* w2, const void* shared_w13, const void* shared_w2, void* out,
                    int32_t* topk_ids, float* topk_w, int batch, cudaStream_t sm, cudaStream_t sa,
                    const Fp8Scales* f8) {
  const moe_decode_shapes& s = h->s;
  cudaError_t e;
  int kernels = 0;
  if (h->dirty) {
    // the per-forward state only: the tensor maps and the counters after it
    // stay as they are
    e = cudaMemsetAsync(h->ws, 0, h->L.state_end, sm);
    if (e != cudaSuccess) return fail_cuda(e);
    h->dirty = false;
  }
  // pointer tables (kernel parameters): the weights, or with e4m3 weights
  // (read through their tensor maps) the block-scale arrays
  for (int i = 0; i < s.n_experts; ++i) {
    h->tab13->p[i] = static_cast<const __nv_bfloat16*>(f8 ? f8->w13s[i] : w13[i]);
    h->tab2->p[i] = static_cast<const __nv_bfloat16*>(f8 ? f8->w2s[i] : w2[i]);
  }
  if (h->use_tmap) {
    const int rc = refresh_maps(h, w13, w2, shared_w13, shared_w2, sm);
    if (rc != MOE_OK) return rc;
  }
  const uint8_t* maps = h->ws + h->L.maps;
  const size_t mb = moe::kTensorMapBytes;
  int* status = h->at<int>(h->L.status);
  const bool two_stream = (s.flags & MOE_FLAG_TWO_STREAM) != 0;
  const bool fork = two_stream && s.n_shared && sa != sm;
  const int n_su = shared_units(s, batch);
  const int kc = kernel_class(batch);
  const MlpKernel mlp = f8 ? pick_mlp_fp8(kc) : (h->use_tc ? moe::expert_tc_kernel : pick_mlp(kc, h->use_tmap));
  const int mlp_threads = f8 ? moe::expert_threads(kc, true) : (h->use_tc ? moe::kTcThreads : moe::expert_threads(kc));
  const int n_stages = h->use_tc ? h->n_stages_tc : h->n_stages;
  const size_t smem = h->use_tc ? moe::tc_smem_bytes(n_stages) : moe::mma_smem_bytes(n_stages);

  auto bail = [&](cudaError_t err) {
    h->dirty = true;
    return fail_cuda(err);
  };
  auto mark = [&](int i, cudaStream_t st) {
    return h->timing ? cudaEventRecord(h->tev[i], st) : cudaSuccess;
  };

  // Arguments common to every expert-kernel launch of this forward.
  MmaArgs base{};
  base.H = s.hidden;
  base.I = s.inter;
  base.Is = s.n_shared ? s.shared_inter : 0;
  base.E = s.n_experts;
  base.top_k = s.top_k;
  base.n_stages = n_stages;
  base.batch = batch;
  base.max_units = (int)max_units(&s);
  base.panel_stride = moe::max_up_panels(s.inter);
  base.panel_stride_s = s.n_shared ? moe::max_up_panels(s.shared_inter) : 0;
  base.w13_s = static_cast<const __nv_bfloat16*>(f8 ? f8->sw13s : shared_w13);
  base.w2_s = static_cast<const __nv_bfloat16*>(f8 ? f8->sw2s : shared_w2);
  base.sc_pitch13 = scale_pitch(2 * s.inter);
  base.sc_pitch13_s = s.n_shared ? scale_pitch(2 * s.shared_inter) : 4;
  base.sc_pitch2 = scale_pitch(s.hidden);
  base.maps13 = maps;
  base.maps2 = maps + (size_t)s.n_experts * mb;
  base.maps13_s = maps + 2 * (size_t)s.n_experts * mb;
  base.maps2_s = maps + (2 * (size_t)s.n_experts + 1) * mb;
  base.plan = h->at<Plan>(h->L.plan);
  base.plan_ready = &h->at<Plan>(h->L.plan)->ready;
  base.stage_counts = h->at<unsigned long long>(h->L.stage_counts);
  base.x = static_cast<const __nv_bfloat16*>(x);
  base.h = h->at<float>(h->L.h);
  base.a = h->at<__nv_bfloat16>(h->L.a);
  base.h_s = h->at<float>(h->L.h_s);
  base.a_s = h->at<__nv_bfloat16>(h->L.a_s);
  base.acc = h->at<float>(h->L.acc);
  base.panel_cnt = h->at<unsigned>(h->L.panel_cnt);
  base.panel_ready = h->at<unsigned>(h->L.panel_ready);
  base.panel_cnt_s = h->at<unsigned>(h->L.panel_cnt_s);
  base.panel_ready_s = h->at<unsigned>(h->L.panel_ready_s);
  base.queue = h->at<unsigned>(h->L.queue);
  base.status = status;
  base.spin_limit = h->spin_limit;
  base.stagger = h->stagger;
  // testing only: the handle's first forward withholds routed UP panel 0
  base.hold_panel = ((s.flags & MOE_FLAG_TEST_HOLD_PANEL) && h->stats.forwards == 0) ? 0 : -1;

  // Router + top-k + plan.
  RouterArgs ra{};
  ra.x = static_cast<const __nv_bfloat16*>(x);
  ra.router_w = static_cast<const __nv_bfloat16*>(router_w);
  ra.bias = s.router_bias;
  ra.B = batch;
  ra.H = s.hidden;
  ra.E = s.n_experts;
  ra.k = s.top_k;
  ra.G = router_grid(h, batch);
  ra.chunk_rows = h->router_chunk_rows;
  ra.logits = h->at<float>(h->L.logits);
  ra.logits_stride = s.max_batch * s.n_experts;
  ra.epoch = h->at<unsigned>(h->L.router_epoch);
  ra.ticket = h->at<unsigned>(h->L.ticket);
  ra.plan = h->at<Plan>(h->L.plan);
  ra.topk_ids = topk_ids;
  ra.topk_w = topk_w;
  ra.status = status;
  ra.spin_limit = h->spin_limit;
  auto launch_router = [&]() -> cudaError_t {
    cudaError_t err = mark(0, sm);
    if (err != cudaSuccess) return err;
    err = launch(pick_router(s.n_experts), ra.G, router_threads_for(s.n_experts),
                 moe::router_smem_bytes(batch, s.n_experts, h->router_chunk_rows), sm, true, ra);
    if (err != cudaSuccess) return err;
    ++kernels;
    return mark(1, sm);
  };

  auto launch_combine = [&](bool pdl) -> cudaError_t {
    cudaError_t err;
    if (s.flags & MOE_FLAG_PARTIAL_SUM) {  // the fp32 expert sum alone
      const int nvec4 = batch * s.hidden / 4;
      err = launch(moe::partial_sum_kernel, ceil_div(nvec4, 256), 256, 0, sm, pdl, base.acc, static_cast<float*>(out),
                   nvec4);
    } else {
      const int nvec = batch * s.hidden / 8;
      err = launch(moe::combine_residual_kernel, ceil_div(nvec, 256), 256, 0, sm, pdl,
                   static_cast<const __nv_bfloat16*>(x), base.acc, static_cast<__nv_bfloat16*>(out), nvec);
    }
    if (err != cudaSuccess) return err;
    ++kernels;
    return mark(3, sm);
  };

  if (!two_stream) {
    // -------------------------------------------- default: three kernels
    MmaArgs ma = base;
    ma.n_su = n_su;
    ma.has_routed = 1;
    if ((e = launch_router()) != cudaSuccess) return bail(e);
    if ((e = mark(4, sm)) != cudaSuccess) return bail(e);
    e = launch(mlp, h->grid_routed, mlp_threads, smem, sm, true, ma, *h->tab13, *h->tab2);
    if (e != cudaSuccess) return bail(e);
    ++kernels;
    if ((e = mark(2, sm)) != cudaSuccess || (e = mark(5, sm)) != cudaSuccess) return bail(e);
    if ((e = launch_combine(true)) != cudaSuccess) return bail(e);
  } else {
    // ------------------------------------ MOE_FLAG_TWO_STREAM: four kernels
    // Shared expert (weight 1, all tokens): on stream_aux, forked after the
    // router is enqueued so the router's CTAs are dispatched first.  Its grid
    // is sized to its share of the bytes (the rest of the SMs stream routed
    // experts), so both finish together instead of contending for every SM.
    auto launch_shared = [&](cudaStream_t st_sh) -> cudaError_t {
      MmaArgs ga = base;
      ga.n_su = n_su;
      ga.has_routed = 0;
      ga.queue = h->at<unsigned>(h->L.queue_s);
      ga.hold_panel = -1;
      cudaError_t err = mark(4, st_sh);
      if (err != cudaSuccess) return err;
      err = launch(mlp, shared_grid(h, batch), mlp_threads, smem, st_sh, false, ga, *h->tab_none, *h->tab_none);
      if (err != cudaSuccess) return err;
      ++kernels;
      return mark(5, st_sh);
    };
    if (fork) {
      if ((e = cudaEventRecord(h->ev_fork, sm)) != cudaSuccess) return bail(e);
      if ((e = cudaStreamWaitEvent(sa, h->ev_fork, 0)) != cudaSuccess) return bail(e);
    }
    if ((e = launch_router()) != cudaSuccess) return bail(e);
    if (fork) {
      if ((e = launch_shared(sa)) != cudaSuccess) return bail(e);
      if ((e = cudaEventRecord(h->ev_join, sa)) != cudaSuccess) return bail(e);
    }
    // Routed experts: UP + SwiGLU + DOWN in one persistent launch.
    MmaArgs ma = base;
    ma.n_su = 0;
    ma.has_routed = 1;
    int g_routed = h->grid_routed;
    if (fork && h->grid_routed_auto) {
      g_routed = h->num_sms - shared_grid(h, batch);
      if (g_routed < 1) g_routed = 1;
    }
    e = launch(mlp, g_routed, mlp_threads, smem, sm, true, ma, *h->tab13, *h->tab2);
    if (e != cudaSuccess) return bail(e);
    ++kernels;
    if ((e = mark(2, sm)) != cudaSuccess) return bail(e);
    if (s.n_shared && !fork) {
      if ((e = launch_shared(sm)) != cudaSuccess) return bail(e);
    }
    if (fork) {
      if ((e = cudaStreamWaitEvent(sm, h->ev_join, 0)) != cudaSuccess) return bail(e);
    }
    if ((e = launch_combine(!fork)) != cudaSuccess) return bail(e);
  }

  {
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if ((e = cudaStreamIsCapturing(sm, &cap)) != cudaSuccess) return fail_cuda(e);
    if (cap == cudaStreamCaptureStatusNone) {
      if ((e = cudaEventRecord(h->ev_done, sm)) != cudaSuccess) return fail_cuda(e);
      h->done_recorded = true;
      h->captured_last = false;
    } else {
      h->captured_last = true;
    }
  }
  h->stats.forwards += 1;
  h->stats.kernels_launched += (uint64_t)kernels;
  h->stats.last_kernels = kernels;
  h->stats.last_token_tiles = ((batch < moe::kMaxUnitTokens ? batch : moe::kMaxUnitTokens) + 7) / 8;
  return MOE_OK;
}

int check_forward_args(moe_decode_ctx* h, const void* x, const void* router_w, const void* const* w13,
                       const void* const* w2, const void* shared_w13, const void* shared_w2, const void* out,
                       const void* topk_ids, const void* topk_w, int batch, bool device_io) {
  if (!h) return MOE_ERR_INVALID_ARG;
  const moe_decode_shapes& s = h->s;
  if (batch < 0 || batch > s.max_batch) return MOE_ERR_INVALID_ARG;
  if (batch == 0) return MOE_OK;  // nothing is read or written
  if (!x || !router_w || !w13 || !w2 || !out || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if (device_io) {
    if (!aligned16(x) || !aligned16(out) || !aligned4(topk_ids) || !aligned4(topk_w)) return MOE_ERR_INVALID_ARG;
    if (x == out) return MOE_ERR_INVALID_ARG;
  }
  if (!aligned16(router_w)) return MOE_ERR_INVALID_ARG;
  if (s.n_shared) {
    if (!shared_w13 || !shared_w2 || !aligned16(shared_w13) || !aligned16(shared_w2)) return MOE_ERR_INVALID_ARG;
  }
  if (s.router_bias && !aligned4(s.router_bias)) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < s.n_experts; ++i) {
    if (!w13[i] || !w2[i] || !aligned16(w13[i]) || !aligned16(w2[i])) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

struct DeviceGuard {
  int prev = -1;
  bool ok = true;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) {
      prev = -1;
      ok = false;
      return;
    }
    if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
  }
  ~DeviceGuard() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// Wait until the handle's enqueued work is done: the event recorded at the
// end of its last forward enqueued outside capture.  When the last forward
// was captured into a graph, its replays run on streams the handle never
// sees, so the whole device is synchronised instead.  Runs with the handle's
// device current.
int wait_for_handle_work(moe_decode_ctx* h) {
  cudaError_t e = cudaSuccess;
  if (h->captured_last)
    e = cudaDeviceSynchronize();
  else if (h->done_recorded)
    e = cudaEventSynchronize(h->ev_done);
  return e == cudaSuccess ? MOE_OK : fail_cuda(e);
}

int enqueue_forward(moe_decode_ctx* h, const void* x, const void* router_w, const void* const* w13,
                    const void* const* w2, const void* shared_w13, const void* shared_w2, void* out,
                    int32_t* topk_ids, float* topk_w, int batch, cudaStream_t sm, cudaStream_t sa,
                    const Fp8Scales* f8);
int refresh_maps(moe_decode_ctx* h, const void* const* w13, const void* const* w2, const void* sw13,
                 const void* sw2, cudaStream_t sm);

// moe_decode_forward_host with every host buffer pinned and mapped: [copy x
// in; the forward, storing its results into the mapped buffers] as one CUDA
// graph, captured on the first call and replayed while the arguments (every
// pointer, the batch, the streams and the wait limit) stay the same -- one
// graph launch instead of a copy and two or three kernel launches with
// kilobytes of parameters each.  Synchronises stream_main.  Returns
// MOE_ERR_UNSUPPORTED_SHAPE when the stream cannot be captured (for example
// it is already being captured), and the caller then runs eagerly.
int forward_host_graph(moe_decode_ctx* h, const void* x_host, const void* router_w, const void* const* w13,
                       const void* const* w2, const void* sw13, const void* sw2, void* out_d, void* ids_d,
                       void* w_d, int batch, cudaStream_t sm, cudaStream_t sa) {
  const int E = h->s.n_experts;
  std::vector<const void*> key;
  key.reserve(2 * (size_t)E + 12);
  key.insert(key.end(), {x_host, router_w, sw13, sw2, out_d, ids_d, w_d, (const void*)sm, (const void*)sa,
                         reinterpret_cast<const void*>((uintptr_t)h->spin_limit)});
  key.insert(key.end(), w13, w13 + E);
  key.insert(key.end(), w2, w2 + E);
  cudaError_t e;
  if (h->dirty) {  // state to re-zero after a device error: not part of the graph
    if ((e = cudaMemsetAsync(h->ws, 0, h->L.state_end, sm)) != cudaSuccess) return fail_cuda(e);
    h->dirty = false;
  }
  if (!h->host_exec || batch != h->host_key_batch || key != h->host_key) {
    // the legacy default stream cannot be captured; nor can a stream that is
    // already being captured
    if (sm == nullptr || sm == cudaStreamLegacy) return MOE_ERR_UNSUPPORTED_SHAPE;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(sm, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone) {
      cudaGetLastError();
      return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    if (h->use_tmap) {  // upload changed tensor maps eagerly, not from inside the graph
      const int rc = refresh_maps(h, w13, w2, sw13, sw2, sm);
      if (rc != MOE_OK) return rc;
    }
    if (cudaStreamBeginCapture(sm, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_UNSUPPORTED_SHAPE;
    }
    const size_t xb = (size_t)batch * h->s.hidden * 2;
    int rc = MOE_OK;
    e = cudaMemcpyAsync(h->ws + h->L.x_stage, x_host, xb, cudaMemcpyHostToDevice, sm);
    if (e != cudaSuccess) rc = fail_cuda(e);
    const uint64_t fw = h->stats.forwards, kl = h->stats.kernels_launched;
    if (rc == MOE_OK)
      rc = enqueue_forward(h, h->ws + h->L.x_stage, router_w, w13, w2, sw13, sw2, out_d,
                           static_cast<int32_t*>(ids_d), static_cast<float*>(w_d), batch, sm, sa, nullptr);
    h->stats.forwards = fw;  // counted below, once per launch
    h->stats.kernels_launched = kl;
    cudaGraph_t g = nullptr;
    e = cudaStreamEndCapture(sm, &g);
    if (rc != MOE_OK || e != cudaSuccess) {
      if (g) cudaGraphDestroy(g);
      cudaGetLastError();
      h->host_key.clear();
      return rc != MOE_OK ? rc : fail_cuda(e);
    }
    if (h->host_exec) {
      cudaGraphExecUpdateResultInfo info{};
      if (cudaGraphExecUpdate(h->host_exec, g, &info) != cudaSuccess) {
        cudaGetLastError();
        cudaGraphExecDestroy(h->host_exec);
        h->host_exec = nullptr;
      }
    }
    if (!h->host_exec && (e = cudaGraphInstantiate(&h->host_exec, g, 0)) != cudaSuccess) {
      cudaGraphDestroy(g);
      h->host_exec = nullptr;
      h->host_key.clear();
      return fail_cuda(e);
    }
    cudaGraphDestroy(g);
    h->host_key.swap(key);
    h->host_key_batch = batch;
    h->host_graph_kernels = h->stats.last_kernels;
  }
  if ((e = cudaGraphLaunch(h->host_exec, sm)) != cudaSuccess) {
    h->dirty = true;
    return fail_cuda(e);
  }
  if ((e = cudaEventRecord(h->ev_done, sm)) != cudaSuccess) return fail_cuda(e);
  h->done_recorded = true;
  h->captured_last = false;
  h->stats.forwards += 1;
  h->stats.kernels_launched += (uint64_t)h->host_graph_kernels;
  h->stats.last_kernels = h->host_graph_kernels;
  if ((e = cudaStreamSynchronize(sm)) != cudaSuccess) return fail_cuda(e);
  return MOE_OK;
}

}  // namespace

// ---------------------------------------------------------------------------
// Router + top-k without a handle and without any allocation.
//
// Its scratch (status word, ticket, fp32 logit accumulators for up to
// MOE_NOALLOC_MAX_BATCH x MOE_NOALLOC_MAX_EXPERTS, and the bucketing plan
// the kernel also writes) lives in the file-scope device array below, which
// every GPU that loads this library keeps until the process exits (~300 KB).
// Host code must not hand the array's name to a kernel -- on the host it is
// only a stand-in -- so the device address is looked up once per device with
// cudaGetSymbolAddress and cached.
namespace {

constexpr size_t kNoAllocLogitsOff = 256;  // bytes [0,4): status, [4,8): ticket
constexpr size_t kNoAllocPlanOff =
    kNoAllocLogitsOff + (size_t)MOE_NOALLOC_MAX_BATCH * MOE_NOALLOC_MAX_EXPERTS * sizeof(float);
constexpr size_t kNoAllocBytes = (kNoAllocPlanOff + sizeof(Plan) + 255) / 256 * 256;
constexpr int kNoAllocMaxDevices = 64;

struct NoAllocDevice {
  bool ready = false;
  uint8_t* scratch = nullptr;
  int num_sms = 0;
};

std::mutex g_noalloc_mu;
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

}  // namespace

static __device__ __align__(256) uint8_t g_router_scratch[kNoAllocBytes];

namespace {

// First call on a device: resolve the scratch address, zero it once, read the
// SM count.  Runs with `dev` current.
int noalloc_setup(int dev, NoAllocDevice** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocDevice& d = g_noalloc_dev[dev];
  if (!d.ready) {
    int major = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e != cudaSuccess) return fail_cuda(e);
    if (major != 10) return MOE_ERR_ARCH;
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_router_scratch)) != cudaSuccess) return fail_cuda(e);
    if ((e = cudaMemset(p, 0, kNoAllocBytes)) != cudaSuccess) return fail_cuda(e);
    if ((e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return fail_cuda(e);
    d.scratch = static_cast<uint8_t*>(p);
    d.ready = true;
  }
  *out = &d;
  return MOE_OK;
}

}  // namespace

extern "C" {

int moe_router_topk_noalloc(const void* x, const void* router_w, const float* router_bias, int32_t* topk_ids,
                            float* topk_w, int32_t batch, int32_t hidden, int32_t n_experts, int32_t top_k,
                            void* stream) {
  if (batch < 0 || batch > MOE_NOALLOC_MAX_BATCH) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (hidden < 8 || hidden > 16384 || hidden % 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (n_experts < 8 || n_experts > MOE_NOALLOC_MAX_EXPERTS || n_experts % 8) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (top_k < 1 || top_k > moe::kMaxTopK || top_k > n_experts) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (batch == 0) return MOE_OK;
  if (!x || !router_w || !topk_ids || !topk_w) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(router_w) || !aligned4(topk_ids) || !aligned4(topk_w)) return MOE_ERR_INVALID_ARG;
  if (router_bias && !aligned4(router_bias)) return MOE_ERR_INVALID_ARG;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  NoAllocDevice* d = nullptr;
  int rc = noalloc_setup(dev, &d);
  if (rc != MOE_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // The scratch keeps the previous call's contents: the status word, the
  // ticket and this call's logit accumulators must start at zero.
  const size_t clear = kNoAllocLogitsOff + (size_t)batch * n_experts * sizeof(float);
  if ((e = cudaMemsetAsync(d->scratch, 0, clear, st)) != cudaSuccess) return fail_cuda(e);

  RouterArgs ra{};
  ra.x = static_cast<const __nv_bfloat16*>(x);
  ra.router_w = static_cast<const __nv_bfloat16*>(router_w);
  ra.bias = router_bias;
  ra.B = batch;
  ra.H = hidden;
  ra.E = n_experts;
  ra.k = top_k;
  int g = d->num_sms < hidden / 8 ? d->num_sms : hidden / 8;
  ra.G = g < 1 ? 1 : g;
  const int rows = ceil_div(hidden, ra.G);
  const int cap_rows = 65536 / (2 * n_experts + 4 * moe::router_bpad(batch));
  ra.chunk_rows = rows < cap_rows ? rows : cap_rows;
  if (ra.chunk_rows < 1) ra.chunk_rows = 1;
  ra.status = reinterpret_cast<int*>(d->scratch);
  ra.ticket = reinterpret_cast<unsigned*>(d->scratch + 4);
  ra.logits = reinterpret_cast<float*>(d->scratch + kNoAllocLogitsOff);
  ra.plan = reinterpret_cast<Plan*>(d->scratch + kNoAllocPlanOff);
  ra.topk_ids = topk_ids;
  ra.topk_w = topk_w;
  ra.spin_limit = moe::kSpinLimit;
  const size_t smem = moe::router_smem_bytes(batch, n_experts, ra.chunk_rows);
  cudaFuncAttributes fa{};
  const RouterKernel rk = pick_router(n_experts);
  if ((e = cudaFuncGetAttributes(&fa, rk)) != cudaSuccess) return fail_cuda(e);
  if ((size_t)fa.maxDynamicSharedSizeBytes < smem) {
    e = cudaFuncSetAttribute(rk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail_cuda(e);
  }
  e = launch(rk, ra.G, router_threads_for(n_experts), smem, st, false, ra);
  if (e != cudaSuccess) return fail_cuda(e);
  return MOE_OK;
}

int moe_router_topk_noalloc_status(void* stream) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail_cuda(e);
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MOE_ERR_NO_DEVICE;
  uint8_t* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_dev[dev].ready) scratch = g_noalloc_dev[dev].scratch;
  }
  if (!scratch) return MOE_OK;  // no call has run on this device
  if ((e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream))) != cudaSuccess) return fail_cuda(e);
  int st = 0;
  if ((e = cudaMemcpy(&st, scratch, sizeof st, cudaMemcpyDeviceToHost)) != cudaSuccess) return fail_cuda(e);
  if (st == moe::kStatusOk) return MOE_OK;
  if ((e = cudaMemset(scratch, 0, sizeof st)) != cudaSuccess) return fail_cuda(e);
  return st == moe::kStatusTimeout ? MOE_ERR_DEVICE_TIMEOUT : MOE_ERR_DEVICE_PLAN;
}

uint64_t moe_decode_workspace_bytes(const moe_decode_shapes* shapes) {
  if (!shapes_valid(shapes)) return 0;
  return (uint64_t)layout_for(shapes).total;
}

int moe_decode_init(const moe_decode_shapes* shapes, moe_decode_t* out_handle) {
  if (!out_handle) return MOE_ERR_INVALID_ARG;
  *out_handle = nullptr;
  if (!shapes) return MOE_ERR_INVALID_ARG;
  if (!shapes_valid(shapes)) return MOE_ERR_UNSUPPORTED_SHAPE;
  int ndev = 0;
  cudaError_t e = cudaGetDeviceCount(&ndev);
  if (e != cudaSuccess || ndev == 0) {
    g_last_cuda_error = (int)e;
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return fail_cuda(e);
  cudaDeviceProp prop;
  if ((e = cudaGetDeviceProperties(&prop, dev)) != cudaSuccess) return fail_cuda(e);
  if (prop.major != 10) return MOE_ERR_ARCH;

  moe_decode_ctx* h = new (std::nothrow) moe_decode_ctx();
  if (!h) return MOE_ERR_OUT_OF_MEMORY;
  h->s = *shapes;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->n_stages = env_int("MOE_DECODE_STAGES", 3, 2, moe::kMaxStagesMma);
  // the deepest rings that fit the opt-in shared memory of a block
  const size_t smem_max = prop.sharedMemPerBlockOptin;
  while (h->n_stages > 2 && moe::mma_smem_bytes(h->n_stages) > smem_max) --h->n_stages;
  h->n_stages_tc = h->n_stages;
  while (h->n_stages_tc > 2 && moe::tc_smem_bytes(h->n_stages_tc) > smem_max) --h->n_stages_tc;
  h->grid_routed = env_int("MOE_DECODE_GRID_ROUTED", 0, 0, 8 * h->num_sms);
  h->grid_routed_auto = h->grid_routed == 0;
  if (h->grid_routed == 0) h->grid_routed = h->num_sms;
  h->grid_shared = env_int("MOE_DECODE_GRID_SHARED", 0, 0, 8 * h->num_sms);  // 0: sized per call
  h->host_graph_on = env_int("MOE_DECODE_HOST_GRAPH", 1, 0, 1) == 1;
  h->stagger = env_int("MOE_DECODE_STAGGER", 8, 0, moe::kMaxChunk);
  {
    int gr = env_int("MOE_DECODE_ROUTER_CTAS", h->num_sms, 1, h->num_sms);
    const int cap = shapes->hidden / 8;
    h->grid_router_max = gr < cap ? gr : cap;
    if (h->grid_router_max < 1) h->grid_router_max = 1;
    const int rows = ceil_div(shapes->hidden, h->grid_router_max);
    const int cap_rows = 65536 / (2 * shapes->n_experts + 4 * moe::router_bpad(shapes->max_batch));
    h->router_chunk_rows = rows < cap_rows ? rows : cap_rows;
    if (h->router_chunk_rows < 1) h->router_chunk_rows = 1;
  }
  h->L = layout_for(shapes);
  h->tab13 = new (std::nothrow) ExpertTable();
  h->tab2 = new (std::nothrow) ExpertTable();
  h->tab_none = new (std::nothrow) ExpertTable();
  if (!h->tab13 || !h->tab2 || !h->tab_none) {
    delete h->tab13;
    delete h->tab2;
    delete h->tab_none;
    delete h;
    return MOE_ERR_OUT_OF_MEMORY;
  }
  int rc = MOE_OK;
  e = cudaMalloc(reinterpret_cast<void**>(&h->ws), h->L.total);
  if (e != cudaSuccess) {
    g_last_cuda_error = (int)e;
    cudaGetLastError();
    rc = MOE_ERR_OUT_OF_MEMORY;
  }
  if (rc == MOE_OK && (e = cudaMemset(h->ws, 0, h->L.total)) != cudaSuccess) rc = fail_cuda(e);
  if (rc == MOE_OK && (e = cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming)) != cudaSuccess)
    rc = fail_cuda(e);
  if (rc == MOE_OK && (e = cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming)) != cudaSuccess)
    rc = fail_cuda(e);
  if (rc == MOE_OK && (e = cudaEventCreateWithFlags(&h->ev_maps, cudaEventDisableTiming)) != cudaSuccess)
    rc = fail_cuda(e);
  if (rc == MOE_OK && (e = cudaEventCreateWithFlags(&h->ev_done, cudaEventDisableTiming)) != cudaSuccess)
    rc = fail_cuda(e);
  if (rc == MOE_OK) {
    // tensor-map path: shapes in whole 64-column chunks and a working encoder
    const bool shapes_ok = shapes->hidden % moe::kChunkCols == 0 && shapes->inter % moe::kChunkCols == 0 &&
                           (!shapes->n_shared || shapes->shared_inter % moe::kChunkCols == 0);
    uint8_t probe[moe::kTensorMapBytes];
    h->use_tmap = env_int("MOE_DECODE_TMAP", 1, 0, 1) == 1 && shapes_ok &&
                  encode_matrix_map(probe, h->ws, shapes->hidden, 2 * shapes->inter);
    h->use_tc = h->use_tmap && (shapes->flags & MOE_FLAG_TCGEN05) != 0;
    if (h->use_tmap) {
      const size_t nm = 2 * (size_t)shapes->n_experts + 2;
      h->map_ptrs.assign(nm, nullptr);
      e = cudaMallocHost(reinterpret_cast<void**>(&h->maps_host), nm * moe::kTensorMapBytes);
      if (e != cudaSuccess) rc = fail_cuda(e);
    }
  }
  if (rc == MOE_OK) rc = set_kernel_attrs(h);
  if (rc != MOE_OK) {
    moe_decode_destroy(h);
    return rc;
  }
  *out_handle = h;
  return MOE_OK;
}

int moe_decode_forward(moe_decode_t h, const void* x, const void* router_w, const void* const* w13,
                       const void* const* w2, const void* shared_w13, const void* shared_w2, void* out,
                       int32_t* topk_ids, float* topk_w, int32_t batch, void* stream_main, void* stream_aux) {
  int rc = check_forward_args(h, x, router_w, w13, w2, shared_w13, shared_w2, out, topk_ids, topk_w, batch, true);
  if (rc != MOE_OK) return rc;
  if (batch == 0) return MOE_OK;
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail_cuda(cudaGetLastError());
  if (h->s.flags & MOE_FLAG_FP8_WEIGHTS) return MOE_ERR_INVALID_ARG;  // moe_decode_forward_fp8
  return enqueue_forward(h, x, router_w, w13, w2, shared_w13, shared_w2, out, topk_ids, topk_w, batch,
                         static_cast<cudaStream_t>(stream_main), static_cast<cudaStream_t>(stream_aux), nullptr);
}

int moe_decode_forward_fp8(moe_decode_t h, const void* x, const void* router_w, const void* const* w13q,
                           const void* const* w13s, const void* const* w2q, const void* const* w2s,
                           const void* shared_w13q, const void* shared_w13s, const void* shared_w2q,
                           const void* shared_w2s, void* out, int32_t* topk_ids, float* topk_w, int32_t batch,
                           void* stream_main, void* stream_aux) {
  if (!h || !(h->s.flags & MOE_FLAG_FP8_WEIGHTS) || !h->use_tmap) return MOE_ERR_INVALID_ARG;
  int rc = check_forward_args(h, x, router_w, w13q, w2q, shared_w13q, shared_w2q, out, topk_ids, topk_w, batch, true);
  if (rc != MOE_OK) return rc;
  if (batch == 0) return MOE_OK;
  if (!w13s || !w2s) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < h->s.n_experts; ++i)
    if (!w13s[i] || !w2s[i] || !aligned16(w13s[i]) || !aligned16(w2s[i])) return MOE_ERR_INVALID_ARG;
  if (h->s.n_shared && (!shared_w13s || !shared_w2s || !aligned16(shared_w13s) || !aligned16(shared_w2s)))
    return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail_cuda(cudaGetLastError());
  const Fp8Scales f8{w13s, w2s, shared_w13s, shared_w2s};
  return enqueue_forward(h, x, router_w, w13q, w2q, shared_w13q, shared_w2q, out, topk_ids, topk_w, batch,
                         static_cast<cudaStream_t>(stream_main), static_cast<cudaStream_t>(stream_aux), &f8);
}

int moe_decode_forward_host(moe_decode_t h, const void* x_host, const void* router_w, const void* const* w13,
                            const void* const* w2, const void* shared_w13, const void* shared_w2,
                            void* out_host, int32_t* ids_host, float* w_host, int32_t batch, void* stream_main,
                            void* stream_aux) {
  if (h && (h->s.flags & MOE_FLAG_FP8_WEIGHTS)) return MOE_ERR_INVALID_ARG;  // bf16 weights only
  if (h && (h->s.flags & MOE_FLAG_PARTIAL_SUM)) return MOE_ERR_INVALID_ARG;  // bf16 out only
  int rc = check_forward_args(h, x_host, router_w, w13, w2, shared_w13, shared_w2, out_host, ids_host, w_host,
                              batch, false);
  if (rc != MOE_OK) return rc;
  if (batch == 0) return MOE_OK;
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail_cuda(cudaGetLastError());
  cudaStream_t sm = static_cast<cudaStream_t>(stream_main);
  const size_t xb = (size_t)batch * h->s.hidden * 2;
  const size_t kb = (size_t)batch * h->s.top_k * 4;
  void* xd = h->at<void>(h->L.x_stage);
  void* od = h->at<void>(h->L.out_stage);
  int32_t* idd = h->at<int32_t>(h->L.ids_stage);
  float* wd = h->at<float>(h->L.w_stage);
  // Outputs: when all three host buffers are pinned and mapped, the router
  // and the combine kernel store into them directly (their writes cross the
  // host link as the kernels run; no copies and no copy latencies after the
  // last kernel); otherwise through device staging and three copies.
  void* od_m = host_buffer_device_view(out_host, 16);
  void* idd_m = od_m ? host_buffer_device_view(ids_host, 4) : nullptr;
  void* wd_m = idd_m ? host_buffer_device_view(w_host, 4) : nullptr;
  const bool direct = od_m && idd_m && wd_m;
  cudaError_t e;
  // Graph path: everything pinned and mapped (a copy from pageable memory
  // cannot be captured), no per-kernel timing, not testing a held panel.
  if (direct && h->host_graph_on && !h->timing && !(h->s.flags & MOE_FLAG_TEST_HOLD_PANEL) &&
      host_buffer_device_view(const_cast<void*>(x_host), 16)) {
    rc = forward_host_graph(h, x_host, router_w, w13, w2, shared_w13, shared_w2, od_m, idd_m, wd_m, batch, sm,
                            static_cast<cudaStream_t>(stream_aux));
    if (rc != MOE_ERR_UNSUPPORTED_SHAPE) return rc;  // else: capture not possible here, run eagerly
  }
  if ((e = cudaMemcpyAsync(xd, x_host, xb, cudaMemcpyHostToDevice, sm)) != cudaSuccess) return fail_cuda(e);
  rc = enqueue_forward(h, xd, router_w, w13, w2, shared_w13, shared_w2, direct ? od_m : od,
                       static_cast<int32_t*>(direct ? idd_m : idd), static_cast<float*>(direct ? wd_m : wd), batch,
                       sm, static_cast<cudaStream_t>(stream_aux), nullptr);
  if (rc != MOE_OK) return rc;
  if (!direct) {
    if ((e = cudaMemcpyAsync(out_host, od, xb, cudaMemcpyDeviceToHost, sm)) != cudaSuccess) return fail_cuda(e);
    if ((e = cudaMemcpyAsync(ids_host, idd, kb, cudaMemcpyDeviceToHost, sm)) != cudaSuccess) return fail_cuda(e);
    if ((e = cudaMemcpyAsync(w_host, wd, kb, cudaMemcpyDeviceToHost, sm)) != cudaSuccess) return fail_cuda(e);
  }
  if ((e = cudaStreamSynchronize(sm)) != cudaSuccess) return fail_cuda(e);
  return MOE_OK;
}

int moe_decode_reduce_residual(const void* const* partials, int32_t n_parts, const void* x, void* out,
                               int32_t batch, int32_t hidden, void* stream) {
  static_assert(MOE_REDUCE_MAX_PARTS == moe::kMaxReduceParts, "partials per reduction");
  if (!partials || !x || !out) return MOE_ERR_INVALID_ARG;
  if (n_parts < 1 || n_parts > MOE_REDUCE_MAX_PARTS) return MOE_ERR_INVALID_ARG;
  if (batch < 1 || batch > moe::kMaxBatch || hidden < 8 || hidden > 16384 || hidden % 8) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  moe::PartialPtrs pp{};
  for (int r = 0; r < n_parts; ++r) {
    if (!partials[r] || !aligned16(partials[r])) return MOE_ERR_INVALID_ARG;
    pp.p[r] = static_cast<const float*>(partials[r]);
  }
  int ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  const int nvec = batch * hidden / 8;
  const cudaError_t e =
      launch(moe::reduce_residual_kernel, ceil_div(nvec, 256), 256, 0, static_cast<cudaStream_t>(stream), false, pp,
             (int)n_parts, static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(out), nvec);
  return e == cudaSuccess ? MOE_OK : fail_cuda(e);
}

int moe_decode_destroy(moe_decode_t h) {
  if (!h) return MOE_OK;
  int rc = MOE_OK;
  {
    DeviceGuard guard(h->device);
    if (h->ws) {
      const int wrc = wait_for_handle_work(h);
      if (wrc != MOE_OK) rc = wrc;
      cudaFree(h->ws);
    }
    if (h->host_exec) cudaGraphExecDestroy(h->host_exec);
    if (h->ev_done) cudaEventDestroy(h->ev_done);
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
    if (h->ev_maps) cudaEventDestroy(h->ev_maps);
    if (h->maps_host) cudaFreeHost(h->maps_host);
  }
  delete h->tab13;
  delete h->tab2;
  delete h->tab_none;
  delete h;
  return rc;
}

int moe_decode_get_status(moe_decode_t h) {
  if (!h) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  const int wrc = wait_for_handle_work(h);
  if (wrc != MOE_OK) return wrc;
  cudaError_t e;
  int st = 0;
  int* dst = h->at<int>(h->L.status);
  if ((e = cudaMemcpy(&st, dst, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess) return fail_cuda(e);
  if (st == moe::kStatusOk) return MOE_OK;
  // The workspace may be inconsistent after a device-side failure: clear
  // the status now and re-zero everything at the next forward.
  if ((e = cudaMemset(dst, 0, sizeof(int))) != cudaSuccess) return fail_cuda(e);
  h->dirty = true;
  return st == moe::kStatusTimeout ? MOE_ERR_DEVICE_TIMEOUT : MOE_ERR_DEVICE_PLAN;
}

int moe_decode_set_timing_events(moe_decode_t h, void* const* events, int32_t n_events) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (!events || n_events == 0) {
    h->timing = false;
    return MOE_OK;
  }
  if (n_events != MOE_TIMING_EVENTS) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < MOE_TIMING_EVENTS; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < MOE_TIMING_EVENTS; ++i) h->tev[i] = static_cast<cudaEvent_t>(events[i]);
  h->timing = true;
  return MOE_OK;
}

int moe_decode_get_stats(moe_decode_t h, moe_decode_stats* stats) {
  if (!h || !stats) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  const int wrc = wait_for_handle_work(h);
  if (wrc != MOE_OK) return wrc;
  unsigned long long c[2 * moe::kNumClasses] = {};
  cudaError_t e = cudaMemcpy(c, h->ws + h->L.stage_counts, sizeof c, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return fail_cuda(e);
  *stats = h->stats;
  for (int i = 0; i < moe::kNumClasses; ++i) {
    stats->stages_up[i] = c[2 * i];
    stats->stages_down[i] = c[2 * i + 1];
  }
  return MOE_OK;
}

int moe_decode_set_wait_limit(moe_decode_t h, uint32_t probes) {
  if (!h) return MOE_ERR_INVALID_ARG;
  h->spin_limit = probes == 0 ? moe::kSpinLimit : probes;
  return MOE_OK;
}

const char* moe_decode_error_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_NO_DEVICE: return "no CUDA device";
    case MOE_ERR_ARCH: return "device is not compute capability 10.x";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_OUT_OF_MEMORY: return "out of memory";
    case MOE_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MOE_ERR_DEVICE_PLAN: return "device-side consistency check failed";
    default: return "unknown error code";
  }
}

int moe_decode_last_cuda_error(void) { return g_last_cuda_error; }

const char* moe_decode_last_cuda_error_string(void) {
  return cudaGetErrorName(static_cast<cudaError_t>(g_last_cuda_error));
}

}  // extern "C"
