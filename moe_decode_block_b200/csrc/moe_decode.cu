// moe_decode.cu -- host side of the C ABI declared in include/moe_decode.h.
//
// One forward enqueues six kernels:
//   stream_aux : shared-expert UP, shared-expert DOWN          (weight 1)
//   stream_main: router+top-k+plan, routed UP, routed DOWN, [join] combine
// The shared expert is forked from stream_main with an event and joined back
// before the combine (pages: "Hyper Optimizing Kimi K3 in vLLM", section
// "Recovering time between operators": the shared expert runs on another
// stream, overlapping routing and the selected experts).  Consecutive kernels
// on one stream use programmatic dependent launch so the next kernel's CTAs
// start (and prefetch static weights) while the previous one drains.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>

#include "moe_decode.h"
#include "expert_gemv.cuh"
#include "moe_device.cuh"
#include "router_topk.cuh"

namespace {

using moe::ExpertTable;
using moe::GemvArgs;
using moe::Plan;
using moe::RouterArgs;

thread_local int g_last_cuda_error = 0;

struct Geom {
  int K, N, I, panel_w, n_cp, stage_rows;
};

struct WorkspaceLayout {
  size_t status, ticket, logits, plan, h, a, counters, h_s, a_s, counters_s, acc, x_stage, out_stage,
      ids_stage, w_stage, total;
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Column panels and stage rows of one projection.  UP panels pair gate
// column c with up column I + c; each panel has at most kMaxPanelCols local
// columns.  stage_rows is the largest power of two (<= 64) whose rows fit
// one 32 KB stage.
Geom make_geom(bool up, int K, int cols) {
  Geom g{};
  g.K = K;
  const int maxw = up ? moe::kMaxPanelCols / 2 : moe::kMaxPanelCols;
  g.N = up ? 2 * cols : cols;
  g.I = up ? cols : 0;
  g.n_cp = ceil_div(cols, maxw);
  g.panel_w = ceil_div(ceil_div(cols, g.n_cp), 8) * 8;
  const int lw = up ? 2 * g.panel_w : g.panel_w;
  int r = moe::kStepRows;
  while (r > 1 && (size_t)r * lw * 2 > (size_t)moe::kStageBytes) r >>= 1;
  g.stage_rows = r;
  return g;
}

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
  if (s->flags != 0) return false;
  return true;
}

WorkspaceLayout layout_for(const moe_decode_shapes* s) {
  WorkspaceLayout L{};
  const size_t A = 256;
  const size_t B = (size_t)s->max_batch, E = (size_t)s->n_experts, k = (size_t)s->top_k;
  const size_t H = (size_t)s->hidden, I = (size_t)s->inter;
  const size_t Is = s->n_shared ? (size_t)s->shared_inter : 0;
  const Geom up = make_geom(true, s->hidden, s->inter);
  const int ncp_s = s->n_shared ? make_geom(true, s->hidden, s->shared_inter).n_cp : 0;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, A);
    return o;
  };
  L.status = take(sizeof(int));
  L.ticket = take(sizeof(unsigned));
  L.logits = take(B * E * 4);
  L.plan = take(sizeof(Plan));
  L.h = take(B * k * 2 * I * 4);
  L.a = take(B * k * I * 4);
  L.counters = take(E * (size_t)up.n_cp * 4);
  L.h_s = take(B * 2 * Is * 4);
  L.a_s = take(B * Is * 4);
  L.counters_s = take((size_t)ncp_s * 4 + 4);
  L.acc = take(B * H * 4);
  L.x_stage = take(B * H * 2);
  L.out_stage = take(B * H * 2);
  L.ids_stage = take(B * k * 4);
  L.w_stage = take(B * k * 4);
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

using GemvKernel = void (*)(GemvArgs, ExpertTable);

template <bool DENSE, bool UP>
GemvKernel pick_gemv(int tg) {
  switch (tg) {
    case 1: return moe::expert_gemv_kernel<1, DENSE, UP>;
    case 2: return moe::expert_gemv_kernel<2, DENSE, UP>;
    case 4: return moe::expert_gemv_kernel<4, DENSE, UP>;
    default: return moe::expert_gemv_kernel<8, DENSE, UP>;
  }
}

inline int token_group_for(int n) { return n <= 1 ? 1 : (n <= 2 ? 2 : (n <= 4 ? 4 : 8)); }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

struct moe_decode_ctx {
  moe_decode_shapes s{};
  int device = 0;
  int num_sms = 0;
  int n_stages = 6;
  int grid_routed = 0, grid_shared = 0, grid_router_max = 0;
  int router_chunk_rows = 0;
  Geom up{}, down{}, sh_up{}, sh_down{};
  WorkspaceLayout L{};
  uint8_t* ws = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_join = nullptr;
  bool dirty = false;
  moe_decode_stats stats{};
  ExpertTable* tab13 = nullptr;  // host staging of the pointer tables (kernel parameters)
  ExpertTable* tab2 = nullptr;
  bool timing = false;
  cudaEvent_t tev[MOE_TIMING_EVENTS] = {};

  template <typename T>
  T* at(size_t off) const {
    return reinterpret_cast<T*>(ws + off);
  }
};

namespace {

int router_grid(const moe_decode_ctx* h, int batch) {
  int g = h->grid_router_max;
  if (batch > 8) {
    const int cap = h->num_sms * 8 / batch;
    g = g < cap ? g : cap;
  }
  if (g < 1) g = 1;
  return g;
}

int set_kernel_attrs(const moe_decode_ctx* h) {
  const int gemv_smem = (int)moe::gemv_smem_bytes(h->n_stages, 8);
  GemvKernel ks[] = {
      pick_gemv<false, true>(1), pick_gemv<false, true>(2), pick_gemv<false, true>(4), pick_gemv<false, true>(8),
      pick_gemv<false, false>(1), pick_gemv<false, false>(2), pick_gemv<false, false>(4), pick_gemv<false, false>(8),
      pick_gemv<true, true>(1), pick_gemv<true, true>(2), pick_gemv<true, true>(4), pick_gemv<true, true>(8),
      pick_gemv<true, false>(1), pick_gemv<true, false>(2), pick_gemv<true, false>(4), pick_gemv<true, false>(8)};
  for (GemvKernel k : ks) {
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, gemv_smem);
    if (e != cudaSuccess) return fail_cuda(e);
  }
  const int rsmem = (int)moe::router_smem_bytes(h->s.max_batch, h->s.n_experts, h->router_chunk_rows);
  cudaError_t e = cudaFuncSetAttribute(moe::router_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, rsmem);
  if (e != cudaSuccess) return fail_cuda(e);
  return MOE_OK;
}

// Enqueue the whole forward (device pointers only).
int enqueue_forward(moe_decode_ctx* h, const void* x, const void* router_w, const void* const* w13,
                    const void* const* w2, const void* shared_w13, const void* shared_w2, void* out,
                    int32_t* topk_ids, float* topk_w, int batch, cudaStream_t sm, cudaStream_t sa) {
  const moe_decode_shapes& s = h->s;
  cudaError_t e;
  int kernels = 0;
  if (h->dirty) {
    e = cudaMemsetAsync(h->ws, 0, h->L.total, sm);
    if (e != cudaSuccess) return fail_cuda(e);
    h->dirty = false;
  }
  for (int i = 0; i < s.n_experts; ++i) {
    h->tab13->p[i] = static_cast<const __nv_bfloat16*>(w13[i]);
    h->tab2->p[i] = static_cast<const __nv_bfloat16*>(w2[i]);
  }
  int* status = h->at<int>(h->L.status);
  float* acc = h->at<float>(h->L.acc);
  const bool fork = s.n_shared && sa != sm;
  const int tg = token_group_for(batch);

  auto bail = [&](cudaError_t err) {
    h->dirty = true;
    return fail_cuda(err);
  };
  auto mark = [&](int i, cudaStream_t st) {
    return h->timing ? cudaEventRecord(h->tev[i], st) : cudaSuccess;
  };

  if (s.n_shared) {
    if (fork) {
      if ((e = cudaEventRecord(h->ev_fork, sm)) != cudaSuccess) return bail(e);
      if ((e = cudaStreamWaitEvent(sa, h->ev_fork, 0)) != cudaSuccess) return bail(e);
    }
    GemvArgs ga{};
    ga.dense_w = static_cast<const __nv_bfloat16*>(shared_w13);
    ga.K = h->sh_up.K;
    ga.N = h->sh_up.N;
    ga.I = h->sh_up.I;
    ga.panel_w = h->sh_up.panel_w;
    ga.n_cp = h->sh_up.n_cp;
    ga.stage_rows = h->sh_up.stage_rows;
    ga.n_stages = h->n_stages;
    ga.batch = batch;
    ga.max_units = 1;
    ga.plan = nullptr;
    ga.x = static_cast<const __nv_bfloat16*>(x);
    ga.h = h->at<float>(h->L.h_s);
    ga.a_out = h->at<float>(h->L.a_s);
    ga.counters = h->at<unsigned>(h->L.counters_s);
    ga.status = status;
    const size_t smem = moe::gemv_smem_bytes(h->n_stages, tg);
    const cudaStream_t st_sh = fork ? sa : sm;
    if ((e = mark(5, st_sh)) != cudaSuccess) return bail(e);
    e = launch(pick_gemv<true, true>(tg), h->grid_shared, moe::kGemvThreads, smem, st_sh, false, ga, *h->tab13);
    if (e != cudaSuccess) return bail(e);
    ++kernels;
    if ((e = mark(6, st_sh)) != cudaSuccess) return bail(e);
    GemvArgs gd{};
    gd.dense_w = static_cast<const __nv_bfloat16*>(shared_w2);
    gd.K = h->sh_down.K;
    gd.N = h->sh_down.N;
    gd.I = 0;
    gd.panel_w = h->sh_down.panel_w;
    gd.n_cp = h->sh_down.n_cp;
    gd.stage_rows = h->sh_down.stage_rows;
    gd.n_stages = h->n_stages;
    gd.batch = batch;
    gd.max_units = 1;
    gd.a_in = h->at<float>(h->L.a_s);
    gd.acc = acc;
    gd.status = status;
    e = launch(pick_gemv<true, false>(tg), h->grid_shared, moe::kGemvThreads, smem, st_sh, true, gd, *h->tab2);
    if (e != cudaSuccess) return bail(e);
    ++kernels;
    if ((e = mark(7, st_sh)) != cudaSuccess) return bail(e);
    if (fork) {
      if ((e = cudaEventRecord(h->ev_join, sa)) != cudaSuccess) return bail(e);
    }
  }

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
  ra.ticket = h->at<unsigned>(h->L.ticket);
  ra.plan = h->at<Plan>(h->L.plan);
  ra.topk_ids = topk_ids;
  ra.topk_w = topk_w;
  ra.status = status;
  if ((e = mark(0, sm)) != cudaSuccess) return bail(e);
  e = launch(moe::router_topk_kernel, ra.G, moe::kRouterThreads,
             moe::router_smem_bytes(batch, s.n_experts, h->router_chunk_rows), sm, true, ra);
  if (e != cudaSuccess) return bail(e);
  ++kernels;
  if ((e = mark(1, sm)) != cudaSuccess) return bail(e);

  const size_t smem = moe::gemv_smem_bytes(h->n_stages, tg);
  GemvArgs ua{};
  ua.K = h->up.K;
  ua.N = h->up.N;
  ua.I = h->up.I;
  ua.panel_w = h->up.panel_w;
  ua.n_cp = h->up.n_cp;
  ua.stage_rows = h->up.stage_rows;
  ua.n_stages = h->n_stages;
  ua.batch = batch;
  ua.max_units = s.n_experts;
  ua.plan = h->at<Plan>(h->L.plan);
  ua.x = static_cast<const __nv_bfloat16*>(x);
  ua.h = h->at<float>(h->L.h);
  ua.a_out = h->at<float>(h->L.a);
  ua.counters = h->at<unsigned>(h->L.counters);
  ua.status = status;
  e = launch(pick_gemv<false, true>(tg), h->grid_routed, moe::kGemvThreads, smem, sm, true, ua, *h->tab13);
  if (e != cudaSuccess) return bail(e);
  ++kernels;
  if ((e = mark(2, sm)) != cudaSuccess) return bail(e);

  GemvArgs da{};
  da.K = h->down.K;
  da.N = h->down.N;
  da.I = 0;
  da.panel_w = h->down.panel_w;
  da.n_cp = h->down.n_cp;
  da.stage_rows = h->down.stage_rows;
  da.n_stages = h->n_stages;
  da.batch = batch;
  da.max_units = s.n_experts;
  da.plan = h->at<Plan>(h->L.plan);
  da.a_in = h->at<float>(h->L.a);
  da.acc = acc;
  da.status = status;
  e = launch(pick_gemv<false, false>(tg), h->grid_routed, moe::kGemvThreads, smem, sm, true, da, *h->tab2);
  if (e != cudaSuccess) return bail(e);
  ++kernels;
  if ((e = mark(3, sm)) != cudaSuccess) return bail(e);

  if (fork) {
    if ((e = cudaStreamWaitEvent(sm, h->ev_join, 0)) != cudaSuccess) return bail(e);
  }
  const int nvec = batch * s.hidden / 8;
  e = launch(moe::combine_residual_kernel, ceil_div(nvec, 256), 256, 0, sm, !fork,
             static_cast<const __nv_bfloat16*>(x), acc, static_cast<__nv_bfloat16*>(out), nvec);
  if (e != cudaSuccess) return bail(e);
  ++kernels;
  if ((e = mark(4, sm)) != cudaSuccess) return bail(e);

  h->stats.forwards += 1;
  h->stats.kernels_launched += (uint64_t)kernels;
  h->stats.last_kernels = kernels;
  h->stats.last_variant = tg;
  h->stats.variant_calls[tg == 1 ? 0 : (tg == 2 ? 1 : (tg == 4 ? 2 : 3))] += 1;
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
  if (batch > 8) {
    const int cap = d->num_sms * 8 / batch;
    g = g < cap ? g : cap;
  }
  ra.G = g < 1 ? 1 : g;
  const int rows = ceil_div(hidden, ra.G);
  const int cap_rows = 40960 / (2 * n_experts);
  ra.chunk_rows = rows < cap_rows ? rows : cap_rows;
  if (ra.chunk_rows < 1) ra.chunk_rows = 1;
  ra.status = reinterpret_cast<int*>(d->scratch);
  ra.ticket = reinterpret_cast<unsigned*>(d->scratch + 4);
  ra.logits = reinterpret_cast<float*>(d->scratch + kNoAllocLogitsOff);
  ra.plan = reinterpret_cast<Plan*>(d->scratch + kNoAllocPlanOff);
  ra.topk_ids = topk_ids;
  ra.topk_w = topk_w;
  const size_t smem = moe::router_smem_bytes(batch, n_experts, ra.chunk_rows);
  cudaFuncAttributes fa{};
  if ((e = cudaFuncGetAttributes(&fa, moe::router_topk_kernel)) != cudaSuccess) return fail_cuda(e);
  if ((size_t)fa.maxDynamicSharedSizeBytes < smem) {
    e = cudaFuncSetAttribute(moe::router_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return fail_cuda(e);
  }
  e = launch(moe::router_topk_kernel, ra.G, moe::kRouterThreads, smem, st, false, ra);
  if (e != cudaSuccess) return fail_cuda(e);
  return MOE_OK;
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
  h->n_stages = env_int("MOE_DECODE_STAGES", 6, 2, moe::kMaxStages);
  h->grid_routed = env_int("MOE_DECODE_GRID_ROUTED", h->num_sms, 1, 8 * h->num_sms);
  h->grid_shared = env_int("MOE_DECODE_GRID_SHARED", h->num_sms, 1, 8 * h->num_sms);
  {
    int gr = h->num_sms;
    const int cap = shapes->hidden / 8;
    h->grid_router_max = gr < cap ? gr : cap;
    if (h->grid_router_max < 1) h->grid_router_max = 1;
    const int rows = ceil_div(shapes->hidden, h->grid_router_max);
    const int cap_rows = 40960 / (2 * shapes->n_experts);
    h->router_chunk_rows = rows < cap_rows ? rows : cap_rows;
    if (h->router_chunk_rows < 1) h->router_chunk_rows = 1;
  }
  h->up = make_geom(true, shapes->hidden, shapes->inter);
  h->down = make_geom(false, shapes->inter, shapes->hidden);
  if (shapes->n_shared) {
    h->sh_up = make_geom(true, shapes->hidden, shapes->shared_inter);
    h->sh_down = make_geom(false, shapes->shared_inter, shapes->hidden);
  }
  h->L = layout_for(shapes);
  h->tab13 = new (std::nothrow) ExpertTable();
  h->tab2 = new (std::nothrow) ExpertTable();
  if (!h->tab13 || !h->tab2) {
    delete h->tab13;
    delete h->tab2;
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
  return enqueue_forward(h, x, router_w, w13, w2, shared_w13, shared_w2, out, topk_ids, topk_w, batch,
                         static_cast<cudaStream_t>(stream_main), static_cast<cudaStream_t>(stream_aux));
}

int moe_decode_forward_host(moe_decode_t h, const void* x_host, const void* router_w, const void* const* w13,
                            const void* const* w2, const void* shared_w13, const void* shared_w2,
                            void* out_host, int32_t* ids_host, float* w_host, int32_t batch, void* stream_main,
                            void* stream_aux) {
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
  cudaError_t e;
  if ((e = cudaMemcpyAsync(xd, x_host, xb, cudaMemcpyHostToDevice, sm)) != cudaSuccess) return fail_cuda(e);
  rc = enqueue_forward(h, xd, router_w, w13, w2, shared_w13, shared_w2, od, idd, wd, batch, sm,
                       static_cast<cudaStream_t>(stream_aux));
  if (rc != MOE_OK) return rc;
  if ((e = cudaMemcpyAsync(out_host, od, xb, cudaMemcpyDeviceToHost, sm)) != cudaSuccess) return fail_cuda(e);
  if ((e = cudaMemcpyAsync(ids_host, idd, kb, cudaMemcpyDeviceToHost, sm)) != cudaSuccess) return fail_cuda(e);
  if ((e = cudaMemcpyAsync(w_host, wd, kb, cudaMemcpyDeviceToHost, sm)) != cudaSuccess) return fail_cuda(e);
  if ((e = cudaStreamSynchronize(sm)) != cudaSuccess) return fail_cuda(e);
  return MOE_OK;
}

int moe_decode_destroy(moe_decode_t h) {
  if (!h) return MOE_OK;
  int rc = MOE_OK;
  {
    DeviceGuard guard(h->device);
    if (h->ws) {
      cudaError_t e = cudaDeviceSynchronize();
      if (e != cudaSuccess) rc = fail_cuda(e);
      cudaFree(h->ws);
    }
    if (h->ev_fork) cudaEventDestroy(h->ev_fork);
    if (h->ev_join) cudaEventDestroy(h->ev_join);
  }
  delete h->tab13;
  delete h->tab2;
  delete h;
  return rc;
}

int moe_decode_get_status(moe_decode_t h) {
  if (!h) return MOE_ERR_INVALID_ARG;
  DeviceGuard guard(h->device);
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail_cuda(e);
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
  *stats = h->stats;
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
