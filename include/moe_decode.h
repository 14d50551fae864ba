/*
 * moe_decode.h -- C ABI of the B200 (sm_100a) MoE decode-block library.
 *
 * One call of moe_decode_forward runs the decode pass of one
 * Mixture-of-Experts block for a batch of 1..64 tokens on one GPU:
 *
 *   1. router scores  logit = x . R (+ bias), softmax over all experts,
 *      top-k selection (logit descending, ties to the smaller id) and
 *      renormalisation of the k selected probabilities;
 *   2. bucketing of the token->expert assignments by expert;
 *   3. per selected expert, the SwiGLU up projection
 *      a = silu(x . W13[:, :I]) * (x . W13[:, I:]);
 *   4. the down projection y = a . W2, weighted by the routing weight;
 *   5. the shared expert (same MLP, weight 1), overlapping steps 1-2;
 *   6. out = x + sum_j w_j y_j + shared, rounded once to bf16.
 *
 * Two execution plans (chosen per handle by moe_decode_shapes.flags):
 *   default: three kernels on stream_main.  The router kernel (steps 1-2);
 *     one persistent expert kernel that streams the shared expert's up
 *     projection first -- it needs nothing from the router, so it runs while
 *     the router is still working (programmatic dependent launch) -- then the
 *     routed experts and the shared expert's down projection; the combine
 *     (step 6).  stream_aux is not used.
 *   MOE_FLAG_TWO_STREAM: the pages' layout.  Router and routed experts on
 *     stream_main, the shared expert on stream_aux (forked and joined with
 *     events), then a separate combine kernel.
 *
 * The steps follow the pages "Hyper Optimizing Kimi K3 in vLLM: Moving Fast
 * and Responsibly" (commentary; section "Recovering time between operators":
 * small-matrix projection kernels at batch 1-2, split work at larger
 * batches, the shared expert on another stream, weights prefetched before
 * their consumer starts) and "vLLM Hyper-Optimizes Kimi K3 on NVIDIA GB300"
 * (section "What's Optimized": batch-dependent kernels, MoE scheduling,
 * weight prefetch).  The pages name the steps but give no formulas; the
 * formulas above are the plainest standard reading (softmax router,
 * renormalised top-k, SwiGLU with the gate in the first half of w13, one
 * shared expert of weight 1, residual = the block input x).
 *
 * Conventions for every entry point:
 *   - Return value: MOE_OK (0) or a negative MOE_ERR_* code.  Argument errors
 *     are detected on the host before anything is enqueued.
 *   - Tensors are row-major bf16 (IEEE binary32 upper halves) unless stated.
 *   - "device" pointers point to memory of the GPU the handle was created
 *     on; "host" pointers to CPU memory.  The caller owns every tensor; the
 *     library owns its handle, its workspace and its events.
 *   - Weights are read-only and must not change while a forward that uses
 *     them may be running.
 *   - A handle must not run two forwards at the same time (it owns one
 *     workspace); use one handle per concurrent stream pair.
 */
#ifndef MOE_DECODE_H_
#define MOE_DECODE_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------ error codes */
#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)       /* NULL pointer, bad batch, misaligned pointer */
#define MOE_ERR_UNSUPPORTED_SHAPE (-2) /* shapes outside the supported envelope */
#define MOE_ERR_NO_DEVICE (-3)         /* no CUDA device visible */
#define MOE_ERR_ARCH (-4)              /* device is not compute capability 10.x (B200) */
#define MOE_ERR_CUDA (-5)              /* a CUDA runtime call failed; see moe_decode_last_cuda_error */
#define MOE_ERR_OUT_OF_MEMORY (-6)     /* workspace allocation failed in init */
#define MOE_ERR_DEVICE_TIMEOUT (-7)    /* a bounded device-side wait gave up (status word) */
#define MOE_ERR_DEVICE_PLAN (-8)       /* device-side consistency check failed (status word) */

/* ---------------------------------------------------------------- shapes */
/*
 * Block shape, fixed for the life of a handle.  Supported envelope:
 *   hidden      : multiple of 8, 8..16384
 *   n_experts   : multiple of 8, 8..1024
 *   top_k       : 1..min(32, n_experts)
 *   inter       : multiple of 8, 8..16384 (routed expert intermediate size I)
 *   shared_inter: multiple of 8, 8..16384 when n_shared == 1 (ignored otherwise)
 *   n_shared    : 0 or 1
 *   max_batch   : 1..64; sizes the workspace, forward accepts batch <= max_batch
 * router_bias (optional) is a device float32 [n_experts] added to the router
 * logits before softmax and selection; NULL means no bias.  It is read by
 * every forward (the pointer is kept, the data is not copied).
 * flags: any combination of MOE_FLAG_TWO_STREAM (see the top of this file),
 * MOE_FLAG_TCGEN05, MOE_FLAG_TEST_HOLD_PANEL and MOE_FLAG_FP8_WEIGHTS
 * (below); other bits are rejected with MOE_ERR_UNSUPPORTED_SHAPE.
 */
#define MOE_FLAG_TWO_STREAM 1u
/*
 * MOE_FLAG_TCGEN05: run the expert kernel on the 5th-generation tensor cores
 * (tcgen05.mma, accumulators in tensor memory, one issuing thread, four
 * epilogue warps) instead of mma.sync with register accumulators.  Used only
 * when hidden, inter and shared_inter are multiples of 64 (otherwise the flag
 * is ignored).  Same results within rounding.  Measured slower on B200 for
 * 1-64 tokens: with the tokens as the N dimension each tcgen05.mma covers
 * 128 x 16 weights, so a 64 KB weight stage takes 16 of them, and issuing
 * those from one thread takes about as long as HBM takes to deliver the stage.
 */
#define MOE_FLAG_TCGEN05 2u
/*
 * MOE_FLAG_TEST_HOLD_PANEL (testing only): the handle's first forward
 * withholds the publication of one routed up-projection panel, so the
 * down-projection stages that need it wait until their bounded wait gives
 * up.  That forward's outputs are wrong and moe_decode_get_status reports
 * MOE_ERR_DEVICE_TIMEOUT; later forwards of the handle are normal.  Used,
 * with a short moe_decode_set_wait_limit, to test the device-side timeout
 * path without faulting or hanging the GPU.
 */
#define MOE_FLAG_TEST_HOLD_PANEL 4u
/*
 * MOE_FLAG_FP8_WEIGHTS: the expert weights (routed and shared) are 8-bit e4m3
 * codes with fp32 block scales, passed to moe_decode_forward_fp8 (the other
 * forward entry points reject such a handle).  Weight-only: the router and
 * the activations stay bf16, products are taken in f16 x f16 -> fp32 (every
 * e4m3 value and the activations are exact in f16) and each 128 x 128 block's
 * partial sums are multiplied by its scale.  Needs hidden, inter and
 * shared_inter to be multiples of 128; not combinable with MOE_FLAG_TCGEN05.
 * An extension beyond the pages, which do not discuss weight precision.
 */
#define MOE_FLAG_FP8_WEIGHTS 8u
/*
 * MOE_FLAG_PARTIAL_SUM: the forward writes, instead of bf16(x + sum), the
 * fp32 sum of the expert outputs alone (routed, weighted, plus the shared
 * expert; no residual, no rounding): `out` is then float32 [batch, hidden].
 * For a tensor-parallel block: rank r's handle is made with inter /
 * shared_inter divided by the TP size and given the rank's slices of every
 * expert (w13: gate columns and up columns [r*I/tp, (r+1)*I/tp) each, w2:
 * the same rows), so the ranks' partial sums add up to the block's expert
 * sum; moe_decode_reduce_residual then forms bf16(x + sum over ranks).  The
 * routing must agree across ranks (same x and router weights; the tests
 * draw inputs whose top-k has a margin).  Not with moe_decode_forward_host.
 * The pages run the block tensor-parallel across GPUs with the expert sum
 * exchanged over NVLink ("Recovering time between operators").
 */
#define MOE_FLAG_PARTIAL_SUM 16u
typedef struct moe_decode_shapes {
  int32_t hidden;
  int32_t n_experts;
  int32_t top_k;
  int32_t inter;
  int32_t shared_inter;
  int32_t n_shared;
  int32_t max_batch;
  const float* router_bias;
  uint32_t flags;
} moe_decode_shapes;

typedef struct moe_decode_ctx* moe_decode_t;

/*
 * Per-handle counters, filled by moe_decode_get_stats.  Host side:
 *   forwards          : successful forwards enqueued by this handle
 *   kernels_launched  : kernels enqueued by this handle since creation
 *   last_kernels      : kernels enqueued by the last forward (default plan:
 *                       3; MOE_FLAG_TWO_STREAM: 4, or 3 without a shared
 *                       expert)
 *   last_token_tiles  : token tiles of 8 the expert kernels were prepared for
 *                       in the last forward (ceil(min(batch, 32) / 8))
 * Device side (added by the last CTA of each expert-kernel launch from the
 * plan it consumed, cumulative since moe_decode_init, graph replays included):
 *   stages_up[c], stages_down[c] : weight stages (64 KB; 32 KB for e4m3
 *                       weights in class 2) the expert kernels
 *                       streamed for units of token class c (0: 1-8 tokens,
 *                       1: 9-16, 2: 17-32), up and down projections -- which
 *                       variants actually ran.
 */
typedef struct moe_decode_stats {
  uint64_t forwards;
  uint64_t kernels_launched;
  int32_t last_kernels;
  int32_t last_token_tiles;
  uint64_t stages_up[3];
  uint64_t stages_down[3];
} moe_decode_stats;

/*
 * Create a handle on the current CUDA device: validates the shapes, checks
 * the device (compute capability 10.x), allocates and zeroes the workspace
 * (sized for shapes->max_batch) and creates the fork/join events.  This is
 * the only entry point that allocates device memory.
 * shapes: host pointer, read during the call only.  out_handle: host pointer
 * that receives the handle (set to NULL on error).
 */
int moe_decode_init(const moe_decode_shapes* shapes, moe_decode_t* out_handle);

/*
 * Enqueue one forward of the block on stream_main / stream_aux (cudaStream_t
 * passed as void*; NULL is the legacy default stream).  Asynchronous, does no
 * host synchronisation and allocates nothing, so it can be captured in a
 * CUDA graph.  With MOE_FLAG_TWO_STREAM the shared expert is forked onto
 * stream_aux with an event and joined back (stream_aux may equal
 * stream_main); by default stream_aux is ignored (it may be NULL).  When the
 * call returns every piece of work is ordered before anything later enqueued
 * on stream_main.
 *
 *   x          device bf16 [batch, hidden]          block input and residual
 *   router_w   device bf16 [hidden, n_experts]      router weights (in x out)
 *   w13        HOST array of n_experts device pointers; w13[e] -> bf16
 *              [hidden, 2*inter], columns [0,inter) gate, [inter,2*inter) up
 *   w2         HOST array of n_experts device pointers; w2[e] -> bf16
 *              [inter, hidden]
 *   shared_w13 device bf16 [hidden, 2*shared_inter] (NULL iff n_shared == 0)
 *   shared_w2  device bf16 [shared_inter, hidden]   (NULL iff n_shared == 0)
 *   out        device bf16 [batch, hidden]          must not alias x
 *   topk_ids   device int32 [batch, top_k]          selected experts, best first
 *   topk_w     device float32 [batch, top_k]        renormalised weights
 *   batch      0..max_batch (0 enqueues nothing, reads no pointer other
 *              than the handle and returns MOE_OK)
 * The host pointer arrays are read during the call only.  Every device
 * pointer must be 16-byte aligned; w13[e]/w2[e] must be non-NULL for every
 * expert (any of them may be selected).
 * Errors: MOE_ERR_INVALID_ARG for NULL/misaligned pointers or a bad batch,
 * MOE_ERR_CUDA if a launch fails (the handle's workspace is then re-zeroed
 * by the next forward).
 */
int moe_decode_forward(moe_decode_t h, const void* x, const void* router_w,
                       const void* const* w13, const void* const* w2,
                       const void* shared_w13, const void* shared_w2, void* out,
                       int32_t* topk_ids, float* topk_w, int32_t batch,
                       void* stream_main, void* stream_aux);

/*
 * Same computation with the per-step tensors in HOST memory: copies x_host
 * (bf16 [batch, hidden]) to the handle's device staging buffer, runs the
 * forward, delivers out/topk_ids/topk_w to out_host/ids_host/w_host and
 * synchronises stream_main before returning.  Weights stay device pointers.
 * When out_host (16-byte aligned), ids_host and w_host are all pinned host
 * memory mapped into the device's address space (cudaHostAlloc'ed or
 * registered memory on a unified-addressing system), the kernels store the
 * results into them directly; otherwise the results go through device
 * staging buffers and three device-to-host copies.  Pinned buffers give the
 * fastest transfers; pageable ones work.  When x_host is pinned too, the
 * copy of x and the forward are captured once into a CUDA graph owned by
 * the handle and replayed by later calls with the same arguments (every
 * pointer, the batch, the streams and the wait limit); any change re-captures
 * it.  (Not on the legacy default stream, not from a stream that is already
 * being captured, and not while per-kernel timing events are set: those
 * calls run eagerly.)
 */
int moe_decode_forward_host(moe_decode_t h, const void* x_host, const void* router_w,
                            const void* const* w13, const void* const* w2,
                            const void* shared_w13, const void* shared_w2,
                            void* out_host, int32_t* ids_host, float* w_host,
                            int32_t batch, void* stream_main, void* stream_aux);

/*
 * moe_decode_forward with e4m3 expert weights (a handle created with
 * MOE_FLAG_FP8_WEIGHTS).  x, router_w, out, topk_ids, topk_w, batch and the
 * streams as for moe_decode_forward.  Each expert matrix is given in [out,
 * in] layout -- every output's weights contiguous -- as uint8 e4m3 codes,
 * with a float32 scale array [ceil(in / 128), P] row-major, P = 4 *
 * ceil(ceil(out / 128) / 4) (rows padded to 16 bytes): the weight of
 * (output o, input i) is decode(code[o, i]) * scale[i / 128, o / 128].
 *   w13q  HOST array of n_experts device pointers -> uint8 [2*inter, hidden]
 *         (outputs [0, inter) the gate, [inter, 2*inter) the up projection)
 *   w13s  HOST array of n_experts device pointers -> float32 scales of w13q
 *   w2q   HOST array of n_experts device pointers -> uint8 [hidden, inter]
 *   w2s   HOST array of n_experts device pointers -> float32 scales of w2q
 *   shared_w13q, shared_w13s, shared_w2q, shared_w2s: the shared expert's,
 *         device pointers (NULL iff n_shared == 0)
 * Code and scale arrays 16-byte aligned.  An all-ones exponent and mantissa
 * (0x7F / 0xFF) is NaN in e4m3 and propagates.  Errors: as
 * moe_decode_forward; MOE_ERR_INVALID_ARG also for a handle made without
 * MOE_FLAG_FP8_WEIGHTS.
 */
int moe_decode_forward_fp8(moe_decode_t h, const void* x, const void* router_w, const void* const* w13q,
                           const void* const* w13s, const void* const* w2q, const void* const* w2s,
                           const void* shared_w13q, const void* shared_w13s, const void* shared_w2q,
                           const void* shared_w2s, void* out, int32_t* topk_ids, float* topk_w, int32_t batch,
                           void* stream_main, void* stream_aux);

/*
 * out[t, c] = bf16_rne(x[t, c] + sum_{r < n_parts} partials[r][t, c]), the
 * residual step of a tensor-parallel block with the all-reduce of the ranks'
 * partial sums folded in: partials[r] are the fp32 [batch, hidden] outputs
 * of MOE_FLAG_PARTIAL_SUM forwards -- device pointers, which on an
 * NVLink/NVSwitch system may be peer memory (another GPU's buffer mapped
 * into this device's address space), so every rank reads all ranks' sums
 * directly.  The sum is taken in the order r = 0 .. n_parts-1, so every
 * rank computes the same bits.  The caller orders the partials' producers
 * before this launch (stream order, or an event / barrier across devices).
 *   partials : HOST array of n_parts device pointers, 16-byte aligned
 *   n_parts  : 1 .. MOE_REDUCE_MAX_PARTS
 *   x, out   : device, bf16 [batch, hidden], 16-byte aligned (out may alias x)
 *   batch, hidden : 1 .. 64, multiple of 8 up to 16384
 *   stream   : cudaStream_t, NULL = legacy default stream
 * Asynchronous.  Errors: MOE_ERR_INVALID_ARG (NULL or misaligned pointer,
 * n_parts or sizes out of range), MOE_ERR_NO_DEVICE, MOE_ERR_CUDA.
 * No counterpart in the pages' API; it is this library's form of the
 * NVLink exchange the pages describe.
 */
#define MOE_REDUCE_MAX_PARTS 16
int moe_decode_reduce_residual(const void* const* partials, int32_t n_parts, const void* x, void* out,
                               int32_t batch, int32_t hidden, void* stream);

/* Free the workspace and events; NULL is accepted.  Waits for the handle's
 * work first, as moe_decode_get_status does. */
int moe_decode_destroy(moe_decode_t h);

/*
 * Wait for the handle's work, then read and clear its device status word.
 * "The handle's work" is its last forward enqueued outside graph capture
 * (an event recorded on stream_main at its end); other streams and other
 * handles' work are not waited for.  If the last forward was captured into
 * a CUDA graph, its replays run on streams the handle does not know, so the
 * whole device is synchronised instead.
 * Returns MOE_OK, MOE_ERR_DEVICE_TIMEOUT (a bounded device wait gave up) or
 * MOE_ERR_DEVICE_PLAN (a device consistency check failed), or MOE_ERR_CUDA.
 * After a device-side error the next forward re-zeroes the workspace state.
 */
int moe_decode_get_status(moe_decode_t h);

/* Copy the handle's counters to *stats (host pointer).  Waits for the
 * handle's work first (as moe_decode_get_status) to read the device-side
 * counters. */
int moe_decode_get_stats(moe_decode_t h, moe_decode_stats* stats);

/*
 * Bound of every device-side wait of this handle's kernels, in probes (one
 * probe is one mbarrier try_wait, which may itself suspend for a while, or
 * one poll of a flag in global memory); 0 restores the default (2^24, well
 * under a minute for a wait that never ends).  A wait that runs out records
 * MOE_ERR_DEVICE_TIMEOUT in the status word, stops its CTA's work and lets
 * the kernel finish.  Applies to forwards enqueued after the call (a
 * captured graph keeps the limit it was captured with).  Host only.
 */
int moe_decode_set_wait_limit(moe_decode_t h, uint32_t probes);

/* Static string for a MOE_* code; never NULL. */
const char* moe_decode_error_string(int code);

/* The last CUDA error seen by any entry point of this thread (cudaError_t
 * value, 0 if none) and its name. */
int moe_decode_last_cuda_error(void);
const char* moe_decode_last_cuda_error_string(void);

/*
 * Per-kernel timing.  events: HOST array of MOE_TIMING_EVENTS cudaEvent_t
 * (passed as void*) created by the caller with timing enabled, or NULL to
 * switch timing off.  While set, every forward records, with
 * MOE_FLAG_TWO_STREAM, on stream_main
 *   [0] before the router, [1] after the router, [2] after the routed
 *   experts (up + SwiGLU + down), [3] after the combine,
 * and on stream_aux
 *   [4] before the shared expert, [5] after it;
 * with the default plan (all on stream_main) [0] before the router, [1] and
 * [4] after it, [2] and [5] after the expert kernel (shared + routed
 * experts), [3] after the combine.  cudaEventElapsedTime gives each kernel's duration.  Recording an event
 * between two kernels also makes the second wait for the first to finish
 * (no early launch), so timed forwards can be slightly slower.  The handle
 * keeps the array's values (not the pointer); the caller keeps the events
 * alive while timing is on.
 */
#define MOE_TIMING_EVENTS 6
int moe_decode_set_timing_events(moe_decode_t h, void* const* events, int32_t n_events);

/*
 * Router step only (scores, softmax, top-k, renormalised weights) without a
 * handle and without allocating anything.  The pages have no counterpart for
 * this entry point; it exists for callers that may not call cudaMalloc at all
 * -- for example code that runs while a CUDA graph is being captured, or a
 * host framework that owns every device allocation through its own pool and
 * forbids plug-ins from allocating behind its back -- and so cannot create a
 * handle with moe_decode_init.
 *
 *   x          device bf16 [batch, hidden]
 *   router_w   device bf16 [hidden, n_experts]
 *   router_bias device float32 [n_experts] or NULL
 *   topk_ids   device int32 [batch, top_k]  (selected experts, best first)
 *   topk_w     device float32 [batch, top_k] (renormalised weights)
 *   stream     cudaStream_t as void* (NULL = legacy default stream)
 * Results equal those of moe_decode_forward for the same inputs.
 *
 * Scratch: a fixed static device array of about 300 KB inside this library
 * (held by every GPU that loads it until the process exits), which bounds the
 * sizes: batch <= MOE_NOALLOC_MAX_BATCH, n_experts <= MOE_NOALLOC_MAX_EXPERTS
 * (plus the limits of moe_decode_shapes); larger sizes return
 * MOE_ERR_UNSUPPORTED_SHAPE.  batch 0 returns MOE_OK without reading any
 * pointer.  The first call on a device does a one-time set-up (looks up the
 * array's device address, zeroes it with a synchronous memset), so make that
 * first call before any stream capture.  Every call clears the part of the
 * array that must start at zero with cudaMemsetAsync on `stream` and then
 * launches one kernel; it calls no cudaMalloc, cudaFree or allocating library
 * routine.  All calls on a device share the one array: calls that may
 * overlap on the GPU (different streams without ordering between them) race
 * and must not be issued; calls on one stream are ordered and safe.
 * Errors: MOE_ERR_UNSUPPORTED_SHAPE, MOE_ERR_INVALID_ARG (NULL or misaligned
 * pointers), MOE_ERR_ARCH, MOE_ERR_CUDA.
 */
#define MOE_NOALLOC_MAX_BATCH 64
#define MOE_NOALLOC_MAX_EXPERTS 1024
int moe_router_topk_noalloc(const void* x, const void* router_w, const float* router_bias,
                            int32_t* topk_ids, float* topk_w, int32_t batch, int32_t hidden,
                            int32_t n_experts, int32_t top_k, void* stream);

/*
 * Device status of the last moe_router_topk_noalloc call on the current
 * device: synchronises `stream` (the stream that call was made on), reads
 * the status word in the static scratch array and clears it.  Returns
 * MOE_OK (also when no call has run on this device), MOE_ERR_DEVICE_TIMEOUT
 * (a bounded wait in the router kernel gave up: the ids and weights may be
 * wrong), MOE_ERR_DEVICE_PLAN or MOE_ERR_CUDA.  It allocates nothing (a
 * synchronous 4-byte copy); it synchronises, so it cannot be called while
 * `stream` is being captured.
 */
int moe_router_topk_noalloc_status(void* stream);

/* Workspace bytes that moe_decode_init would allocate for these shapes (0 if
 * the shapes are invalid).  Pure host computation. */
uint64_t moe_decode_workspace_bytes(const moe_decode_shapes* shapes);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DECODE_H_ */
