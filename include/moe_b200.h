/*
 * moe_b200.h -- C ABI of the B200 (sm_100a) routed int4 mixture-of-experts layer.
 *
 * The layer is the one the pages single out as the bulk of prefill time
 * ("Perplexity open sources Lily, a Rust and Metal inference engine for Apple
 * Silicon", sections "Requirements and model layout" and "Measurements"; the
 * aioga.com record of the same report, article body paragraphs 3-6):
 *
 *   - a router that scores every expert of a token and picks the top k
 *     (256 and 8 on the pages): p = softmax(logits) over all E experts, the k
 *     largest float32 logits are chosen (equal logits: lower expert id first)
 *     and their probabilities renormalised to sum to one;
 *   - one shared expert that sees every token, with weight 1;
 *   - SwiGLU experts y = W_down (silu(W_gate x) * (W_up x)) whose weights are
 *     groupwise-affine 4-bit: every group of 64 weights along K shares one
 *     bfloat16 scale and one bfloat16 bias, w = q * scale + bias, q in 0..15;
 *   - out_t = sum_j w_{t,j} y_{ids[t,j]}(x_t) + y_shared(x_t), summed in the
 *     fixed order j = 0..k-1 then shared, rounded once to bfloat16.
 *
 * Conventions for every call below:
 *   - Tensor pointers are device pointers owned by the caller unless a call
 *     says otherwise; the library never frees them. They must be 16-byte
 *     aligned. All matrices are row-major with the last index contiguous.
 *   - bfloat16 and float16 values are passed as their 16-bit patterns
 *     (uint16_t / void*).
 *   - Calls enqueue work on the given CUDA stream (a cudaStream_t; NULL is the
 *     legacy default stream) and return without waiting for the GPU, except
 *     moe_status_sync and moe_forward_host.
 *   - Arguments are checked before anything is enqueued. A failed check
 *     returns a negative moe_status, enqueues nothing and sets the message
 *     returned by moe_last_error() for the calling thread.
 *   - Errors that the GPU detects while running (a bounded wait that gave up,
 *     an index out of range) are recorded in a status word on the device and
 *     reported by the next moe_status_sync.
 *   - One plan must not be used by two streams at the same time: its
 *     workspace is shared by all calls made with it.
 *
 * Weight layout (shared with the tests' input generator):
 *   packed_w : uint32 [E][ gate I*H/8 | up I*H/8 | down H*I/8 ]
 *              gate and up are I rows of H/8 words, down is H rows of I/8
 *              words; word w of a row holds elements 8w..8w+7 of that row,
 *              element 8w+j in bits 4j..4j+3 (low nibble first).
 *   scales, biases : bfloat16 [E][ gate I*H/64 | up I*H/64 | down H*I/64 ]
 *              group g of a row covers elements [64g, 64g+64).
 *   shared_* : the same layout for the one shared expert, intermediate Is.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream handle; pass a cudaStream_t (or NULL). */
typedef struct CUstream_st *moe_stream_t;

/* Opaque plan: problem sizes plus the device workspace the layer needs. */
typedef struct moe_plan_s moe_plan_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,    /* a size, pointer or alignment check failed */
  MOE_ERR_UNSUPPORTED = -2,    /* valid request this build does not support */
  MOE_ERR_CUDA = -3,           /* a CUDA runtime or driver call failed */
  MOE_ERR_DEVICE_TIMEOUT = -4, /* a kernel's bounded wait ran out */
  MOE_ERR_DEVICE_BOUNDS = -5,  /* a kernel found an index out of range */
  MOE_ERR_NO_DEVICE = -6       /* no sm_100 CUDA device is visible */
} moe_status;

/* Plan flags. */
enum {
  MOE_FLAG_NONE = 0,
  /* Route every batch through the grouped-GEMM path, even T <= 8 (testing). */
  MOE_FLAG_FORCE_GROUPED = 1,
  /* Route every batch through the small-T path (T <= 8 only; testing). */
  MOE_FLAG_FORCE_SMALL_T = 2,
  /* Range-check, on the device, every index the kernels read from the
   * routing artefacts: each grouped-GEMM work item (expert, weight-row block,
   * first activation row and row count, hence every TMA coordinate derived
   * from it) and each inverse-permutation entry the combine reads. A bad one
   * is skipped and recorded as MOE_ERR_DEVICE_BOUNDS for moe_status_sync;
   * nothing traps. The checks cost a few instructions per work item. */
  MOE_FLAG_DEBUG = 4,
  /* Testing only: the plan's first small-T launch makes one of its bounded
   * waits run out (row block 0 of the shared expert does not store its
   * SwiGLU output, so its readers never see this launch's tag on it) with a
   * 2 ms budget instead of 2 s; every
   * other wait of that launch is bounded too and the launch ends normally.
   * moe_status_sync then reports MOE_ERR_DEVICE_TIMEOUT and clears the
   * state, and later calls on the plan run normally. */
  MOE_FLAG_TEST_WAIT_TIMEOUT = 8,
  /* Launch the layer's kernels in plain stream order. By default each of them
   * goes out with programmatic dependent launch: it may be scheduled while
   * the kernel before it on the stream finishes, runs its prologue (barrier
   * set-up, tensor-memory allocation; the small-batch kernel also requests
   * the shared expert's weights) and waits for that kernel to complete
   * before it touches any other global memory. Results are identical. A
   * caller whose kernel right before the layer writes the layer's weights
   * sets this flag (a copy or memset before it needs nothing). */
  MOE_FLAG_NO_PDL = 16
};

/* Device pointers of one layer's weights, for moe_stack_forward. */
typedef struct {
  const uint32_t *packed_w;
  const void *scales;  /* bfloat16 */
  const void *biases;  /* bfloat16 */
  const uint32_t *shared_packed_w;
  const void *shared_scales;
  const void *shared_biases;
} moe_layer_weights;

/*
 * Create a plan for batches of up to T_max tokens.
 * The pages say only that the engine keeps execution plans and chooses its
 * kernels per shape ("Perplexity open sources Lily...", section
 * "Requirements and model layout"); a plan here is the sizes plus the
 * device workspace of the routing, the grouped GEMMs and the small-T kernel.
 *   hidden (H), inter (I), shared_inter (Is): multiples of 128 (a multiple of
 *   the pages' 64-weight group, as the tensor-core tiles take whole 128-row
 *   blocks of every weight matrix; the small-T kernel also needs H % 256 == 0).
 *   n_experts (E): 1..256; top_k (k): 1..min(E, 16).
 * Allocates the device workspace on the current device (cudaMalloc); the
 * plan owns it until moe_plan_destroy. *out receives the plan.
 * Errors: MOE_ERR_INVALID_ARG (sizes, unknown or conflicting flags),
 * MOE_ERR_NO_DEVICE, MOE_ERR_CUDA (allocation failed; nothing is leaked).
 */
moe_status moe_plan(int T_max, int hidden, int n_experts, int top_k, int inter,
                    int shared_inter, int flags, moe_plan_t **out);

/* Free a plan and its workspace. Waits for the device to finish using it. */
moe_status moe_plan_destroy(moe_plan_t *plan);

/* Bytes of device workspace the plan holds. */
int64_t moe_plan_workspace_bytes(const moe_plan_t *plan);

/*
 * One MoE layer for T tokens (0 <= T <= T_max): the top-k routing over all
 * experts plus the always-on shared expert ("Perplexity open sources
 * Lily...", section "Requirements and model layout"), with the 4-bit weights
 * dequantised one tile at a time inside the grouped expert GEMMs and fp32
 * accumulation (aioga.com record, article body paragraph 4) and the routing
 * kept on the GPU in one stream (same record, paragraph 5).
 *   x_bf16        [T, H] bfloat16 input activations.
 *   router_logits [T, E] float32 router scores (finite values).
 *   packed_w, scales, biases, shared_*: the layer's weights (layout above).
 *   out_bf16      [T, H] bfloat16 output; must not overlap x_bf16.
 * T <= 8 runs the fused small-T kernel when the layer fits it (H a multiple
 * of 256, H/16 no more than the GPU's SMs, its stages within shared memory);
 * otherwise, and for larger T, routing, gather, grouped gate/up GEMM +
 * SwiGLU, grouped down GEMM and the combine run.
 * Deterministic: the same inputs give bit-identical outputs.
 */
moe_status moe_forward(moe_plan_t *plan, int T, const void *x_bf16,
                       const float *router_logits, const uint32_t *packed_w,
                       const void *scales, const void *biases,
                       const uint32_t *shared_packed_w, const void *shared_scales,
                       const void *shared_biases, void *out_bf16,
                       moe_stream_t stream);

/*
 * One MoE layer whose router scores are computed here instead of being
 * passed in: the router "scores 256 experts and picks eight" ("Perplexity
 * open sources Lily...", section "Requirements and model layout"), so
 *   logits[t, e] = sum_h x[t, h] * router_w[e, h]
 * in float32 (bfloat16 operands, float32 accumulation), then the layer of
 * moe_forward on those logits.
 *   router_w_bf16 [E, H] bfloat16 router weight (device, 16-byte aligned).
 * Other arguments as moe_forward. T <= 8 computes the scores inside the
 * fused small-T kernel (each CTA a slice of the experts, published to the
 * others through the plan's workspace); larger T runs a tensor-core router
 * kernel ahead of the routing. The selection compares the float32 scores, so
 * two experts whose exact scores lie within float32 rounding of each other
 * may be ordered either way.
 */
moe_status moe_forward_router(moe_plan_t *plan, int T, const void *x_bf16,
                              const void *router_w_bf16, const uint32_t *packed_w,
                              const void *scales, const void *biases,
                              const uint32_t *shared_packed_w, const void *shared_scales,
                              const void *shared_biases, void *out_bf16,
                              moe_stream_t stream);

/*
 * The router scores alone (the tensor-core router kernel), for checks:
 *   logits_out [T, E] float32 (device) = x [T, H] . router_w [E, H]^T.
 */
moe_status moe_router_logits(moe_plan_t *plan, int T, const void *x_bf16, const void *router_w_bf16,
                             float *logits_out, moe_stream_t stream);

/*
 * moe_forward with HOST activations: x_bf16_host, router_logits_host and
 * out_bf16_host are host pointers (pinned memory gives asynchronous copies);
 * the weights are device pointers. Copies the inputs into the plan's device
 * staging buffers, runs the layer, copies the output back and waits for the
 * stream, so the host buffers may be reused on return. When the batch takes
 * the small-batch kernel (T <= 8) and the three host buffers are pinned
 * (page-locked and mapped, e.g. cudaHostAlloc), with x and out 16-byte and
 * the logits 4-byte aligned, one block reads the inputs through the host
 * mapping into the staging buffers and the kernel writes the output straight
 * into out_bf16_host (no copy engine involved). With pinned host buffers, a
 * call whose arguments (buffers, weights, T) the plan has seen before is
 * captured into a CUDA graph and replayed on later such calls (one launch),
 * for up to 64 argument sets (a decode loop over a model's layers); results
 * are the same.
 * Not while profiling is enabled.
 */
moe_status moe_forward_host(moe_plan_t *plan, int T, const void *x_bf16_host,
                            const float *router_logits_host, const uint32_t *packed_w,
                            const void *scales, const void *biases,
                            const uint32_t *shared_packed_w, const void *shared_scales,
                            const void *shared_biases, void *out_bf16_host,
                            moe_stream_t stream);

/*
 * n_layers stacked MoE layers with a residual, in place (the pages' model has
 * 40 such layers, "Perplexity open sources Lily...", section "Requirements
 * and model layout"; the engine runs them back to back on the GPU without
 * host round trips, aioga.com record, article body paragraphs 5-6):
 *   x <- bfloat16(x + moe_l(x)) for l = 0..n_layers-1,
 * the residual add fused into each layer's combine (one rounding per layer).
 *   x_inout_bf16 [T, H] device, logits [n_layers, T, E] device float32,
 *   layers: HOST array of n_layers weight pointer sets (device pointers).
 * Everything is enqueued on one stream with no host synchronisation, so the
 * call can be captured into a CUDA graph.
 */
moe_status moe_stack_forward(moe_plan_t *plan, int n_layers, int T, void *x_inout_bf16,
                             const float *logits, const moe_layer_weights *layers,
                             moe_stream_t stream);

/*
 * Routing only, for bit-exact checks (the histogram, prefix scan and scatter
 * the report lists, aioga.com record, article body paragraph 5):
 *   ids     [T, k] int32  chosen experts, largest logit first
 *   w       [T, k] float32 renormalised weights
 *   offsets [E+1]  int32  exclusive prefix sum of per-expert counts
 *   perm    [T*k]  int32  flat indices t*k+j sorted by (expert, token)
 * Any output pointer may be NULL.
 */
moe_status moe_route(moe_plan_t *plan, int T, const float *logits, int32_t *ids,
                     float *w, int32_t *offsets, int32_t *perm, moe_stream_t stream);

/*
 * Wait for the stream, then read the plan's device status word. After a
 * device error it also clears the status word and the small-T kernel's
 * counters, so the plan can be used again. The pages describe no error
 * reporting; this is the library's own.
 * Returns MOE_OK, MOE_ERR_DEVICE_TIMEOUT, MOE_ERR_DEVICE_BOUNDS or
 * MOE_ERR_CUDA (with the CUDA error in moe_last_error()).
 */
moe_status moe_status_sync(moe_plan_t *plan, moe_stream_t stream);

/*
 * Per-kernel timing. While enabled, every kernel the plan enqueues is
 * bracketed by two CUDA events recorded on the launching stream (up to
 * max_launches launches; later ones are not recorded). moe_profile_read waits
 * for the stream, adds up the elapsed times per kernel kind into
 * ms[MOE_KERNEL_COUNT] and launches[MOE_KERNEL_COUNT] (either may be NULL)
 * and starts a new recording window. max_launches = 0 disables recording.
 * Not for use while the stream is being captured into a CUDA graph.
 */
enum {
  MOE_KERNEL_ROUTE_TOPK = 0,
  MOE_KERNEL_ROUTE_SCAN = 1,
  MOE_KERNEL_ROUTE_SCATTER = 2,
  MOE_KERNEL_GATHER = 3,
  MOE_KERNEL_GATE_UP = 4,
  MOE_KERNEL_DOWN = 5,
  MOE_KERNEL_COMBINE = 6,
  MOE_KERNEL_SMALL_T = 7,
  MOE_KERNEL_ROUTER = 8,
  MOE_KERNEL_COUNT = 9
};
moe_status moe_profile_enable(moe_plan_t *plan, int max_launches);
moe_status moe_profile_read(moe_plan_t *plan, moe_stream_t stream, double *ms, int32_t *launches);

/*
 * The small-T layer (0 <= T <= 8 tokens) without any device allocation.
 * The source pages describe no such call; it exists for callers that
 * cannot call cudaMalloc (code running inside an allocator or memory-pool
 * callback, runtimes that reserve all device memory up front), and so cannot
 * create a plan. Its scratch memory (SwiGLU outputs, the kernel's counters
 * and launch tag, status word) lives in one static __device__ array of 512 KiB
 * inside the library, which every GPU that loads the library holds until the
 * process exits; the caller passes only inputs and outputs, as for
 * moe_forward, and gets the same result bit for bit.
 *   Sizes: hidden a multiple of 256 (at most 16384), inter and shared_inter
 *   multiples of 128 (at most 8192), top_k <= min(n_experts, 16),
 *   n_experts <= 256; and the SwiGLU outputs (fp16 values stored in pairs
 *   with a 4-byte launch tag), 8 * (top_k + 1) * max(inter, shared_inter)
 *   * 4 bytes, must fit in 512 KiB - 1280 bytes. Larger layers get
 *   MOE_ERR_UNSUPPORTED, T > 8 and bad sizes MOE_ERR_INVALID_ARG.
 *   status_out: optional device pointer to 16 bytes (16-byte aligned) that
 *   receive the device status word of this call ({code, site, detail, 0};
 *   code 0 = OK); a call with T == 0 writes a zero status there.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current; a failed lookup is retried by the next
 * call); make that first call before capturing the stream into a CUDA graph.
 * Each call clears the counters and the status word on the stream (the
 * launch tag is kept, so no call reuses an earlier call's tag) and calls
 * no cudaMalloc, cudaFree or allocating library routine. All calls on one
 * device share that device's copy of the array, so calls that overlap on the
 * GPU (for example on two streams) race: serialise them on one stream.
 */
moe_status moe_forward_small_t_noalloc(int T, int hidden, int n_experts, int top_k, int inter,
                                       int shared_inter, const void *x_bf16,
                                       const float *router_logits, const uint32_t *packed_w,
                                       const void *scales, const void *biases,
                                       const uint32_t *shared_packed_w, const void *shared_scales,
                                       const void *shared_biases, void *out_bf16, void *status_out,
                                       moe_stream_t stream);

/* Message of the last failed call on this thread ("" if none). */
const char *moe_last_error(void);

/* Library version string. */
const char *moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
