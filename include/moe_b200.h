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
  MOE_FLAG_FORCE_SMALL_T = 2
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
 *   hidden (H), inter (I), shared_inter (Is): multiples of 128.
 *   n_experts (E): 1..256; top_k (k): 1..min(E, 16).
 * Allocates the device workspace on the current device (cudaMalloc); the
 * plan owns it until moe_plan_destroy. *out receives the plan.
 * Errors: MOE_ERR_INVALID_ARG (sizes), MOE_ERR_NO_DEVICE, MOE_ERR_CUDA
 * (allocation failed; nothing is leaked).
 */
moe_status moe_plan(int T_max, int hidden, int n_experts, int top_k, int inter,
                    int shared_inter, int flags, moe_plan_t **out);

/* Free a plan and its workspace. Waits for the device to finish using it. */
moe_status moe_plan_destroy(moe_plan_t *plan);

/* Bytes of device workspace the plan holds. */
int64_t moe_plan_workspace_bytes(const moe_plan_t *plan);

/*
 * One MoE layer for T tokens (0 <= T <= T_max).
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
 * moe_forward with HOST activations: x_bf16_host, router_logits_host and
 * out_bf16_host are host pointers (pinned memory gives asynchronous copies);
 * the weights are device pointers. Copies the inputs into the plan's device
 * staging buffers, runs the layer, copies the output back and waits for the
 * stream, so the host buffers may be reused on return.
 */
moe_status moe_forward_host(moe_plan_t *plan, int T, const void *x_bf16_host,
                            const float *router_logits_host, const uint32_t *packed_w,
                            const void *scales, const void *biases,
                            const uint32_t *shared_packed_w, const void *shared_scales,
                            const void *shared_biases, void *out_bf16_host,
                            moe_stream_t stream);

/*
 * n_layers stacked MoE layers with a residual, in place:
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
 * Wait for the stream, then read and clear the plan's device status word.
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
  MOE_KERNEL_COUNT = 8
};
moe_status moe_profile_enable(moe_plan_t *plan, int max_launches);
moe_status moe_profile_read(moe_plan_t *plan, moe_stream_t stream, double *ms, int32_t *launches);

/*
 * The small-T layer (0 <= T <= 8 tokens) without any device allocation.
 * The source pages describe no such call; it exists for callers that
 * cannot call cudaMalloc (code running inside an allocator or memory-pool
 * callback, runtimes that reserve all device memory up front), and so cannot
 * create a plan. Its scratch memory (SwiGLU outputs, grid-barrier words,
 * status word) lives in one static __device__ array of 512 KiB inside the
 * library, which every GPU that loads the library holds until the process
 * exits; the caller passes only inputs and outputs, as for moe_forward.
 *   Sizes: as moe_plan, plus 8 * (top_k + 1) * max(inter, shared_inter) * 4
 *   bytes must fit in 512 KiB - 256 bytes; larger layers get
 *   MOE_ERR_UNSUPPORTED, T > 8 gets MOE_ERR_INVALID_ARG.
 *   status_out: optional device pointer to 16 bytes that receive the device
 *   status word of this call ({code, site, detail, 0}; code 0 = OK).
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before capturing
 * the stream into a CUDA graph. Each call clears the barrier and status words
 * on the stream and calls no cudaMalloc, cudaFree or allocating library
 * routine. All calls on one device share that device's copy of the array,
 * so calls that overlap on the GPU (for example on two streams) race:
 * serialise them on one stream.
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
