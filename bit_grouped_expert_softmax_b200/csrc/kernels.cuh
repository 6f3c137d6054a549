// kernels.cuh -- argument blocks and launch declarations of the MoE kernels.
#pragma once

#include <utility>

#include "common.cuh"

namespace moe {

constexpr int kTileM = 128;   // down GEMM: weight rows per tile (MMA M)
constexpr int kTileN = 128;   // down GEMM: activation rows per tile (MMA N, max)
constexpr int kGuTileM = 128; // gate/up GEMM: output rows per tile (the same rows of W_gate and W_up)
constexpr int kGuTileN = 128; // gate/up GEMM: activation rows per tile (MMA N, max)
constexpr int kGuTileNSmall = 32;  // the same, when the expert groups are small

// Activation rows per gate/up tile for a batch: the small tile when the
// groups average at most 32 rows (T*k routed rows over E experts).
inline int gu_tile_rows(int64_t T, int64_t k, int64_t E) {
  return T * k <= static_cast<int64_t>(kGuTileNSmall) * E ? kGuTileNSmall : kGuTileN;
}
constexpr int kTileK = 64;    // K elements per pipeline stage (one 128-byte fp16 row)

struct RouteScanArgs {
  int E, nchunk;
  int32_t *chunk_cnt;   // [nchunk][E] counts in, per-chunk prefixes out
  int32_t *totals;      // [E] rows routed to each expert
};

struct RouteScatterArgs {
  int T, E, k, H, I, Is;
  int chunk;                  // tokens per routing chunk (one scatter block each)
  const int32_t *ids;         // [T*k]
  int32_t *chunk_base;        // [nchunk][E] per-chunk prefixes in; zeroed on the way out
  const int32_t *totals;      // [E] rows routed to each expert
  int32_t *offsets;           // [E+1] first row of each expert (written by block 0)
  WorkItem *gu_items;         // gate/up work list
  int max_gu;
  int gu_tile;                // activation rows per gate/up tile (down: kTileN)
  WorkItem *dn_items;         // down work list
  int max_dn;
  int32_t *item_counts;       // [0] gate/up items, [1] down items (written by block 0)
  int32_t *perm;              // [T*k]
  int32_t *inv;               // [T*k]
  const uint16_t *x;          // [T, H] bf16, or null (routing only)
  __half *xt;                 // [T*k + T, H] gathered fp16 rows
  int32_t *xexp;              // [T] power-of-two exponent of each token's row scale
  const float *wts;           // [T*k] routing weights by flat index
  int32_t *row_exp;           // [T*k + T] exponent of the token of each gathered row
  float *row_w;               // [T*k + T] routing weight of each row (1 for shared rows)
  DevStatus *status;
};

// Weights of one layer (device pointers, layout of the public header).
struct LayerWeights {
  const uint32_t *packed;
  const uint16_t *scales;
  const uint16_t *biases;
  const uint32_t *sh_packed;
  const uint16_t *sh_scales;
  const uint16_t *sh_biases;
};

struct GemmArgs {
  int T, E, k, H, I, Is;
  int R;                    // T*k routed rows; shared rows follow at R..R+T-1
  LayerWeights w;
  const __half *xt;         // [R+T, H] gathered activations (gate/up operand)
  __half *h;                // routed rows [R, I] at h, shared rows [T, Is] at h + h_shared_off
  int64_t h_shared_off;     // elements
  __half *y;                // [R+T, H] weighted expert outputs (down result)
  const int32_t *perm;      // [R] row -> flat index t*k+j
  const float *wts;         // [T*k] routing weights by flat index
  const int32_t *xexp;      // [T]
  const int32_t *row_exp;   // [R+T] exponent of each row's token
  const float *row_w;       // [R+T] routing weight of each row (1 for shared rows)
  const WorkItem *items;
  const int32_t *item_count;
  int max_items;
  int64_t xt_rows;          // rows allocated for xt (tensor-map extent)
  int gu_tile;              // activation rows per gate/up tile (kGuTileN or kGuTileNSmall; down: kTileN)
  int64_t h_rows;           // routed h rows allocated
  int64_t hs_rows;          // shared h rows allocated
  DevStatus *status;
  int debug;                // MOE_FLAG_DEBUG: range-check every work item, skip and report bad ones
};

struct CombineArgs {
  int T, k, H, R;
  const int32_t *inv;        // [T*k] flat index -> row
  const __half *y;           // [R+T, H]
  const int32_t *xexp;       // [T]
  const uint16_t *residual;  // [T, H] bf16 or null
  uint16_t *out;             // [T, H] bf16 (may alias residual)
  DevStatus *status;
  int debug;                 // MOE_FLAG_DEBUG: range-check every inverse-permutation entry
};

// Distinct experts one small-T launch can use: the shared one plus T*k routed.
constexpr int kSmallTMaxU = kSmallT * kMaxTopK + 1;
// Synchronisation words of the small-T kernel: the exit count and the count of
// CTAs whose router scores are published (zero before a launch; each launch
// leaves them zero), then the tag of the last launch (zero in a new buffer;
// kept across launches, never cleared).
constexpr int kSmallTExitWord = 0;
constexpr int kSmallTRouterWord = 1;
constexpr int kSmallTEpochWord = 2;
constexpr int kSmallTCounterWords = 2;  // the words a recovery clears
constexpr int kSmallTSyncWords = 3;

struct SmallTArgs {
  int T, E, k, H, I, Is;
  const uint16_t *x;        // [T, H] bf16
  const float *logits;      // [T, E]; written by the kernel itself when router_w is set
  const uint16_t *router_w; // [E, H] bf16 router weight, or null (logits given)
  LayerWeights w;
  uint64_t *hbuf;           // [8][k+1][max(I,Is)/2] SwiGLU outputs by token and slot: two fp16 values and
                            // the launch tag per word (cleared to zero before the first launch)
  uint32_t *sync;           // [kSmallTSyncWords] exit and router counters, last launch tag
  const uint16_t *residual; // [T, H] or null
  uint16_t *out;            // [T, H]
  DevStatus *status;
  unsigned long long wait_ns;  // budget of every bounded wait
  int test_fault;           // testing only: row block 0 of the shared expert does not publish its h
};

// A host-buffer call's inputs, from their host mapping to the device staging
// buffers (x in 16-byte chunks, the logits in 4-byte words).
struct HostStageArgs {
  const uint4 *x_host;
  uint4 *x_dev;
  int x16;
  const uint32_t *l_host;
  uint32_t *l_dev;
  int l4;
};

struct RouterArgs {
  int T, E, H;
  const uint16_t *x;        // [T, H] bf16
  const uint16_t *w;        // [E, H] bf16 router weight
  float *logits;            // [T, E] float32 scores
  DevStatus *status;
};

__global__ void route_topk_kernel(int T, int E, int k, int chunk, const float *__restrict__ logits,
                                  int32_t *__restrict__ ids, float *__restrict__ wts,
                                  int32_t *__restrict__ chunk_cnt);
__global__ void route_scan_kernel(RouteScanArgs a);
__global__ void route_scatter_kernel(RouteScatterArgs a);
__global__ void gather_kernel(RouteScatterArgs a);

// Launch with the programmatic-stream-serialisation attribute when pdl is set
// (the kernel must call pdl_wait() before its first global-memory access).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                            Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// host-side launchers (each returns the launch's cudaError_t)
cudaError_t launch_gemm_gate_up(const GemmArgs &a, int num_sms, cudaStream_t s, bool pdl);
cudaError_t launch_gemm_down(const GemmArgs &a, int num_sms, cudaStream_t s, bool pdl);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s, bool pdl);
cudaError_t launch_router(const RouterArgs &a, cudaStream_t s, bool pdl);
cudaError_t launch_host_stage(const HostStageArgs &a, cudaStream_t s, bool pdl);
cudaError_t launch_small_t(const SmallTArgs &a, int num_sms, cudaStream_t s, bool pdl);
int small_t_grid(int num_sms);
// whether the fused small-T kernel can run this layer (shared memory, grid)
bool small_t_fits(int T, int H, int k, int I, int Is, int num_sms);

}  // namespace moe
