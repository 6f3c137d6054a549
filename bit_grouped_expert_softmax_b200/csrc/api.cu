// api.cu -- the C ABI declared in include/moe_b200.h.
//
// A plan holds the problem sizes and one device allocation carved into the
// workspace buffers. Every call validates its arguments on the host, then
// enqueues kernels on the caller's stream without synchronising.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "moe_b200.h"
#include "kernels.cuh"

namespace moe {
size_t small_t_smem_bytes(int T, int H, int k, int I, int Is);
void set_last_error(const char *msg);
}

using namespace moe;

namespace {

thread_local std::string g_last_error;

}  // namespace

void moe::set_last_error(const char *msg) { g_last_error = msg; }

namespace {

moe_status fail(moe_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

moe_status cuda_fail(cudaError_t err, const char *what) {
  return fail(MOE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(err), cudaGetErrorString(err));
}

#define MOE_CUDA(call, what)                       \
  do {                                             \
    cudaError_t err__ = (call);                    \
    if (err__ != cudaSuccess) return cuda_fail(err__, what); \
  } while (0)

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Upper bounds of the two work lists for T tokens.
// Gate/up work items of a batch of T tokens with tiles of `tile` activation rows, at most.
int64_t max_gu_items(int64_t T, int64_t E, int64_t k, int64_t I, int64_t Is, int64_t tile) {
  const int64_t R = T * k;
  return (cdiv(R, tile) + std::min<int64_t>(E, R)) * (I / kGuTileM) + cdiv(T, tile) * (Is / kGuTileM);
}
// ... over every batch a plan for T_max tokens may see (each with its own tile size)
int64_t max_gu_items_plan(int64_t T_max, int64_t E, int64_t k, int64_t I, int64_t Is) {
  const int64_t t_small = std::min<int64_t>(T_max, kGuTileNSmall * E / k);  // largest T that takes small tiles
  return std::max(max_gu_items(T_max, E, k, I, Is, gu_tile_rows(T_max, k, E)),
                  max_gu_items(t_small, E, k, I, Is, kGuTileNSmall));
}
int64_t max_dn_items(int64_t T, int64_t E, int64_t k, int64_t H) {
  const int64_t R = T * k;
  return (cdiv(R, kTileN) + std::min<int64_t>(E, R) + cdiv(T, kTileN)) * (H / kTileM);
}

}  // namespace

struct moe_plan_s {
  int T_max, H, E, k, I, Is, flags;
  int device, num_sms;
  size_t ws_bytes;
  char *ws;
  // workspace views
  int32_t *ids;
  float *wts;
  int32_t *xexp;
  int32_t *chunk;
  int32_t *offsets;
  int32_t *perm;
  int32_t *inv;
  int32_t *row_exp;
  float *row_w;
  WorkItem *gu_items;
  WorkItem *dn_items;
  int32_t *item_counts;
  int32_t *totals;
  __half *xt;
  __half *h;
  __half *y;
  uint64_t *hsmall;  // small-T SwiGLU outputs (tagged fp16 pairs)
  DevStatus *status;
  uint32_t *small_sync;
  uint16_t *x_stage;
  float *logits_stage;
  float *router_logits;  // [T_max, E] scores computed from a router weight
  uint16_t *out_stage;
  int64_t max_gu, max_dn;
  bool test_fault_armed = false;  // MOE_FLAG_TEST_WAIT_TIMEOUT: the next small-T launch carries the fault
  // moe_forward_host: the copies and the layer of a call whose arguments
  // (pinned host buffers, weights, T) were seen before, captured into a CUDA
  // graph and replayed; up to kHostGraphs argument sets, the oldest replaced
  static constexpr int kHostKey = 10;
  static constexpr int kHostGraphs = 64;
  struct HostKey {
    const void *v[kHostKey];
    bool operator==(const HostKey &o) const { return std::memcmp(v, o.v, sizeof v) == 0; }
  };
  struct HostGraph {
    HostKey key;
    cudaGraphExec_t exec;  // null: capture was refused, run eagerly
  };
  std::vector<HostKey> host_seen;    // argument sets run once eagerly
  std::vector<HostGraph> host_graphs;
  cudaStream_t capture_stream = nullptr;
  // per-kernel timing (moe_profile_enable / moe_profile_read)
  std::vector<cudaEvent_t> prof_events;  // 2 per recorded launch
  std::vector<int> prof_kind;
  int prof_used = 0;
};

namespace {

moe_status check_dims(int T_max, int H, int E, int k, int I, int Is) {
  if (T_max < 1 || T_max > (1 << 20)) return fail(MOE_ERR_INVALID_ARG, "T_max=%d must be in [1, 2^20]", T_max);
  if (H < kTileM || H % kTileM) return fail(MOE_ERR_INVALID_ARG, "hidden=%d must be a positive multiple of %d", H, kTileM);
  if (H > 16384) return fail(MOE_ERR_INVALID_ARG, "hidden=%d exceeds 16384", H);
  if (I < kTileM || I % kTileM) return fail(MOE_ERR_INVALID_ARG, "inter=%d must be a positive multiple of %d", I, kTileM);
  if (Is < kTileM || Is % kTileM)
    return fail(MOE_ERR_INVALID_ARG, "shared_inter=%d must be a positive multiple of %d", Is, kTileM);
  if (I > 8192 || Is > 8192) return fail(MOE_ERR_INVALID_ARG, "inter sizes above 8192 are not supported");
  if (E < 1 || E > kMaxExperts) return fail(MOE_ERR_INVALID_ARG, "n_experts=%d must be in [1, %d]", E, kMaxExperts);
  if (k < 1 || k > E || k > kMaxTopK) return fail(MOE_ERR_INVALID_ARG, "top_k=%d must be in [1, min(E, %d)]", k, kMaxTopK);
  const int64_t rows = static_cast<int64_t>(T_max) * (k + 1);
  if (rows * H > (int64_t(1) << 31)) return fail(MOE_ERR_INVALID_ARG, "T_max*(top_k+1)*hidden too large");
  return MOE_OK;
}

moe_status check_weights(const moe_plan_s *p, const void *packed, const void *scales, const void *biases,
                         const void *spacked, const void *sscales, const void *sbiases) {
  const void *ptrs[6] = {packed, scales, biases, spacked, sscales, sbiases};
  const char *names[6] = {"packed_w", "scales", "biases", "shared_packed_w", "shared_scales", "shared_biases"};
  for (int i = 0; i < 6; ++i) {
    if (!ptrs[i]) return fail(MOE_ERR_INVALID_ARG, "%s is NULL", names[i]);
    if (!aligned16(ptrs[i])) return fail(MOE_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
  }
  (void)p;
  return MOE_OK;
}

bool use_small_t(const moe_plan_s *p, int T) {
  if (p->flags & MOE_FLAG_FORCE_GROUPED) return false;
  return small_t_fits(T, p->H, p->k, p->I, p->Is, p->num_sms);
}

LayerWeights make_weights(const void *packed, const void *scales, const void *biases, const void *spacked,
                          const void *sscales, const void *sbiases) {
  LayerWeights w;
  w.packed = static_cast<const uint32_t *>(packed);
  w.scales = static_cast<const uint16_t *>(scales);
  w.biases = static_cast<const uint16_t *>(biases);
  w.sh_packed = static_cast<const uint32_t *>(spacked);
  w.sh_scales = static_cast<const uint16_t *>(sscales);
  w.sh_biases = static_cast<const uint16_t *>(sbiases);
  return w;
}

// Whether the grouped path's kernels go out with programmatic dependent launch.
// Not while profiling: the events between kernels would separate them anyway.
bool pdl(const moe_plan_s *p) { return !(p->flags & MOE_FLAG_NO_PDL) && p->prof_kind.empty(); }

// Brackets one kernel launch with the plan's profiling events, if enabled.
struct ProfScope {
  moe_plan_s *p;
  cudaStream_t s;
  int slot = -1;
  ProfScope(moe_plan_s *p_, int kind, cudaStream_t s_) : p(p_), s(s_) {
    if (p->prof_used < static_cast<int>(p->prof_kind.size())) {
      slot = p->prof_used++;
      p->prof_kind[slot] = kind;
      cudaEventRecord(p->prof_events[2 * slot], s);
    }
  }
  ~ProfScope() {
    if (slot >= 0) cudaEventRecord(p->prof_events[2 * slot + 1], s);
  }
};

// routing kernels: ids/weights + histogram, scan + work lists, scatter, gather (if x)
moe_status enqueue_routing(moe_plan_s *p, int T, const float *logits, const uint16_t *x, cudaStream_t s) {
  const int chunk = route_chunk(T);
  const int nchunk = static_cast<int>(cdiv(T, chunk));
  // one warp per token, two per block: a few hundred tokens still spread over every SM
  const int tok_blocks = static_cast<int>(cdiv(T, 2));
  {
    ProfScope ps(p, MOE_KERNEL_ROUTE_TOPK, s);
    MOE_CUDA(launch_k(route_topk_kernel, dim3(tok_blocks), dim3(64), 0, s, pdl(p), T, p->E, p->k, chunk, logits,
                      p->ids, p->wts, p->chunk),
             "route_topk launch");
  }
  RouteScanArgs sa{};
  sa.E = p->E; sa.nchunk = nchunk; sa.chunk_cnt = p->chunk; sa.totals = p->totals;
  {
    ProfScope ps(p, MOE_KERNEL_ROUTE_SCAN, s);
    MOE_CUDA(launch_k(route_scan_kernel, dim3(static_cast<int>(cdiv(p->E, 8))), dim3(256), 0, s, pdl(p), sa),
             "route_scan launch");
  }
  RouteScatterArgs ca{};
  ca.T = T; ca.E = p->E; ca.k = p->k; ca.H = p->H; ca.I = p->I; ca.Is = p->Is; ca.chunk = chunk;
  ca.ids = p->ids; ca.chunk_base = p->chunk; ca.totals = p->totals; ca.offsets = p->offsets; ca.perm = p->perm;
  ca.inv = p->inv;
  ca.gu_items = p->gu_items; ca.max_gu = static_cast<int>(p->max_gu); ca.gu_tile = gu_tile_rows(T, p->k, p->E);
  ca.dn_items = p->dn_items; ca.max_dn = static_cast<int>(p->max_dn); ca.item_counts = p->item_counts;
  ca.x = x; ca.xt = p->xt; ca.xexp = p->xexp; ca.status = p->status;
  ca.wts = p->wts; ca.row_exp = p->row_exp; ca.row_w = p->row_w;
  {
    ProfScope ps(p, MOE_KERNEL_ROUTE_SCATTER, s);
    MOE_CUDA(launch_k(route_scatter_kernel, dim3(nchunk), dim3(256), 0, s, pdl(p), ca), "route_scatter launch");
  }
  if (x) {
    ProfScope ps(p, MOE_KERNEL_GATHER, s);
    MOE_CUDA(launch_k(gather_kernel, dim3(tok_blocks), dim3(64), 0, s, pdl(p), ca), "gather launch");
  }
  return MOE_OK;
}

// Router scores of T tokens into the plan's workspace (grouped path).
moe_status enqueue_router(moe_plan_s *p, int T, const uint16_t *x, const uint16_t *router_w, float *logits,
                          cudaStream_t s) {
  RouterArgs r{};
  r.T = T; r.E = p->E; r.H = p->H; r.x = x; r.w = router_w; r.logits = logits; r.status = p->status;
  ProfScope ps(p, MOE_KERNEL_ROUTER, s);
  MOE_CUDA(launch_router(r, s, pdl(p)), "router launch");
  return MOE_OK;
}

// One layer. With router_w set, the logits are computed from it (and the
// logits argument is ignored): inside the small-T kernel, or by the router
// kernel ahead of the grouped path's routing.
moe_status enqueue_layer(moe_plan_s *p, int T, const uint16_t *x, const float *logits, const LayerWeights &w,
                         const uint16_t *residual, uint16_t *out, cudaStream_t s,
                         const uint16_t *router_w = nullptr) {
  if (T == 0) return MOE_OK;
  if (use_small_t(p, T) || (p->flags & MOE_FLAG_FORCE_SMALL_T)) {
    if (!small_t_fits(T, p->H, p->k, p->I, p->Is, p->num_sms))
      return fail(MOE_ERR_UNSUPPORTED, "small-T path needs T <= %d and a small enough layer", kSmallT);
    SmallTArgs a{};
    a.T = T; a.E = p->E; a.k = p->k; a.H = p->H; a.I = p->I; a.Is = p->Is;
    a.x = x; a.logits = router_w ? p->router_logits : logits; a.router_w = router_w;
    a.w = w; a.hbuf = p->hsmall; a.sync = p->small_sync;
    a.residual = residual; a.out = out; a.status = p->status;
    a.wait_ns = kWaitBudgetNs;
    a.test_fault = 0;
    if (p->test_fault_armed) {  // one launch only
      a.test_fault = 1;
      a.wait_ns = kTestWaitBudgetNs;
      p->test_fault_armed = false;
    }
    ProfScope ps(p, MOE_KERNEL_SMALL_T, s);
    MOE_CUDA(launch_small_t(a, p->num_sms, s, pdl(p)), "small-T kernel launch");
    return MOE_OK;
  }
  if (router_w) {
    moe_status st = enqueue_router(p, T, x, router_w, p->router_logits, s);
    if (st != MOE_OK) return st;
    logits = p->router_logits;
  }
  moe_status st = enqueue_routing(p, T, logits, x, s);
  if (st != MOE_OK) return st;
  GemmArgs g{};
  g.T = T; g.E = p->E; g.k = p->k; g.H = p->H; g.I = p->I; g.Is = p->Is; g.R = T * p->k;
  g.w = w; g.xt = p->xt; g.h = p->h;
  g.h_shared_off = static_cast<int64_t>(p->T_max) * p->k * p->I;
  g.y = p->y; g.perm = p->perm; g.wts = p->wts; g.xexp = p->xexp; g.status = p->status;
  g.row_exp = p->row_exp; g.row_w = p->row_w;
  g.debug = (p->flags & MOE_FLAG_DEBUG) ? 1 : 0;
  g.xt_rows = static_cast<int64_t>(p->T_max) * (p->k + 1);
  g.h_rows = static_cast<int64_t>(p->T_max) * p->k;
  g.hs_rows = p->T_max;
  g.items = p->gu_items;
  g.item_count = p->item_counts;
  g.gu_tile = gu_tile_rows(T, p->k, p->E);
  g.max_items = static_cast<int>(std::min<int64_t>(max_gu_items(T, p->E, p->k, p->I, p->Is, g.gu_tile), p->max_gu));
  {
    ProfScope ps(p, MOE_KERNEL_GATE_UP, s);
    MOE_CUDA(launch_gemm_gate_up(g, p->num_sms, s, pdl(p)), "gate/up GEMM launch");
  }
  g.items = p->dn_items;
  g.item_count = p->item_counts + 1;
  g.max_items = static_cast<int>(max_dn_items(T, p->E, p->k, p->H));
  {
    ProfScope ps(p, MOE_KERNEL_DOWN, s);
    MOE_CUDA(launch_gemm_down(g, p->num_sms, s, pdl(p)), "down GEMM launch");
  }
  CombineArgs c{};
  c.T = T; c.k = p->k; c.H = p->H; c.R = T * p->k;
  c.inv = p->inv; c.y = p->y; c.xexp = p->xexp; c.residual = residual; c.out = out;
  c.status = p->status; c.debug = (p->flags & MOE_FLAG_DEBUG) ? 1 : 0;
  {
    ProfScope ps(p, MOE_KERNEL_COMBINE, s);
    MOE_CUDA(launch_combine(c, s, pdl(p)), "combine launch");
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

const char *moe_last_error(void) { return g_last_error.c_str(); }

const char *moe_version(void) { return "moe_b200 0.1 (sm_100a)"; }

moe_status moe_plan(int T_max, int hidden, int n_experts, int top_k, int inter, int shared_inter, int flags,
                    moe_plan_t **out) {
  g_last_error.clear();
  if (!out) return fail(MOE_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  moe_status st = check_dims(T_max, hidden, n_experts, top_k, inter, shared_inter);
  if (st != MOE_OK) return st;
  if ((flags & MOE_FLAG_FORCE_GROUPED) && (flags & MOE_FLAG_FORCE_SMALL_T))
    return fail(MOE_ERR_INVALID_ARG, "flags FORCE_GROUPED and FORCE_SMALL_T exclude each other");
  if (flags & ~(MOE_FLAG_FORCE_GROUPED | MOE_FLAG_FORCE_SMALL_T | MOE_FLAG_DEBUG | MOE_FLAG_TEST_WAIT_TIMEOUT |
                MOE_FLAG_NO_PDL))
    return fail(MOE_ERR_INVALID_ARG, "unknown flags 0x%x", flags);
  int dev = 0, ndev = 0;
  if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
    cudaGetLastError();
    return fail(MOE_ERR_NO_DEVICE, "no CUDA device is visible");
  }
  MOE_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  cudaDeviceProp prop;
  MOE_CUDA(cudaGetDeviceProperties(&prop, dev), "cudaGetDeviceProperties");
  if (prop.major != 10 || prop.minor != 0)
    return fail(MOE_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, prop.major,
                prop.minor);

  moe_plan_s *p = new moe_plan_s();
  p->T_max = T_max; p->H = hidden; p->E = n_experts; p->k = top_k; p->I = inter; p->Is = shared_inter;
  p->flags = flags; p->device = dev; p->num_sms = prop.multiProcessorCount;
  p->test_fault_armed = (flags & MOE_FLAG_TEST_WAIT_TIMEOUT) != 0;
  p->max_gu = max_gu_items_plan(T_max, n_experts, top_k, inter, shared_inter);
  p->max_dn = max_dn_items(T_max, n_experts, top_k, hidden);
  const size_t T = T_max, H = hidden, E = n_experts, k = top_k, I = inter, Is = shared_inter;
  const size_t R = T * k, nchunk = (T + kRouteChunkMin - 1) / kRouteChunkMin;  // the most chunks any batch has
  const size_t sizes[] = {
      R * 4,                                 // ids
      R * 4,                                 // wts
      T * 4,                                 // xexp
      nchunk * E * 4,                        // chunk
      (E + 1) * 4,                           // offsets
      R * 4,                                 // perm
      R * 4,                                 // inv
      (R + T) * 4,                           // row_exp
      (R + T) * 4,                           // row_w
      static_cast<size_t>(p->max_gu) * sizeof(WorkItem),
      static_cast<size_t>(p->max_dn) * sizeof(WorkItem),
      16,                                    // item counts
      E * 4,                                 // rows routed to each expert
      (R + T) * H * 2,                       // xt
      (R * I + T * Is) * 2,                  // h
      (R + T) * H * 2,                       // y
      static_cast<size_t>(kSmallT) * (k + 1) * std::max(I, Is) * 4,  // small-T h (tagged fp16 pairs)
      sizeof(DevStatus),                     // status
      kSmallTSyncWords * 4,                  // small-T counters and launch tag
      T * H * 2,                             // x staging
      T * E * 4,                             // logits staging
      T * E * 4,                             // router scores
      T * H * 2,                             // out staging
  };
  constexpr int nbuf = sizeof(sizes) / sizeof(sizes[0]);
  size_t offs[nbuf], total = 0;
  for (int i = 0; i < nbuf; ++i) {
    offs[i] = total;
    total += align_up(sizes[i]);
  }
  cudaError_t err = cudaMalloc(&p->ws, total);
  if (err != cudaSuccess) {
    delete p;
    return cuda_fail(err, "workspace cudaMalloc");
  }
  p->ws_bytes = total;
  char *b = p->ws;
  int i = 0;
  p->ids = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->wts = reinterpret_cast<float *>(b + offs[i++]);
  p->xexp = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->chunk = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->offsets = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->perm = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->inv = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->row_exp = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->row_w = reinterpret_cast<float *>(b + offs[i++]);
  p->gu_items = reinterpret_cast<WorkItem *>(b + offs[i++]);
  p->dn_items = reinterpret_cast<WorkItem *>(b + offs[i++]);
  p->item_counts = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->totals = reinterpret_cast<int32_t *>(b + offs[i++]);
  p->xt = reinterpret_cast<__half *>(b + offs[i++]);
  p->h = reinterpret_cast<__half *>(b + offs[i++]);
  p->y = reinterpret_cast<__half *>(b + offs[i++]);
  p->hsmall = reinterpret_cast<uint64_t *>(b + offs[i++]);
  p->status = reinterpret_cast<DevStatus *>(b + offs[i++]);
  p->small_sync = reinterpret_cast<uint32_t *>(b + offs[i++]);
  p->x_stage = reinterpret_cast<uint16_t *>(b + offs[i++]);
  p->logits_stage = reinterpret_cast<float *>(b + offs[i++]);
  p->router_logits = reinterpret_cast<float *>(b + offs[i++]);
  p->out_stage = reinterpret_cast<uint16_t *>(b + offs[i++]);
  err = cudaMemset(p->ws, 0, total);
  if (err == cudaSuccess) err = cudaDeviceSynchronize();
  if (err != cudaSuccess) {
    cudaFree(p->ws);
    delete p;
    return cuda_fail(err, "workspace clear");
  }
  *out = p;
  return MOE_OK;
}

moe_status moe_plan_destroy(moe_plan_t *plan) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  cudaError_t err = cudaDeviceSynchronize();
  cudaError_t err2 = cudaFree(plan->ws);
  for (cudaEvent_t e : plan->prof_events) cudaEventDestroy(e);
  for (auto &g : plan->host_graphs)
    if (g.exec) cudaGraphExecDestroy(g.exec);
  if (plan->capture_stream) cudaStreamDestroy(plan->capture_stream);
  delete plan;
  if (err != cudaSuccess) return cuda_fail(err, "synchronize before free");
  if (err2 != cudaSuccess) return cuda_fail(err2, "workspace cudaFree");
  return MOE_OK;
}

int64_t moe_plan_workspace_bytes(const moe_plan_t *plan) { return plan ? static_cast<int64_t>(plan->ws_bytes) : -1; }

moe_status moe_forward(moe_plan_t *plan, int T, const void *x_bf16, const float *router_logits,
                       const uint32_t *packed_w, const void *scales, const void *biases,
                       const uint32_t *shared_packed_w, const void *shared_scales, const void *shared_biases,
                       void *out_bf16, moe_stream_t stream) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  if (T < 0 || T > plan->T_max) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [0, T_max=%d]", T, plan->T_max);
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !router_logits || !out_bf16) return fail(MOE_ERR_INVALID_ARG, "x, logits and out must not be NULL");
  if (!aligned16(x_bf16) || !aligned16(router_logits) || !aligned16(out_bf16))
    return fail(MOE_ERR_INVALID_ARG, "x, logits and out must be 16-byte aligned");
  if (x_bf16 == out_bf16) return fail(MOE_ERR_INVALID_ARG, "out must not alias x (use moe_stack_forward)");
  moe_status st = check_weights(plan, packed_w, scales, biases, shared_packed_w, shared_scales, shared_biases);
  if (st != MOE_OK) return st;
  const LayerWeights w = make_weights(packed_w, scales, biases, shared_packed_w, shared_scales, shared_biases);
  return enqueue_layer(plan, T, static_cast<const uint16_t *>(x_bf16), router_logits, w, nullptr,
                       static_cast<uint16_t *>(out_bf16), reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_forward_router(moe_plan_t *plan, int T, const void *x_bf16, const void *router_w_bf16,
                              const uint32_t *packed_w, const void *scales, const void *biases,
                              const uint32_t *shared_packed_w, const void *shared_scales, const void *shared_biases,
                              void *out_bf16, moe_stream_t stream) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  if (T < 0 || T > plan->T_max) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [0, T_max=%d]", T, plan->T_max);
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !router_w_bf16 || !out_bf16) return fail(MOE_ERR_INVALID_ARG, "x, router_w and out must not be NULL");
  if (!aligned16(x_bf16) || !aligned16(router_w_bf16) || !aligned16(out_bf16))
    return fail(MOE_ERR_INVALID_ARG, "x, router_w and out must be 16-byte aligned");
  if (x_bf16 == out_bf16) return fail(MOE_ERR_INVALID_ARG, "out must not alias x");
  moe_status st = check_weights(plan, packed_w, scales, biases, shared_packed_w, shared_scales, shared_biases);
  if (st != MOE_OK) return st;
  const LayerWeights w = make_weights(packed_w, scales, biases, shared_packed_w, shared_scales, shared_biases);
  return enqueue_layer(plan, T, static_cast<const uint16_t *>(x_bf16), nullptr, w, nullptr,
                       static_cast<uint16_t *>(out_bf16), reinterpret_cast<cudaStream_t>(stream),
                       static_cast<const uint16_t *>(router_w_bf16));
}

moe_status moe_router_logits(moe_plan_t *plan, int T, const void *x_bf16, const void *router_w_bf16,
                             float *logits_out, moe_stream_t stream) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  if (T < 0 || T > plan->T_max) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [0, T_max=%d]", T, plan->T_max);
  if (T == 0) return MOE_OK;
  if (!x_bf16 || !router_w_bf16 || !logits_out)
    return fail(MOE_ERR_INVALID_ARG, "x, router_w and logits_out must not be NULL");
  if (!aligned16(x_bf16) || !aligned16(router_w_bf16) || !aligned16(logits_out))
    return fail(MOE_ERR_INVALID_ARG, "x, router_w and logits_out must be 16-byte aligned");
  return enqueue_router(plan, T, static_cast<const uint16_t *>(x_bf16), static_cast<const uint16_t *>(router_w_bf16),
                        logits_out, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_forward_host(moe_plan_t *plan, int T, const void *x_bf16_host, const float *router_logits_host,
                            const uint32_t *packed_w, const void *scales, const void *biases,
                            const uint32_t *shared_packed_w, const void *shared_scales, const void *shared_biases,
                            void *out_bf16_host, moe_stream_t stream) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  if (T < 0 || T > plan->T_max) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [0, T_max=%d]", T, plan->T_max);
  if (T == 0) return MOE_OK;
  if (!x_bf16_host || !router_logits_host || !out_bf16_host)
    return fail(MOE_ERR_INVALID_ARG, "host x, logits and out must not be NULL");
  moe_status st = check_weights(plan, packed_w, scales, biases, shared_packed_w, shared_scales, shared_biases);
  if (st != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t xb = static_cast<size_t>(T) * plan->H * 2, lb = static_cast<size_t>(T) * plan->E * 4;
  const LayerWeights w = make_weights(packed_w, scales, biases, shared_packed_w, shared_scales, shared_biases);
  // the device address of a pinned (page-locked, mapped) host buffer aligned
  // to `align` bytes, or null
  auto mapped = [](const void *ptr, uintptr_t align) -> void * {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || !at.devicePointer) return nullptr;
    return (reinterpret_cast<uintptr_t>(at.devicePointer) % align) == 0 ? at.devicePointer : nullptr;
  };
  void *x_map = mapped(x_bf16_host, 16), *l_map = mapped(router_logits_host, 4), *o_map = mapped(out_bf16_host, 16);
  const bool pinned_all = x_map && l_map && o_map;
  // On the small-batch path one block reads the inputs through the host
  // mapping into the staging buffers and the kernel writes its output straight
  // into the host buffer: two short kernels instead of three copies and the
  // kernel. (Letting the kernel read x and the logits through the mapping
  // itself was slower: every one of its CTAs reads all of them.)
  const bool host_direct = pinned_all && (use_small_t(plan, T) || (plan->flags & MOE_FLAG_FORCE_SMALL_T));
  // the copies and the layer, enqueued on stream q
  auto enqueue_all = [&](cudaStream_t q) -> moe_status {
    if (host_direct) {
      HostStageArgs hs{};
      hs.x_host = static_cast<const uint4 *>(x_map);
      hs.x_dev = reinterpret_cast<uint4 *>(plan->x_stage);
      hs.x16 = static_cast<int>(xb / 16);
      hs.l_host = static_cast<const uint32_t *>(l_map);
      hs.l_dev = reinterpret_cast<uint32_t *>(plan->logits_stage);
      hs.l4 = static_cast<int>(lb / 4);
      MOE_CUDA(launch_host_stage(hs, q, pdl(plan)), "host staging launch");
      return enqueue_layer(plan, T, plan->x_stage, plan->logits_stage, w, nullptr, static_cast<uint16_t *>(o_map), q);
    }
    MOE_CUDA(cudaMemcpyAsync(plan->x_stage, x_bf16_host, xb, cudaMemcpyHostToDevice, q), "copy x to device");
    MOE_CUDA(cudaMemcpyAsync(plan->logits_stage, router_logits_host, lb, cudaMemcpyHostToDevice, q),
             "copy logits to device");
    moe_status s2 = enqueue_layer(plan, T, plan->x_stage, plan->logits_stage, w, nullptr, plan->out_stage, q);
    if (s2 != MOE_OK) return s2;
    MOE_CUDA(cudaMemcpyAsync(out_bf16_host, plan->out_stage, xb, cudaMemcpyDeviceToHost, q), "copy out to host");
    return MOE_OK;
  };
  // A call whose arguments (pinned host buffers, no profiling or test fault
  // pending) were seen before is captured into a CUDA graph on a private
  // stream and replayed from then on: one launch instead of three copies and
  // the layer's kernels. The first occurrence runs eagerly (it also sets the
  // kernels' launch attributes, outside any capture).
  moe_plan_s::HostKey key = {{x_bf16_host, router_logits_host, out_bf16_host, packed_w, scales, biases,
                              shared_packed_w, shared_scales, shared_biases,
                              reinterpret_cast<const void *>(static_cast<intptr_t>(T))}};
  const bool graphable = plan->prof_kind.empty() && !plan->test_fault_armed && pinned_all;
  if (graphable) {
    for (auto &g : plan->host_graphs)
      if (g.key == key) {
        if (!g.exec) break;  // refused before: eager
        MOE_CUDA(cudaGraphLaunch(g.exec, s), "graph launch");
        MOE_CUDA(cudaStreamSynchronize(s), "stream synchronize");
        return MOE_OK;
      }
    bool seen = false;
    for (auto &k2 : plan->host_seen) seen = seen || k2 == key;
    bool known = false;
    for (auto &g : plan->host_graphs) known = known || g.key == key;
    if (seen && !known) {
      if (!plan->capture_stream)
        MOE_CUDA(cudaStreamCreateWithFlags(&plan->capture_stream, cudaStreamNonBlocking), "capture stream");
      cudaGraph_t graph = nullptr;
      cudaGraphExec_t exec = nullptr;
      MOE_CUDA(cudaStreamBeginCapture(plan->capture_stream, cudaStreamCaptureModeThreadLocal), "begin capture");
      const moe_status sc = enqueue_all(plan->capture_stream);
      const cudaError_t ec = cudaStreamEndCapture(plan->capture_stream, &graph);
      cudaError_t ei = cudaErrorUnknown;
      if (sc == MOE_OK && ec == cudaSuccess && graph) ei = cudaGraphInstantiate(&exec, graph, 0);
      if (graph) cudaGraphDestroy(graph);
      if (ei != cudaSuccess) {  // refused: this argument set runs eagerly from now on
        cudaGetLastError();
        g_last_error.clear();
        exec = nullptr;
      }
      if (static_cast<int>(plan->host_graphs.size()) == moe_plan_s::kHostGraphs) {
        if (plan->host_graphs.front().exec) cudaGraphExecDestroy(plan->host_graphs.front().exec);
        plan->host_graphs.erase(plan->host_graphs.begin());
      }
      plan->host_graphs.push_back({key, exec});
      if (exec) {
        MOE_CUDA(cudaGraphLaunch(exec, s), "graph launch");
        MOE_CUDA(cudaStreamSynchronize(s), "stream synchronize");
        return MOE_OK;
      }
    } else if (!seen) {
      if (static_cast<int>(plan->host_seen.size()) == moe_plan_s::kHostGraphs)
        plan->host_seen.erase(plan->host_seen.begin());
      plan->host_seen.push_back(key);
    }
  }
  st = enqueue_all(s);
  if (st != MOE_OK) return st;
  MOE_CUDA(cudaStreamSynchronize(s), "stream synchronize");
  return MOE_OK;
}

moe_status moe_stack_forward(moe_plan_t *plan, int n_layers, int T, void *x_inout_bf16, const float *logits,
                             const moe_layer_weights *layers, moe_stream_t stream) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  if (n_layers < 0) return fail(MOE_ERR_INVALID_ARG, "n_layers=%d is negative", n_layers);
  if (T < 0 || T > plan->T_max) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [0, T_max=%d]", T, plan->T_max);
  if (T == 0 || n_layers == 0) return MOE_OK;
  if (!x_inout_bf16 || !logits || !layers) return fail(MOE_ERR_INVALID_ARG, "x, logits and layers must not be NULL");
  if (!aligned16(x_inout_bf16) || !aligned16(logits)) return fail(MOE_ERR_INVALID_ARG, "x and logits must be 16-byte aligned");
  for (int l = 0; l < n_layers; ++l) {
    const moe_layer_weights &L = layers[l];
    moe_status st = check_weights(plan, L.packed_w, L.scales, L.biases, L.shared_packed_w, L.shared_scales,
                                  L.shared_biases);
    if (st != MOE_OK) return fail(st, "layer %d: %s", l, g_last_error.c_str());
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint16_t *x = static_cast<uint16_t *>(x_inout_bf16);
  for (int l = 0; l < n_layers; ++l) {
    const moe_layer_weights &L = layers[l];
    const LayerWeights w =
        make_weights(L.packed_w, L.scales, L.biases, L.shared_packed_w, L.shared_scales, L.shared_biases);
    moe_status st = enqueue_layer(plan, T, x, logits + static_cast<size_t>(l) * T * plan->E, w, x, x, s);
    if (st != MOE_OK) return st;
  }
  return MOE_OK;
}

moe_status moe_route(moe_plan_t *plan, int T, const float *logits, int32_t *ids, float *w, int32_t *offsets,
                     int32_t *perm, moe_stream_t stream) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  if (T < 0 || T > plan->T_max) return fail(MOE_ERR_INVALID_ARG, "T=%d outside [0, T_max=%d]", T, plan->T_max);
  if (T == 0) return MOE_OK;
  if (!logits) return fail(MOE_ERR_INVALID_ARG, "logits is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  moe_status st = enqueue_routing(plan, T, logits, nullptr, s);
  if (st != MOE_OK) return st;
  const size_t R = static_cast<size_t>(T) * plan->k;
  if (ids) MOE_CUDA(cudaMemcpyAsync(ids, plan->ids, R * 4, cudaMemcpyDeviceToDevice, s), "copy ids");
  if (w) MOE_CUDA(cudaMemcpyAsync(w, plan->wts, R * 4, cudaMemcpyDeviceToDevice, s), "copy w");
  if (offsets)
    MOE_CUDA(cudaMemcpyAsync(offsets, plan->offsets, (plan->E + 1) * 4, cudaMemcpyDeviceToDevice, s), "copy offsets");
  if (perm) MOE_CUDA(cudaMemcpyAsync(perm, plan->perm, R * 4, cudaMemcpyDeviceToDevice, s), "copy perm");
  return MOE_OK;
}

moe_status moe_profile_enable(moe_plan_t *plan, int max_launches) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  if (max_launches < 0 || max_launches > (1 << 20)) return fail(MOE_ERR_INVALID_ARG, "max_launches out of range");
  for (cudaEvent_t e : plan->prof_events) cudaEventDestroy(e);
  plan->prof_events.clear();
  plan->prof_kind.assign(max_launches, 0);
  plan->prof_used = 0;
  plan->prof_events.resize(2 * static_cast<size_t>(max_launches));
  for (auto &e : plan->prof_events) {
    cudaError_t err = cudaEventCreate(&e);
    if (err != cudaSuccess) {
      plan->prof_kind.clear();
      return cuda_fail(err, "cudaEventCreate");
    }
  }
  return MOE_OK;
}

moe_status moe_profile_read(moe_plan_t *plan, moe_stream_t stream, double *ms, int32_t *launches) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  MOE_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)), "stream synchronize");
  double acc[MOE_KERNEL_COUNT] = {0};
  int32_t cnt[MOE_KERNEL_COUNT] = {0};
  for (int i = 0; i < plan->prof_used; ++i) {
    float t = 0.f;
    MOE_CUDA(cudaEventElapsedTime(&t, plan->prof_events[2 * i], plan->prof_events[2 * i + 1]), "event time");
    acc[plan->prof_kind[i]] += t;
    cnt[plan->prof_kind[i]] += 1;
  }
  plan->prof_used = 0;
  for (int k = 0; k < MOE_KERNEL_COUNT; ++k) {
    if (ms) ms[k] = acc[k];
    if (launches) launches[k] = cnt[k];
  }
  return MOE_OK;
}

moe_status moe_status_sync(moe_plan_t *plan, moe_stream_t stream) {
  g_last_error.clear();
  if (!plan) return fail(MOE_ERR_INVALID_ARG, "plan is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  MOE_CUDA(cudaStreamSynchronize(s), "stream synchronize");
  DevStatus h;
  MOE_CUDA(cudaMemcpy(&h, plan->status, sizeof h, cudaMemcpyDeviceToHost), "read status");
  if (h.code == kDevOk) return MOE_OK;
  // clear the status and the small-T counters so the plan can be used again
  // (the small-T launch tag is kept: a later launch must not reuse it)
  MOE_CUDA(cudaMemset(plan->status, 0, sizeof(DevStatus)), "clear status");
  MOE_CUDA(cudaMemset(plan->small_sync, 0, kSmallTCounterWords * 4), "clear small-T counters");
  MOE_CUDA(cudaDeviceSynchronize(), "synchronize");
  if (h.code == kDevTimeout)
    return fail(MOE_ERR_DEVICE_TIMEOUT, "device wait ran out (site %u, block %u)", h.where, h.detail);
  return fail(MOE_ERR_DEVICE_BOUNDS, "device index out of range (site %u, value %u)", h.where, h.detail);
}

}  // extern "C"
