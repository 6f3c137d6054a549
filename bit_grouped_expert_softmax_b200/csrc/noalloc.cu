// noalloc.cu -- the small-T layer without any device allocation.
//
// Some callers cannot call cudaMalloc: code that runs inside an allocator
// callback or a custom memory pool that owns all device memory, embedded
// runtimes that pre-reserve every byte at start-up, or hosts where the
// allocation API is not reachable from the thread that issues work. For them,
// moe_forward_small_t_noalloc runs the fused small-T kernel (batches of at
// most 8 tokens) with its scratch memory -- the per-token SwiGLU outputs, the
// kernel's counters and launch tag, and the device status word -- taken from one
// file-scope __device__ array instead of a plan's workspace. The caller still
// passes all inputs and outputs.
//
// The array is created when the library's module is loaded on a device and
// stays until the process exits, on every GPU that loads the library.
#include <mutex>

#include "moe_b200.h"
#include "kernels.cuh"

namespace moe {
size_t small_t_smem_bytes(int T, int H, int k, int I, int Is);
void set_last_error(const char *msg);  // the message moe_last_error() returns on this thread
}

using namespace moe;

namespace {

constexpr size_t kStaticScratchBytes = 512 * 1024;  // stated maximum
constexpr size_t kSyncOff = 0;                      // the kernel's counters, then its launch tag
constexpr size_t kStatusOff = 1024;                 // DevStatus
constexpr size_t kHeaderBytes = 1280;
constexpr size_t kHOff = kHeaderBytes;              // SwiGLU outputs, 8 * (top_k + 1) * max(I, Is) tagged values
constexpr int kMaxDevices = 64;
static_assert(kSmallTSyncWords * 4 <= kStatusOff - kSyncOff, "counters fit the header");

// [0, 12): the kernel's exit and router counters (cleared before every
// launch) and its last launch tag (kept: a launch must not reuse the tag of
// one before it); [1024, 1040): DevStatus (cleared before every launch);
// [1280, kStaticScratchBytes): SwiGLU outputs by token and slot as 8-byte
// words of two fp16 values and a launch tag (zero-initialised with the module).
static __device__ __align__(256) unsigned char g_small_t_scratch[kStaticScratchBytes];

struct DeviceSlot {
  bool ready = false;
  unsigned char *ptr = nullptr;  // device address of g_small_t_scratch on this device
  int num_sms = 0;
};
DeviceSlot g_slots[kMaxDevices];
std::mutex g_slots_mu;

moe_status fail(moe_status st, const char *msg) {
  set_last_error(msg);
  return st;
}

// The array's device address on the current device, looked up (with that
// device current) on the first call that succeeds; a failed lookup is not
// remembered, so a later call retries it.
cudaError_t device_slot(int dev, DeviceSlot *&out) {
  std::lock_guard<std::mutex> lock(g_slots_mu);
  DeviceSlot &slot = g_slots[dev];
  if (!slot.ready) {
    unsigned char *ptr = nullptr;
    int sms = 0;
    cudaError_t err = cudaGetSymbolAddress(reinterpret_cast<void **>(&ptr), g_small_t_scratch);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess || !ptr) {
      cudaGetLastError();  // clear the (non-sticky) error so the caller's next CUDA call does not see it
      return err != cudaSuccess ? err : cudaErrorInvalidSymbol;
    }
    slot.ptr = ptr;
    slot.num_sms = sms;
    slot.ready = true;
  }
  out = &slot;
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_forward_small_t_noalloc(int T, int hidden, int n_experts, int top_k, int inter,
                                                  int shared_inter, const void *x_bf16, const float *router_logits,
                                                  const uint32_t *packed_w, const void *scales, const void *biases,
                                                  const uint32_t *shared_packed_w, const void *shared_scales,
                                                  const void *shared_biases, void *out_bf16, void *status_out,
                                                  moe_stream_t stream) {
  set_last_error("");
  if (T < 0 || T > kSmallT) return fail(MOE_ERR_INVALID_ARG, "T must be in [0, 8]");
  if (hidden < 256 || hidden % 256 || hidden > 16384)
    return fail(MOE_ERR_INVALID_ARG, "hidden must be a positive multiple of 256 (at most 16384)");
  if (inter < 128 || inter % 128 || inter > 8192 || shared_inter < 128 || shared_inter % 128 || shared_inter > 8192)
    return fail(MOE_ERR_INVALID_ARG, "inter and shared_inter must be positive multiples of 128 (at most 8192)");
  if (n_experts < 1 || n_experts > kMaxExperts || top_k < 1 || top_k > n_experts || top_k > kMaxTopK)
    return fail(MOE_ERR_INVALID_ARG, "need 1 <= top_k <= min(n_experts, 16) and n_experts <= 256");
  const size_t imax = static_cast<size_t>(inter > shared_inter ? inter : shared_inter);
  const size_t h_bytes = static_cast<size_t>(kSmallT) * (top_k + 1) * imax * 4;  // a tagged word per 2 values
  if (kHOff + h_bytes > kStaticScratchBytes)
    return fail(MOE_ERR_UNSUPPORTED, "8 * (top_k + 1) * max(inter, shared_inter) * 4 bytes exceeds the 512 KiB "
                                     "static scratch (less its 1280-byte header)");
  if (status_out && (reinterpret_cast<uintptr_t>(status_out) & 15u))
    return fail(MOE_ERR_INVALID_ARG, "status_out must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) {  // nothing to compute; the status of this call is OK
    if (status_out && cudaMemsetAsync(status_out, 0, sizeof(DevStatus), s) != cudaSuccess)
      return fail(MOE_ERR_CUDA, "clearing status_out failed");
    return MOE_OK;
  }
  const void *ptrs[9] = {x_bf16, router_logits, packed_w, scales, biases, shared_packed_w, shared_scales,
                         shared_biases, out_bf16};
  for (int i = 0; i < 9; ++i)
    if (!ptrs[i] || (reinterpret_cast<uintptr_t>(ptrs[i]) & 15u))
      return fail(MOE_ERR_INVALID_ARG, "tensor pointers must be non-NULL and 16-byte aligned");
  if (x_bf16 == out_bf16) return fail(MOE_ERR_INVALID_ARG, "out must not alias x");

  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(MOE_ERR_NO_DEVICE, "no current CUDA device");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOE_ERR_UNSUPPORTED, "device ordinal above 63");
  DeviceSlot *slot = nullptr;
  if (device_slot(dev, slot) != cudaSuccess)
    return fail(MOE_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed");
  if (!small_t_fits(T, hidden, top_k, inter, shared_inter, slot->num_sms))
    return fail(MOE_ERR_UNSUPPORTED, "layer too large for the small-T kernel (shared memory or hidden/16 > SMs)");

  // the array keeps the previous call's contents: clear the counters and the
  // status word (the launch tag stays)
  err = cudaMemsetAsync(slot->ptr + kSyncOff, 0, kSmallTCounterWords * 4, s);
  if (err == cudaSuccess) err = cudaMemsetAsync(slot->ptr + kStatusOff, 0, sizeof(DevStatus), s);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "clearing the static scratch header failed");
  SmallTArgs a{};  // value-initialised: every field not set below is zero (no router: logits are given)
  a.T = T; a.E = n_experts; a.k = top_k; a.H = hidden; a.I = inter; a.Is = shared_inter;
  a.x = static_cast<const uint16_t *>(x_bf16);
  a.logits = router_logits;
  a.router_w = nullptr;
  a.w.packed = packed_w;
  a.w.scales = static_cast<const uint16_t *>(scales);
  a.w.biases = static_cast<const uint16_t *>(biases);
  a.w.sh_packed = shared_packed_w;
  a.w.sh_scales = static_cast<const uint16_t *>(shared_scales);
  a.w.sh_biases = static_cast<const uint16_t *>(shared_biases);
  a.sync = reinterpret_cast<uint32_t *>(slot->ptr + kSyncOff);
  a.status = reinterpret_cast<DevStatus *>(slot->ptr + kStatusOff);
  a.hbuf = reinterpret_cast<uint64_t *>(slot->ptr + kHOff);
  a.residual = nullptr;
  a.out = static_cast<uint16_t *>(out_bf16);
  a.wait_ns = kWaitBudgetNs;
  a.test_fault = 0;
  err = launch_small_t(a, slot->num_sms, s, false);
  if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "small-T kernel launch failed");
  if (status_out) {
    err = cudaMemcpyAsync(status_out, slot->ptr + kStatusOff, sizeof(DevStatus), cudaMemcpyDeviceToDevice, s);
    if (err != cudaSuccess) return fail(MOE_ERR_CUDA, "copying the device status failed");
  }
  return MOE_OK;
}
