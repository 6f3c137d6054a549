// common.cuh -- device helpers shared by the MoE kernels (sm_100a only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library is written for sm_100a (B200) only"
#endif

namespace moe {

constexpr int kGroup = 64;       // weights per scale/bias group (along K)
constexpr int kMaxExperts = 256; // one warp holds a token's logits in 8 registers per lane
constexpr int kMaxTopK = 16;
constexpr int kSmallT = 8;       // batches up to this size take the fused small-T kernel
constexpr int kRouteChunk = 32;     // tokens per routing block, at most
constexpr int kRouteChunkMin = 8;   // ... and at least

// Tokens per routing block for a batch of T: 8 while the batch is small
// (more blocks share the scatter's serial ranking), 32 when it is large
// (fewer chunk columns for the scan, fewer blocks repeating the offset scan);
// measured at T = 512, 4096 and 8192.
inline int route_chunk(int64_t T) {
  return T <= 512 ? kRouteChunkMin : T <= 1024 ? 16 : kRouteChunk;
}

// Device status word: first error wins, later ones are dropped.
enum DevError : uint32_t { kDevOk = 0, kDevTimeout = 1, kDevBounds = 2 };

struct DevStatus {
  uint32_t code;    // DevError
  uint32_t where;   // kernel-specific site id
  uint32_t detail;  // e.g. the offending index
  uint32_t pad;
};

__device__ __forceinline__ void report_error(DevStatus *st, uint32_t code, uint32_t where,
                                             uint32_t detail) {
  if (atomicCAS(&st->code, 0u, code) == 0u) {
    st->where = where;
    st->detail = detail;
  }
}

// Budget for every spin-wait: about two seconds of wall clock.
constexpr unsigned long long kWaitBudgetNs = 2000000000ull;
// Budget of the waits of a launch that carries the test fault (plan flag
// MOE_FLAG_TEST_WAIT_TIMEOUT): the wait that cannot succeed gives up quickly.
constexpr unsigned long long kTestWaitBudgetNs = 2000000ull;

// Programmatic dependent launch. Every kernel of the grouped path runs its
// independent prologue (barrier set-up, tensor-memory allocation, descriptor
// prefetch), then pdl_wait() -- which returns once the kernels it depends on
// have completed and their writes are visible (at once when it was launched
// in plain stream order) -- before its first global-memory access, and then
// pdl_trigger() so the next kernel on the stream may be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------------------
// number formats
// ---------------------------------------------------------------------------

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// float -> bfloat16 bits, round to nearest even (CUDA's conversion)
__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
  __nv_bfloat16 h = __float2bfloat16_rn(f);
  return *reinterpret_cast<uint16_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_half2(__half lo, __half hi) {
  return static_cast<uint32_t>(__half_as_ushort(lo)) |
         (static_cast<uint32_t>(__half_as_ushort(hi)) << 16);
}

// Position of K element j (0..7) of an 8-element block in the fp16 operand
// tiles. The int4 -> fp16 conversion of one packed word naturally yields the
// pairs (0,4), (1,5), (2,6), (3,7); every fp16 operand (dequantised weights,
// gathered activations, the SwiGLU output) stores its K axis in that order
// within each block of 8, so the dot products are unchanged.
//   stored position s holds element kperm_src(s) = (s & 1) * 4 + (s >> 1)
//   element j is stored at position kperm_dst(j) = (j & 3) * 2 + (j >> 2)
__host__ __device__ __forceinline__ int kperm_dst(int j) { return (j & 3) * 2 + (j >> 2); }
__host__ __device__ __forceinline__ int kperm_src(int s) { return (s & 1) * 4 + (s >> 1); }

// ---------------------------------------------------------------------------
// grouped-GEMM work items
// ---------------------------------------------------------------------------

// One output tile of a grouped GEMM: weight rows [mblk*128, mblk*128+128) of
// group g, against rows [row0, row0+nrows) of the gathered activations.
struct WorkItem {
  int32_t group;  // 0..E-1 routed expert, E = shared expert
  int32_t row0;   // first activation row (permuted order)
  int32_t nrows;  // 1..kTileN
  int32_t mblk;   // 128-row block of the weight matrix
};

}  // namespace moe

namespace moe {

// 8 codes of one packed word -> 8 fp16 weights q*scale + bias (one rounding
// each, by one fp16 FMA), returned in the K-permuted operand order.
// The nibble is placed in the mantissa of an fp16 with a fixed exponent
// (1024 + q for bits 0..3, 64 + q for bits 4..7) and the offset subtracted
// exactly: the magic-number int4 -> fp16 conversion published with the MARLIN
// mixed-precision kernels (Frantar et al., arXiv:2408.11743), which also
// yields the pair order (0,4), (1,5), (2,6), (3,7) used for the operands.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, __half2 s2, __half2 b2) {
  const uint32_t hi = w >> 8;
  const uint32_t a0 = (w & 0x000F000Fu) | 0x64006400u;   // {1024+n0, 1024+n4}
  const uint32_t a1 = (w & 0x00F000F0u) | 0x54005400u;   // {64+n1,   64+n5}
  const uint32_t a2 = (hi & 0x000F000Fu) | 0x64006400u;  // {1024+n2, 1024+n6}
  const uint32_t a3 = (hi & 0x00F000F0u) | 0x54005400u;  // {64+n3,   64+n7}
  const __half2 k1024 = __halves2half2(__ushort_as_half(0x6400), __ushort_as_half(0x6400));
  const __half2 k64 = __halves2half2(__ushort_as_half(0x5400), __ushort_as_half(0x5400));
  __half2 q0 = __hsub2(*reinterpret_cast<const __half2 *>(&a0), k1024);
  __half2 q1 = __hsub2(*reinterpret_cast<const __half2 *>(&a1), k64);
  __half2 q2 = __hsub2(*reinterpret_cast<const __half2 *>(&a2), k1024);
  __half2 q3 = __hsub2(*reinterpret_cast<const __half2 *>(&a3), k64);
  q0 = __hfma2(q0, s2, b2);
  q1 = __hfma2(q1, s2, b2);
  q2 = __hfma2(q2, s2, b2);
  q3 = __hfma2(q3, s2, b2);
  uint4 r;
  r.x = *reinterpret_cast<uint32_t *>(&q0);
  r.y = *reinterpret_cast<uint32_t *>(&q1);
  r.z = *reinterpret_cast<uint32_t *>(&q2);
  r.w = *reinterpret_cast<uint32_t *>(&q3);
  return r;
}

// bf16 scale/bias bits -> broadcast fp16x2 pair
__device__ __forceinline__ __half2 bf16_to_half2_bcast(uint16_t b) {
  const __half h = __float2half_rn(bf16_bits_to_float(b));
  return __halves2half2(h, h);
}

// silu applied to the unscaled gate value, the result rescaled back:
// with gate = g * 2^e and up = u * 2^e, returns silu(gate) * up * 2^-2e.
__device__ __forceinline__ float swiglu_scaled(float g, float u, int e) {
  const float gt = ldexpf(g, e);
  const float sg = gt / (1.0f + __expf(-gt));
  return ldexpf(sg, -e) * u;
}

}  // namespace moe
