// router.cu -- router scores of the grouped path on the 5th-generation tensor
// cores: logits[t, e] = sum_h x[t, h] * W_router[e, h] (bfloat16 operands,
// float32 accumulation).
//
// The router scores every expert of a token before the top k are chosen
// ("Perplexity open sources Lily...", section "Requirements and model
// layout"). It is a plain dense contraction, so it runs as one: tiles of 128
// tokens x 128 experts, K = H in 64-element blocks, both operands staged by
// TMA (128-byte swizzle) and multiplied by tcgen05.mma into a 128-column fp32
// accumulator in tensor memory.
//
// Warp roles (128 threads): warp 0 lane 0 issues the TMA loads, warp 1 one
// elected lane issues the MMAs, all four warps read the accumulator back
// (warp w owns tensor-memory lanes 32w..32w+31, i.e. tokens) and store the
// float32 scores. Every wait is bounded.
#include <algorithm>

#include "gemm_common.cuh"

namespace moe {

namespace {

using namespace sm100;
using namespace gemm;

constexpr int kRThreads = 128;
constexpr int kRM = 128;        // tokens per tile (MMA M)
constexpr int kRN = 128;        // experts per tile (MMA N, at most)
constexpr int kRStages = 4;
constexpr int kRAtom = kRM * 128;  // one K-block (64 bf16) of 128 rows
constexpr int kRStageBytes = 2 * kRAtom;
constexpr int kRSmem = kRStages * kRStageBytes + 2 * kRStages * 8 + 8 + 64 + 1024;
static_assert(kRSmem <= 227 * 1024, "shared memory budget");

// Instruction descriptor: bf16 A and B, both K-major, fp32 accumulator, M x N.
constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7) | (1u << 10)                    // A, B format: bf16 (the same type on both sides)
         | (0u << 15) | (0u << 16)                   // A, B K-major
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

struct RouterTmaMaps {
  CUtensorMap x;  // [T, H] bf16
  CUtensorMap w;  // [E, H] bf16
};

__global__ void __launch_bounds__(kRThreads, 1) router_kernel(const RouterArgs a,
                                                              const __grid_constant__ RouterTmaMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kRStages * kRStageBytes);
  uint64_t *empty = full + kRStages;
  uint64_t *done = empty + kRStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  volatile int *abort = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kRM, e0 = blockIdx.y * kRN;
  const int ne = min(kRN, a.E - e0);           // experts of this tile
  const int n_mma = (ne + 15) & ~15;           // MMA N: a multiple of 16
  const int nkb = a.H / 64;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kRN);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&maps.x);
    tma_prefetch_desc(&maps.w);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();  // x may come from the kernel before this one
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      TmaRing<kRStages> ring;
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb, ring.advance()) {
        if (!ring.claim(empty, full, kRStageBytes, abort, a.status, 300)) {
          ok = false;
          break;
        }
        uint8_t *st = smem + ring.s * kRStageBytes;
        tma_load_2d(st, &maps.x, &full[ring.s], kb * 64, t0);  // rows past T (or E) read as zeros
        tma_load_2d(st + kRAtom, &maps.w, &full[ring.s], kb * 64, e0);
      }
      if (!ok) ring.drain(full);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kRM, n_mma);
    bool ok = true;
    for (int kb = 0; kb < nkb && ok; ++kb) {
      const int s = kb % kRStages;
      if (!warp_wait(&full[s], (kb / kRStages) & 1u, abort, a.status, 301)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t aa = smem_u32(smem + s * kRStageBytes), bb = aa + kRAtom;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          tc_mma_f16(tmem_base, smem_desc_sw128(aa + kk * 32), smem_desc_sw128(bb + kk * 32), idesc,
                     (kb | kk) != 0 ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      __syncwarp();
    }
    // the accumulator is complete once every MMA issued so far has finished
    if (elect_one()) tc_commit(done);
    __syncwarp();
  }
  // ------------------------------------------------ epilogue (all warps)
  int okd = 1;
  if (lane == 0) {
    const unsigned long long tw = global_ns();
    while (!mbar_try_wait(done, 0)) {
      if (global_ns() - tw > kWaitBudgetNs) {
        report_error(a.status, kDevTimeout, 302, blockIdx.x);
        okd = 0;
        break;
      }
    }
  }
  okd = __shfl_sync(0xffffffffu, okd, 0);
  tc_fence_after();
  const int t = t0 + warp * 32 + lane;  // this thread's token (tensor-memory lane)
  if (okd && !*abort) {
    for (int c0 = 0; c0 < ne; c0 += 32) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + c0, r);
      tmem_ld_wait();
      if (t < a.T) {
        float *dst = a.logits + static_cast<size_t>(t) * a.E + e0 + c0;
        if (c0 + 32 <= ne && (a.E % 4) == 0) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(dst + i) = make_float4(__uint_as_float(r[i]), __uint_as_float(r[i + 1]),
                                                               __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (c0 + i < ne) dst[i] = __uint_as_float(r[i]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kRN);
  }
}

}  // namespace

cudaError_t launch_router(const RouterArgs &a, cudaStream_t s, bool pdl) {
  if (a.T <= 0) return cudaSuccess;
  RouterTmaMaps maps;
  bool ok = make_map(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.x, static_cast<uint64_t>(a.T), a.H, kRM, 64,
                     CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.w, static_cast<uint64_t>(a.E), a.H, kRN, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e = ensure_smem_limit(router_kernel, kRSmem, smem_set);
  if (e != cudaSuccess) return e;
  const dim3 grid((a.T + kRM - 1) / kRM, (a.E + kRN - 1) / kRN);
  return launch_k(router_kernel, grid, dim3(kRThreads), kRSmem, s, pdl, a, maps);
}

}  // namespace moe
