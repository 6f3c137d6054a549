// combine.cu -- deterministic combine of the expert outputs of each token.
//
// out_t = bf16( [x_t +] 2^{2e_t} * ( sum_{j=0}^{k-1} Y[inv[t*k+j]] + Y[R+t] ) )
// The routed rows of Y already carry their routing weight; the shared expert's
// row (the expert that sees every token, "Perplexity open sources Lily...",
// section "Requirements and model layout") enters with weight 1. The sum runs in
// this fixed order in fp32 with one final rounding, so the result does not
// depend on scheduling (no floating-point atomics).
#include "kernels.cuh"

namespace moe {

// U rows of a chunk are requested before any of them is added (the adds stay
// in slot order): U = 1 streams one row at a time, which suits the DRAM when
// thousands of tokens keep it busy; a few hundred tokens leave each SM a
// handful of blocks, whose row-by-row round trips then set the time.
template <int U>
__global__ void __launch_bounds__(256) combine_kernel(CombineArgs a) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const int H = a.H, k = a.k;
  __shared__ int rows[kMaxTopK + 1];
  if (threadIdx.x < k) {
    int r = a.inv[static_cast<size_t>(t) * k + threadIdx.x];
    if (a.debug && (r < 0 || r >= a.R)) {  // MOE_FLAG_DEBUG: report and leave the slot out
      report_error(a.status, kDevBounds, 60, static_cast<uint32_t>(t * k + threadIdx.x));
      r = -1;
    }
    rows[threadIdx.x] = r;
  }
  if (threadIdx.x == 0) rows[k] = a.R + t;
  __syncthreads();
  const int e2 = 2 * a.xexp[t];
  for (int c = threadIdx.x; c < H / 8; c += blockDim.x) {
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
    for (int j0 = 0; j0 <= k; j0 += U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u;
        v[u] = make_uint4(0, 0, 0, 0);
        if (j <= k && rows[j] >= 0)
          v[u] = __ldcs(reinterpret_cast<const uint4 *>(a.y + static_cast<size_t>(rows[j]) * H) + c);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int j = j0 + u;
        if (j > k || rows[j] < 0) continue;
        const __half2 *hv = reinterpret_cast<const __half2 *>(&v[u]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __half22float2(hv[q]);
          acc[2 * q] += f.x;
          acc[2 * q + 1] += f.y;
        }
      }
    }
    uint4 res;
    uint32_t *rp = reinterpret_cast<uint32_t *>(&res);
    uint4 xr = make_uint4(0, 0, 0, 0);
    if (a.residual) xr = *(reinterpret_cast<const uint4 *>(a.residual + static_cast<size_t>(t) * H) + c);
    const uint32_t *xp = reinterpret_cast<const uint32_t *>(&xr);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float lo = ldexpf(acc[2 * q], e2), hi = ldexpf(acc[2 * q + 1], e2);
      if (a.residual) {
        lo += __uint_as_float(xp[q] << 16);
        hi += __uint_as_float(xp[q] & 0xffff0000u);
      }
      rp[q] = static_cast<uint32_t>(float_to_bf16_bits(lo)) |
              (static_cast<uint32_t>(float_to_bf16_bits(hi)) << 16);
    }
    *(reinterpret_cast<uint4 *>(a.out + static_cast<size_t>(t) * H) + c) = res;
  }
}

// One block copies a host-buffer call's inputs (pinned host memory, read
// through the host mapping once) into the plan's device staging buffers;
// n16: 16-byte chunks, tail: the last bytes of the logits, 4 at a time.
__global__ void __launch_bounds__(256) host_stage_kernel(HostStageArgs a) {
  pdl_wait();  // the staging buffers may still be read by the kernel ahead
  pdl_trigger();
  for (int i = threadIdx.x; i < a.x16; i += blockDim.x) a.x_dev[i] = a.x_host[i];
  for (int i = threadIdx.x; i < a.l4; i += blockDim.x) a.l_dev[i] = a.l_host[i];
}

cudaError_t launch_host_stage(const HostStageArgs &a, cudaStream_t s, bool pdl) {
  return launch_k(host_stage_kernel, dim3(1), dim3(256), 0, s, pdl, a);
}

constexpr int kCombineFewTokens = 1024;  // at most this many tokens: rows requested nine at a time

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t s, bool pdl) {
  if (a.T <= 0) return cudaSuccess;
  if (a.T <= kCombineFewTokens) return launch_k(combine_kernel<9>, dim3(a.T), dim3(256), 0, s, pdl, a);
  return launch_k(combine_kernel<1>, dim3(a.T), dim3(256), 0, s, pdl, a);
}

}  // namespace moe
