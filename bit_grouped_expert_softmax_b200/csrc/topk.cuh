// topk.cuh -- warp-level router: softmax over the experts, top-k selection by
// the float32 logits (equal logits: lower expert id first), renormalisation.
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  // larger logit wins; equal logits: lower expert id wins
  return (va > vb) || (va == vb && ia < ib);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// inclusive warp scan of ints
__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Top-k of one token by one warp. Lane l holds experts l, l+32, ... (E <= 256).
// Writes the token's k ids (largest logit first) and weights to lanes 0..k-1's
// out_id / out_w. Every lane returns the same psum.
__device__ __forceinline__ void warp_topk(const float *__restrict__ row, int E, int k, int lane,
                                          int &out_id, float &out_w) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
  }
  // softmax over all E experts (fp32, max-subtracted)
  float m = v[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, v[i]);
  m = warp_max(m);
  float z = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (lane + 32 * i < E) z += expf(v[i] - m);
  z = warp_sum(z);

  uint32_t taken = 0;
  float psum = 0.f, my_p = 0.f;
  int my_id = 0;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      if (e < E && !(taken >> i & 1u) && better(v[i], e, bv, bi)) {
        bv = v[i];
        bi = e;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (better(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    const float p = expf(bv - m) / z;  // softmax probability of the chosen expert
    psum += p;
    if (lane == j) {
      my_id = bi;
      my_p = p;
    }
  }
  out_id = my_id;
  out_w = my_p / psum;  // renormalise the k chosen probabilities to sum to one
}

}  // namespace moe
