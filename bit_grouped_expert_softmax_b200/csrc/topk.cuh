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

// Order-preserving unsigned key of a float (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Top-k of one token by one warp. Lane l holds experts l, l+32, ... (E <= 256).
// Each round takes the largest remaining float32 logit (two warp reductions:
// the maximum key, then the lowest expert id holding it), so equal logits go
// to the lower id. Lanes 0..k-1 return the chosen ids (largest logit first)
// in out_id and their weights in out_w: the softmax over all E experts (fp32,
// max-subtracted) restricted to the chosen k and renormalised to sum to one.
__device__ __forceinline__ void warp_topk(const float *__restrict__ row, int E, int k, int lane,
                                          int &out_id, float &out_w) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane + 32 * i;
    v[i] = (e < E) ? __ldg(row + e) : -INFINITY;
  }
  uint32_t taken = 0, my_key = 0;
  int my_id = 0;
  float m = 0.f, z = 0.f;
  for (int j = 0; j < k; ++j) {
    uint32_t bk = 0;  // 0: no candidate in this lane (every float key is > 0)
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int e = lane + 32 * i;
      const uint32_t kk = float_key(v[i]);
      if (e < E && !(taken >> i & 1u) && kk > bk) {  // ascending e: ties keep the lower id
        bk = kk;
        bi = e;
      }
    }
    const uint32_t mk = __reduce_max_sync(0xffffffffu, bk);
    const int win = static_cast<int>(__reduce_min_sync(0xffffffffu, bk == mk ? static_cast<uint32_t>(bi) : 0xffffffffu));
    if ((win & 31) == lane) taken |= 1u << (win >> 5);
    if (lane == j) {
      my_id = win;
      my_key = mk;
    }
    if (j == 0) {  // the first pick is the maximum: softmax denominator over all E
      m = key_float(mk);
      float zz = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (lane + 32 * i < E) zz += expf(v[i] - m);
      z = warp_sum(zz);
    }
  }
  const float p = (lane < k) ? expf(key_float(my_key) - m) / z : 0.f;  // softmax probability
  const float psum = warp_sum(p);
  out_id = my_id;
  out_w = p / psum;  // renormalise the k chosen probabilities to sum to one
}

}  // namespace moe
