// small_t.cu -- fused MoE layer for batches of up to 8 tokens.
//
// Batch-1 decode has almost no weight reuse, so memory bandwidth sets the
// ceiling (aioga.com record of the Lily report, article body paragraph 6).
// One persistent kernel, one CTA per SM, does the whole layer:
//   phase 0  every CTA routes the (<= 8) tokens itself (same result everywhere),
//            builds the list of distinct experts used, stages x in shared memory
//   phase 1  gate/up rows of the used experts, one row pair per warp at a time,
//            128-bit coalesced loads of the packed words; each group of 64 uses
//            sum_i x_i (q_i s + b) = s * sum_i x_i q_i + b * sum_i x_i in fp32;
//            h = silu(gate) * up goes to a small fp32 scratch buffer
//   barrier  bounded grid barrier (the launch is cooperative)
//   phase 2  down rows: each warp owns output columns n and sums, per token,
//            w_j * y_j over j = 0..k-1 then the shared expert, in that fixed order
#include "kernels.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kSTWarps = 16;
constexpr int kSTThreads = kSTWarps * 32;
constexpr int kXPitch = 68;  // floats per 64-element group of x in shared memory (padded)

struct SmallTShared {
  int ids[kSmallT][kMaxTopK];
  float wt[kSmallT][kMaxTopK];
  int ulist[kSmallT * kMaxTopK + 1];
  uint32_t umask[kSmallT * kMaxTopK + 1];
  int8_t uslot[kSmallT * kMaxTopK + 1][kSmallT];  // slot j of expert u in token t (-1: unused)
  int nU;
  int ok;
};

__device__ __forceinline__ float code_f(uint32_t w, int j) {
  // exact float of the 4-bit code j of w: 2^23 + q as a float, minus 2^23
  return __uint_as_float(0x4B000000u | ((w >> (4 * j)) & 0xFu)) - 8388608.0f;
}

// sum over the 8 codes of a word of q_j * x[j]
__device__ __forceinline__ float dot8(uint32_t w, const float *x) {
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) acc = fmaf(code_f(w, j), x[j], acc);
  return acc;
}

// Grid barrier on {count, generation}; returns false if the wait ran out.
__device__ bool grid_barrier(uint32_t *bar, DevStatus *st, int *ok_flag) {
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile uint32_t *vgen = bar + 1;
    const uint32_t gen = *vgen;
    __threadfence();
    const uint32_t arrived = atomicAdd(bar, 1u);
    if (arrived == gridDim.x - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
      *ok_flag = 1;
    } else {
      const unsigned long long t0 = global_ns();
      int ok = 1;
      unsigned it = 0;
      while (*vgen == gen) {
        if ((++it & 1023u) == 0 && global_ns() - t0 > kWaitBudgetNs) {
          report_error(st, kDevTimeout, 30, blockIdx.x);
          ok = 0;
          break;
        }
      }
      *ok_flag = ok;
    }
    __threadfence();
  }
  __syncthreads();
  return *ok_flag != 0;
}

}  // namespace

int small_t_grid(int num_sms) { return num_sms; }

size_t small_t_smem_bytes(int T, int H, int k, int I, int Is) {
  const size_t ng = H / kGroup;
  const size_t x_bytes = static_cast<size_t>(T) * ng * kXPitch * 4 + static_cast<size_t>(T) * ng * 4;
  const size_t h_bytes = static_cast<size_t>(T) * (k + 1) * (I > Is ? I : Is) * 4;
  return x_bytes > h_bytes ? x_bytes : h_bytes;
}

__global__ void __launch_bounds__(kSTThreads, 1) small_t_kernel(SmallTArgs a) {
  extern __shared__ __align__(16) float dyn[];
  __shared__ SmallTShared sh;
  const int T = a.T, E = a.E, k = a.k, H = a.H;
  const int ng = H / kGroup;
  const int Imax = a.I > a.Is ? a.I : a.Is;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float *xs = dyn;                             // [T][ng][kXPitch]
  float *xg = dyn + static_cast<size_t>(T) * ng * kXPitch;  // [T][ng] group sums

  // ---- phase 0: routing and staging -------------------------------------------
  if (warp < T) {
    int id;
    float w;
    warp_topk(a.logits + static_cast<size_t>(warp) * E, E, k, lane, id, w);
    if (lane < k) {
      sh.ids[warp][lane] = id;
      sh.wt[warp][lane] = w;
    }
  }
  for (int idx = threadIdx.x; idx < T * H / 2; idx += kSTThreads) {
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t *>(a.x) + idx);
    const int t = (2 * idx) / H, h = (2 * idx) % H;
    float *dst = xs + (static_cast<size_t>(t) * ng + h / kGroup) * kXPitch + (h % kGroup);
    dst[0] = __uint_as_float(v << 16);
    dst[1] = __uint_as_float(v & 0xffff0000u);
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < T * ng; idx += kSTThreads) {
    const float *src = xs + static_cast<size_t>(idx) * kXPitch;
    float s = 0.f;
    for (int i = 0; i < kGroup; ++i) s += src[i];
    xg[idx] = s;
  }
  if (warp == 0) {
    // distinct experts in ascending order, then the shared expert
    int n = 0;
    for (int eb = 0; eb < E; eb += 32) {
      const int e = eb + lane;
      uint32_t m = 0;
      int8_t slots[kSmallT];
#pragma unroll
      for (int t = 0; t < kSmallT; ++t) slots[t] = -1;
      if (e < E)
        for (int t = 0; t < T; ++t)
          for (int j = 0; j < k; ++j)
            if (sh.ids[t][j] == e) {
              m |= 1u << t;
              slots[t] = static_cast<int8_t>(j);
            }
      const unsigned bal = __ballot_sync(0xffffffffu, m != 0);
      if (m) {
        const int pos = n + __popc(bal & ((1u << lane) - 1u));
        sh.ulist[pos] = e;
        sh.umask[pos] = m;
#pragma unroll
        for (int t = 0; t < kSmallT; ++t) sh.uslot[pos][t] = slots[t];
      }
      n += __popc(bal);
    }
    if (lane == 0) {
      sh.ulist[n] = E;
      sh.umask[n] = (1u << T) - 1u;
      for (int t = 0; t < kSmallT; ++t) sh.uslot[n][t] = static_cast<int8_t>(k);
      sh.nU = n + 1;
    }
  }
  __syncthreads();
  const int nU = sh.nU;

  // ---- phase 1: gate/up ---------------------------------------------------------
  const int gw = blockIdx.x * kSTWarps + warp, W = gridDim.x * kSTWarps;
  const int routed_rows = (nU - 1) * a.I;
  const int total_rows = routed_rows + a.Is;
  for (int ur = gw; ur < total_rows; ur += W) {
    int u, i, Iu;
    const uint32_t *P;
    const uint16_t *S, *B;
    if (ur < routed_rows) {
      u = ur / a.I;
      i = ur % a.I;
      Iu = a.I;
      const size_t e = sh.ulist[u];
      P = a.w.packed + e * 3 * a.I * H / 8;
      S = a.w.scales + e * 3 * a.I * H / kGroup;
      B = a.w.biases + e * 3 * a.I * H / kGroup;
    } else {
      u = nU - 1;
      i = ur - routed_rows;
      Iu = a.Is;
      P = a.w.sh_packed;
      S = a.w.sh_scales;
      B = a.w.sh_biases;
    }
    const uint32_t mask = sh.umask[u];
    float accg[kSmallT], accu[kSmallT];
#pragma unroll
    for (int t = 0; t < kSmallT; ++t) accg[t] = accu[t] = 0.f;
    for (int g = lane; g < ng; g += 32) {
      const uint4 *pg = reinterpret_cast<const uint4 *>(P + static_cast<size_t>(i) * (H / 8) + g * 8);
      const uint4 *pu = reinterpret_cast<const uint4 *>(P + static_cast<size_t>(Iu + i) * (H / 8) + g * 8);
      const uint4 g0 = __ldcs(pg), g1 = __ldcs(pg + 1), u0 = __ldcs(pu), u1 = __ldcs(pu + 1);
      const float sg = bf16_bits_to_float(S[static_cast<size_t>(i) * ng + g]);
      const float bg = bf16_bits_to_float(B[static_cast<size_t>(i) * ng + g]);
      const float su = bf16_bits_to_float(S[static_cast<size_t>(Iu + i) * ng + g]);
      const float bu = bf16_bits_to_float(B[static_cast<size_t>(Iu + i) * ng + g]);
      const uint32_t gw8[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      const uint32_t uw8[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
      for (int t = 0; t < kSmallT; ++t) {
        if (t >= T || !((mask >> t) & 1u)) continue;
        const float *xr = xs + (static_cast<size_t>(t) * ng + g) * kXPitch;
        float dg = 0.f, du = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          float xv[8];
          *reinterpret_cast<float4 *>(&xv[0]) = *reinterpret_cast<const float4 *>(xr + 8 * q);
          *reinterpret_cast<float4 *>(&xv[4]) = *reinterpret_cast<const float4 *>(xr + 8 * q + 4);
          dg += dot8(gw8[q], xv);
          du += dot8(uw8[q], xv);
        }
        const float xsum = xg[t * ng + g];
        accg[t] += sg * dg + bg * xsum;
        accu[t] += su * du + bu * xsum;
      }
    }
#pragma unroll
    for (int t = 0; t < kSmallT; ++t) {
      if (t >= T || !((mask >> t) & 1u)) continue;
      const float G = warp_sum(accg[t]), U = warp_sum(accu[t]);
      if (lane == 0) {
        const int j = sh.uslot[u][t];
        a.hbuf[(static_cast<size_t>(t) * (k + 1) + j) * Imax + i] = G / (1.0f + __expf(-G)) * U;
      }
    }
  }

  // ---- grid barrier ---------------------------------------------------------------
  if (!grid_barrier(a.barrier, a.status, &sh.ok)) return;

  // ---- phase 2: down + combine -----------------------------------------------------
  float *hp = dyn;  // [T][k+1][Imax], reuses the x staging area
  const int npair = T * (k + 1);
  for (int idx = threadIdx.x; idx < npair * Imax / 4; idx += kSTThreads)
    reinterpret_cast<float4 *>(hp)[idx] = __ldcg(reinterpret_cast<const float4 *>(a.hbuf) + idx);
  __syncthreads();
  for (int n = gw; n < H; n += W) {
    for (int t = 0; t < T; ++t) {
      float acc = 0.f;
      for (int j = 0; j <= k; ++j) {
        const bool shared = j == k;
        const int Iu = shared ? a.Is : a.I;
        const uint32_t *P;
        const uint16_t *S, *B;
        if (shared) {
          P = a.w.sh_packed;
          S = a.w.sh_scales;
          B = a.w.sh_biases;
        } else {
          const size_t e = sh.ids[t][j];
          P = a.w.packed + e * 3 * a.I * H / 8;
          S = a.w.scales + e * 3 * a.I * H / kGroup;
          B = a.w.biases + e * 3 * a.I * H / kGroup;
        }
        P += static_cast<size_t>(2) * Iu * H / 8 + static_cast<size_t>(n) * (Iu / 8);
        S += static_cast<size_t>(2) * Iu * H / kGroup + static_cast<size_t>(n) * (Iu / kGroup);
        B += static_cast<size_t>(2) * Iu * H / kGroup + static_cast<size_t>(n) * (Iu / kGroup);
        const float *hv = hp + (static_cast<size_t>(t) * (k + 1) + j) * Imax;
        float part = 0.f;
        for (int w2 = lane; w2 < Iu / 16; w2 += 32) {
          const uint2 wd = __ldcs(reinterpret_cast<const uint2 *>(P) + w2);
          const int g = w2 / 4;
          const float s = bf16_bits_to_float(S[g]), b = bf16_bits_to_float(B[g]);
          const float *hr = hv + 16 * w2;
          float hx[16];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<float4 *>(&hx[4 * q]) = *reinterpret_cast<const float4 *>(hr + 4 * q);
          const float d = dot8(wd.x, hx) + dot8(wd.y, hx + 8);
          float hs = 0.f;
#pragma unroll
          for (int q = 0; q < 16; ++q) hs += hx[q];
          part += s * d + b * hs;
        }
        const float y = warp_sum(part);
        acc += (shared ? 1.0f : sh.wt[t][j]) * y;
      }
      if (lane == 0) {
        float o = acc;
        if (a.residual) o += bf16_bits_to_float(a.residual[static_cast<size_t>(t) * H + n]);
        a.out[static_cast<size_t>(t) * H + n] = float_to_bf16_bits(o);
      }
    }
  }
}

cudaError_t launch_small_t(const SmallTArgs &a, int num_sms, cudaStream_t s) {
  const size_t smem = small_t_smem_bytes(a.T, a.H, a.k, a.I, a.Is);
  cudaError_t err = cudaFuncSetAttribute(small_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  SmallTArgs args = a;
  void *params[] = {&args};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void *>(small_t_kernel),
                                     dim3(small_t_grid(num_sms)), dim3(kSTThreads), params, smem, s);
}

}  // namespace moe
