// gemm_simt.cu -- grouped gate/up and down GEMMs on CUDA cores.
//
// Same work lists, operand layouts and epilogues as the tensor-core kernels;
// kept only while those are brought up.
#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kSimtThreads = 256;
constexpr int kSubN = 32;  // activation rows per inner pass

__device__ __forceinline__ const __half *h_row(const GemmArgs &a, int row, bool shared) {
  return shared ? a.h + a.h_shared_off + static_cast<int64_t>(row - a.R) * a.Is
                : a.h + static_cast<int64_t>(row) * a.I;
}

__device__ __forceinline__ int row_token(const GemmArgs &a, int row) {
  return row < a.R ? a.perm[row] / a.k : row - a.R;
}

}  // namespace

__global__ void __launch_bounds__(kSimtThreads) gemm_gate_up_simt(GemmArgs a) {
  __shared__ __align__(16) __half Ws[2][kTileM][kTileK + 8];
  __shared__ __align__(16) __half Xs[kSubN][kTileK + 8];
  if (blockIdx.x >= *a.item_count) return;
  const WorkItem wi = a.items[blockIdx.x];
  const bool shared = wi.group == a.E;
  const int I = shared ? a.Is : a.I, H = a.H;
  const uint32_t *P = shared ? a.w.sh_packed : a.w.packed + static_cast<size_t>(wi.group) * 3 * a.I * H / 8;
  const uint16_t *S = shared ? a.w.sh_scales : a.w.scales + static_cast<size_t>(wi.group) * 3 * a.I * H / 64;
  const uint16_t *B = shared ? a.w.sh_biases : a.w.biases + static_cast<size_t>(wi.group) * 3 * a.I * H / 64;
  const int tid = threadIdx.x, i = tid & (kTileM - 1), tg = tid >> 7;
  for (int tb = 0; tb < wi.nrows; tb += kSubN) {
    float ag[16], au[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) ag[t] = au[t] = 0.f;
    for (int kb = 0; kb < H; kb += kTileK) {
      for (int idx = tid; idx < 2 * kTileM * 8; idx += kSimtThreads) {
        const int mat = idx >> 10, r = (idx >> 3) & (kTileM - 1), c = idx & 7;
        const int row = mat * I + wi.mblk * kTileM + r;
        const uint32_t word = P[static_cast<size_t>(row) * (H / 8) + kb / 8 + c];
        const size_t gi = static_cast<size_t>(row) * (H / 64) + kb / 64;
        *reinterpret_cast<uint4 *>(&Ws[mat][r][c * 8]) =
            dequant_word(word, bf16_to_half2_bcast(S[gi]), bf16_to_half2_bcast(B[gi]));
      }
      {
        const int r = tid >> 3, c = tid & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (tb + r < wi.nrows)
          v = *reinterpret_cast<const uint4 *>(a.xt + static_cast<size_t>(wi.row0 + tb + r) * H + kb + c * 8);
        *reinterpret_cast<uint4 *>(&Xs[r][c * 8]) = v;
      }
      __syncthreads();
      for (int kk = 0; kk < kTileK; ++kk) {
        const float wg = __half2float(Ws[0][i][kk]), wu = __half2float(Ws[1][i][kk]);
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const float xv = __half2float(Xs[tg * 16 + t][kk]);
          ag[t] = fmaf(wg, xv, ag[t]);
          au[t] = fmaf(wu, xv, au[t]);
        }
      }
      __syncthreads();
    }
    const int col = wi.mblk * kTileM + i;
    const int stored = (col & ~7) + kperm_dst(col & 7);
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const int r = tb + tg * 16 + t;
      if (r < wi.nrows) {
        const int row = wi.row0 + r;
        const int e = a.xexp[row_token(a, row)];
        const float hv = swiglu_scaled(ag[t], au[t], e);
        const_cast<__half *>(h_row(a, row, shared))[stored] = __float2half_rn(hv);
      }
    }
  }
}

__global__ void __launch_bounds__(kSimtThreads) gemm_down_simt(GemmArgs a) {
  __shared__ __align__(16) __half Ws[kTileM][kTileK + 8];
  __shared__ __align__(16) __half Xs[kSubN][kTileK + 8];
  if (blockIdx.x >= *a.item_count) return;
  const WorkItem wi = a.items[blockIdx.x];
  const bool shared = wi.group == a.E;
  const int I = shared ? a.Is : a.I, H = a.H;
  const uint32_t *P = (shared ? a.w.sh_packed : a.w.packed + static_cast<size_t>(wi.group) * 3 * a.I * H / 8) +
                      static_cast<size_t>(2) * I * H / 8;
  const size_t goff = static_cast<size_t>(2) * I * H / 64;
  const uint16_t *S = (shared ? a.w.sh_scales : a.w.scales + static_cast<size_t>(wi.group) * 3 * a.I * H / 64) + goff;
  const uint16_t *B = (shared ? a.w.sh_biases : a.w.biases + static_cast<size_t>(wi.group) * 3 * a.I * H / 64) + goff;
  const int tid = threadIdx.x, i = tid & (kTileM - 1), tg = tid >> 7;
  for (int tb = 0; tb < wi.nrows; tb += kSubN) {
    float acc[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) acc[t] = 0.f;
    for (int kb = 0; kb < I; kb += kTileK) {
      for (int idx = tid; idx < kTileM * 8; idx += kSimtThreads) {
        const int r = idx >> 3, c = idx & 7;
        const int row = wi.mblk * kTileM + r;
        const uint32_t word = P[static_cast<size_t>(row) * (I / 8) + kb / 8 + c];
        const size_t gi = static_cast<size_t>(row) * (I / 64) + kb / 64;
        *reinterpret_cast<uint4 *>(&Ws[r][c * 8]) =
            dequant_word(word, bf16_to_half2_bcast(S[gi]), bf16_to_half2_bcast(B[gi]));
      }
      {
        const int r = tid >> 3, c = tid & 7;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (tb + r < wi.nrows) v = *reinterpret_cast<const uint4 *>(h_row(a, wi.row0 + tb + r, shared) + kb + c * 8);
        *reinterpret_cast<uint4 *>(&Xs[r][c * 8]) = v;
      }
      __syncthreads();
      for (int kk = 0; kk < kTileK; ++kk) {
        const float wv = __half2float(Ws[i][kk]);
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = fmaf(wv, __half2float(Xs[tg * 16 + t][kk]), acc[t]);
      }
      __syncthreads();
    }
    const int n = wi.mblk * kTileM + i;
#pragma unroll
    for (int t = 0; t < 16; ++t) {
      const int r = tb + tg * 16 + t;
      if (r < wi.nrows) {
        const int row = wi.row0 + r;
        const float w = row < a.R ? a.wts[a.perm[row]] : 1.0f;
        a.y[static_cast<size_t>(row) * H + n] = __float2half_rn(w * acc[t]);
      }
    }
  }
}

cudaError_t launch_gemm_gate_up(const GemmArgs &a, int, cudaStream_t s) {
  if (a.max_items <= 0) return cudaSuccess;
  gemm_gate_up_simt<<<a.max_items, kSimtThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gemm_down(const GemmArgs &a, int, cudaStream_t s) {
  if (a.max_items <= 0) return cudaSuccess;
  gemm_down_simt<<<a.max_items, kSimtThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
