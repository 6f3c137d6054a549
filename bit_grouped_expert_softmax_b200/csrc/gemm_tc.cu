// gemm_tc.cu -- grouped expert GEMMs on the 5th-generation tensor cores.
//
// The pages' engine rebuilds the 4-bit weights one tile at a time inside the
// grouped GEMM, keeping the expanded tile on chip and accumulating in fp32, so
// the expanded array never reaches memory ("Perplexity open sources Lily...",
// section "Measurements"; aioga.com record, article body paragraph 4). This is
// that scheme on sm_100a:
//
//   TMA (packed int4 words, fp16 activation rows)
//     -> dequant warps: q*scale + bias -> fp16, written in the 128-byte swizzle
//        layout the tensor core reads
//     -> one thread issues tcgen05.mma (A = weights, 128 rows; B = activation
//        rows, N <= 128), fp32 accumulators in tensor memory (TMEM)
//     -> epilogue warps read TMEM (tcgen05.ld):
//          gate/up: h = silu(gate) * up, fp16, into the down GEMM's operand
//          down:    Y = w_routing * (h W_down^T), fp16, by permuted row
//
// The weights are the MMA's M side ("swap AB"): uneven expert groups, including
// ones with a handful of tokens (aioga.com record, paragraph 3: "uneven expert
// groups"), become the N side, which the instruction allows down to 16.
// A persistent grid walks the device-built work list (the block map of the
// routing step); accumulators are double-buffered in TMEM so one tile's
// epilogue overlaps the next tile's main loop. Every wait is bounded.
//
// Warp roles (448 threads): 0 TMA producer, 1 MMA issuer, 2-5 epilogue,
// 6-13 dequantisation.
#include <algorithm>

#include "kernels.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int kThreads = 448;
constexpr int kProducerWarp = 0;
constexpr int kMmaWarp = 1;
constexpr int kEpiWarp0 = 2;
constexpr int kDqWarp0 = 6;
constexpr int kDqThreads = 256;
constexpr int kRawStages = 4;
constexpr int kBRows = 32;                    // TMA box height of activation rows
constexpr int kATileBytes = kTileM * 128;     // 128 rows x 64 fp16
constexpr int kBTileBytes = kTileN * 128;     // 128 rows x 64 fp16
constexpr int kPackedBytes = kTileM * 32;     // 128 rows x 8 words

template <int NMAT>
struct Cfg {
  static constexpr int kAStages = NMAT == 2 ? 3 : 4;
  static constexpr int kAccStages = 2;
  static constexpr int kTmemCols = kAccStages * NMAT * kTileN;  // 512 or 256
  // byte offsets inside the 1024-aligned dynamic shared memory
  static constexpr int kOffA = 0;
  static constexpr int kOffB = kOffA + kAStages * NMAT * kATileBytes;
  static constexpr int kOffP = kOffB + kRawStages * kBTileBytes;
  static constexpr int kOffBar = kOffP + kRawStages * NMAT * kPackedBytes;
  static constexpr int kNumBars = 2 * kRawStages + 2 * kAStages + 2 * kAccStages + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  static constexpr int kSmem = kBytes + 1024;  // slack for aligning the base
};

struct alignas(64) TmaMaps {
  CUtensorMap w;     // packed weights of the routed experts
  CUtensorMap w_sh;  // packed weights of the shared expert
  CUtensorMap b;     // activation rows (gate/up: gathered x; down: routed h)
  CUtensorMap b_sh;  // down only: shared-expert h rows
};

// Lane 0 waits, the whole warp gets the outcome.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort, DevStatus *st,
                                          uint32_t site) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, st, site) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

template <int NMAT>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const GemmArgs a,
                                                                    const __grid_constant__ TmaMaps maps) {
  using C = Cfg<NMAT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sA = smem + C::kOffA;
  uint8_t *sB = smem + C::kOffB;
  uint8_t *sP = smem + C::kOffP;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *raw_full = bars;
  uint64_t *raw_empty = raw_full + kRawStages;
  uint64_t *a_full = raw_empty + kRawStages;
  uint64_t *a_empty = a_full + C::kAStages;
  uint64_t *acc_full = a_empty + C::kAStages;
  uint64_t *acc_empty = acc_full + C::kAccStages;
  uint64_t *mma_done = acc_empty + C::kAccStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool gate_up = NMAT == 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRawStages; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kDqThreads / 32 + 1);  // dequant warps + the MMA's commit
    }
    for (int s = 0; s < C::kAStages; ++s) {
      mbar_init(&a_full[s], kDqThreads / 32);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < C::kAccStages; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], 4);  // four epilogue warps
    }
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&maps.w);
    tma_prefetch_desc(&maps.w_sh);
    tma_prefetch_desc(&maps.b);
    if (!gate_up) tma_prefetch_desc(&maps.b_sh);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int nitems = min(*a.item_count, a.max_items);
  const int H = a.H;

  if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0, issued_ph = 0;  // per-stage bookkeeping for a clean abort
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        const WorkItem wi = a.items[it];
        const bool sh = wi.group == a.E;
        const int Ig = sh ? a.Is : a.I;
        int wrow[NMAT];
        int K;
        if (gate_up) {
          K = H;
          const int base = sh ? 0 : wi.group * 3 * a.I;
          wrow[0] = base + wi.mblk * kTileM;
          if (NMAT == 2) wrow[NMAT - 1] = base + Ig + wi.mblk * kTileM;
        } else {
          K = Ig;
          wrow[0] = (sh ? 0 : wi.group * 3 * H) + 2 * H + wi.mblk * kTileM;
        }
        const CUtensorMap *mw = sh ? &maps.w_sh : &maps.w;
        const CUtensorMap *mb = (!gate_up && sh) ? &maps.b_sh : &maps.b;
        const int brow0 = (!gate_up && sh) ? wi.row0 - a.R : wi.row0;
        const int nb = (wi.nrows + kBRows - 1) / kBRows;
        const uint32_t bytes = NMAT * kPackedBytes + nb * kBRows * 128;
        for (int kb = 0; kb < K / kTileK; ++kb) {
          if (!mbar_wait(&raw_empty[s], ph ^ 1u, abort, a.status, 100)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&raw_full[s], bytes);
          issued |= 1u << s;
          issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
#pragma unroll
          for (int m = 0; m < NMAT; ++m)
            tma_load_2d(sP + (s * NMAT + m) * kPackedBytes, mw, &raw_full[s], kb * 8, wrow[m]);
          for (int j = 0; j < nb; ++j)
            tma_load_2d(sB + s * kBTileBytes + j * kBRows * 128, mb, &raw_full[s], kb * kTileK,
                        brow0 + j * kBRows);
          if (++s == kRawStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // wait (bounded, ignoring the abort flag) for copies still in flight
        for (int t = 0; t < kRawStages; ++t) {
          if (!(issued >> t & 1u)) continue;
          const unsigned long long t0 = global_ns();
          while (!mbar_try_wait(&raw_full[t], issued_ph >> t & 1u) && global_ns() - t0 < kWaitBudgetNs) {
          }
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0, sa = 0;
      uint32_t ph = 0, pha = 0;
      bool ok = true;
      int li = 0;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
        const WorkItem wi = a.items[it];
        const bool sh = wi.group == a.E;
        const int K = gate_up ? H : (sh ? a.Is : a.I);
        const int st = li & 1;
        const uint32_t acc_ph = (li >> 1) & 1;
        if (!mbar_wait(&acc_empty[st], acc_ph ^ 1u, abort, a.status, 110)) break;
        tc_fence_after();
        const int n16 = (wi.nrows + 15) & ~15;
        const uint32_t idesc = idesc_f16_f32(kTileM, n16);
        const uint32_t d0 = tmem_base + st * NMAT * kTileN;
        for (int kb = 0; kb < K / kTileK; ++kb) {
          if (!mbar_wait(&a_full[sa], pha, abort, a.status, 111) ||
              !mbar_wait(&raw_full[s], ph, abort, a.status, 112)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b_addr = smem_u32(sB + s * kBTileBytes);
#pragma unroll
          for (int kk = 0; kk < kTileK / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(b_addr + kk * 32);
#pragma unroll
            for (int m = 0; m < NMAT; ++m) {
              const uint64_t adesc = smem_desc_sw128(smem_u32(sA + (sa * NMAT + m) * kATileBytes) + kk * 32);
              tc_mma_f16(d0 + m * kTileN, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          tc_commit(&raw_empty[s]);
          tc_commit(&a_empty[sa]);
          if (++s == kRawStages) {
            s = 0;
            ph ^= 1u;
          }
          if (++sa == C::kAStages) {
            sa = 0;
            pha ^= 1u;
          }
        }
        if (ok) tc_commit(&acc_full[st]);
      }
      // all issued MMAs finish before tensor memory is released
      tc_commit(mma_done);
      const unsigned long long t0 = global_ns();
      while (!mbar_try_wait(mma_done, 0) && global_ns() - t0 < kWaitBudgetNs) {
      }
    }
  } else if (warp < kDqWarp0) {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int li = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
      const WorkItem wi = a.items[it];
      const bool sh = wi.group == a.E;
      const int st = li & 1;
      const uint32_t acc_ph = (li >> 1) & 1;
      if (!warp_wait(&acc_full[st], acc_ph, abort, a.status, 120)) break;
      tc_fence_after();
      const int mrow = wi.mblk * kTileM + q * 32 + lane;  // weight row of this thread
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + st * NMAT * kTileN;
      for (int c0 = 0; c0 < wi.nrows; c0 += 32) {
        // per-column factor, one column per lane, broadcast by shuffles
        const int jl = c0 + lane;
        float fl = 0.f;
        if (jl < wi.nrows) {
          const int row = wi.row0 + jl;
          if (gate_up) {
            const int tok = row < a.R ? a.perm[row] / a.k : row - a.R;
            fl = __int_as_float(a.xexp[tok]);
          } else {
            fl = row < a.R ? a.wts[a.perm[row]] : 1.0f;
          }
        }
        uint32_t r0[32];
        tmem_ld_32x32b_x32(tq + c0, r0);
        if (gate_up) {
          uint32_t r1[32];
          tmem_ld_32x32b_x32(tq + kTileN + c0, r1);
          tmem_ld_wait();
          const int stored = (mrow & ~7) + kperm_dst(mrow & 7);
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const float f = __shfl_sync(0xffffffffu, fl, jj);
            const int j = c0 + jj;
            if (j < wi.nrows) {
              const int row = wi.row0 + j;
              const float hv = swiglu_scaled(__uint_as_float(r0[jj]), __uint_as_float(r1[jj]), __float_as_int(f));
              __half *hrow = sh ? a.h + a.h_shared_off + static_cast<int64_t>(row - a.R) * a.Is
                                : a.h + static_cast<int64_t>(row) * a.I;
              hrow[stored] = __float2half_rn(hv);
            }
          }
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const float f = __shfl_sync(0xffffffffu, fl, jj);
            const int j = c0 + jj;
            if (j < wi.nrows)
              a.y[static_cast<size_t>(wi.row0 + j) * H + mrow] = __float2half_rn(f * __uint_as_float(r0[jj]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[st]);
    }
  } else {
    // ---------------------------------------------------------------- dequantisation
    const int dq = threadIdx.x - kDqWarp0 * 32;
    const int c = dq & 7;   // word of the 64-element row slice
    const int r0 = dq >> 3; // rows r0, r0+32, r0+64, r0+96
    int s = 0, sa = 0;
    uint32_t ph = 0, pha = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const WorkItem wi = a.items[it];
      const bool sh = wi.group == a.E;
      const int Ig = sh ? a.Is : a.I;
      const uint16_t *S[NMAT];
      const uint16_t *B[NMAT];
      int K;
      if (gate_up) {
        K = H;
        const size_t gbase = sh ? 0 : static_cast<size_t>(wi.group) * 3 * a.I * H / kGroup;
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          const size_t off = gbase + static_cast<size_t>(m * Ig + wi.mblk * kTileM) * (H / kGroup);
          S[m] = (sh ? a.w.sh_scales : a.w.scales) + off;
          B[m] = (sh ? a.w.sh_biases : a.w.biases) + off;
        }
      } else {
        K = Ig;
        const size_t off = (sh ? 0 : static_cast<size_t>(wi.group) * 3 * a.I * H / kGroup) +
                           static_cast<size_t>(2) * Ig * H / kGroup +
                           static_cast<size_t>(wi.mblk * kTileM) * (Ig / kGroup);
        S[0] = (sh ? a.w.sh_scales : a.w.scales) + off;
        B[0] = (sh ? a.w.sh_biases : a.w.biases) + off;
      }
      const int ngr = K / kGroup;  // groups per weight row
      for (int kb = 0; kb < K / kTileK; ++kb) {
        __half2 s2[NMAT][4], b2[NMAT][4];
#pragma unroll
        for (int m = 0; m < NMAT; ++m)
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int r = r0 + 32 * qq;
            s2[m][qq] = bf16_to_half2_bcast(__ldg(S[m] + r * ngr + kb));
            b2[m][qq] = bf16_to_half2_bcast(__ldg(B[m] + r * ngr + kb));
          }
        if (!warp_wait(&raw_full[s], ph, abort, a.status, 130) ||
            !warp_wait(&a_empty[sa], pha ^ 1u, abort, a.status, 131)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int m = 0; m < NMAT; ++m) {
          const uint32_t *pk = reinterpret_cast<const uint32_t *>(sP + (s * NMAT + m) * kPackedBytes);
          uint8_t *at = sA + (sa * NMAT + m) * kATileBytes;
#pragma unroll
          for (int qq = 0; qq < 4; ++qq) {
            const int r = r0 + 32 * qq;
            const uint4 d = dequant_word(pk[r * 8 + c], s2[m][qq], b2[m][qq]);
            *reinterpret_cast<uint4 *>(at + r * 128 + ((c ^ (r & 7)) << 4)) = d;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&a_full[sa]);
          mbar_arrive(&raw_empty[s]);
        }
        if (++s == kRawStages) {
          s = 0;
          ph ^= 1u;
        }
        if (++sa == C::kAStages) {
          sa = 0;
          pha ^= 1u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// host side: tensor maps and launches
// ---------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// rows x cols matrix, row-major; box = box_rows x box_cols elements
bool make_map(CUtensorMap *m, CUtensorMapDataType dt, size_t elem, const void *base, uint64_t rows, uint64_t cols,
              uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NMAT>
cudaError_t launch(const GemmArgs &a, const TmaMaps &maps, int num_sms, cudaStream_t s) {
  using C = Cfg<NMAT>;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<NMAT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int grid = std::max(1, std::min(num_sms, a.max_items));
  grouped_gemm_kernel<NMAT><<<grid, kThreads, C::kSmem, s>>>(a, maps);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm_gate_up(const GemmArgs &a, int num_sms, cudaStream_t s) {
  if (a.max_items <= 0) return cudaSuccess;
  TmaMaps maps;
  const int H = a.H;
  bool ok = make_map(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.packed,
                     static_cast<uint64_t>(a.E) * 3 * a.I, H / 8, kTileM, 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  ok = ok && make_map(&maps.w_sh, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.sh_packed,
                      static_cast<uint64_t>(3) * a.Is, H / 8, kTileM, 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  ok = ok && make_map(&maps.b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.xt, static_cast<uint64_t>(a.xt_rows), H,
                      kBRows, kTileK, CU_TENSOR_MAP_SWIZZLE_128B);
  maps.b_sh = maps.b;
  if (!ok) return cudaErrorInvalidValue;
  return launch<2>(a, maps, num_sms, s);
}

cudaError_t launch_gemm_down(const GemmArgs &a, int num_sms, cudaStream_t s) {
  if (a.max_items <= 0) return cudaSuccess;
  TmaMaps maps;
  const int H = a.H;
  bool ok = make_map(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.packed,
                     static_cast<uint64_t>(a.E) * 3 * H, a.I / 8, kTileM, 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  ok = ok && make_map(&maps.w_sh, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.sh_packed,
                      static_cast<uint64_t>(3) * H, a.Is / 8, kTileM, 8, CU_TENSOR_MAP_SWIZZLE_NONE);
  ok = ok && make_map(&maps.b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.h, static_cast<uint64_t>(a.h_rows), a.I,
                      kBRows, kTileK, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.b_sh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.h + a.h_shared_off,
                      static_cast<uint64_t>(a.hs_rows), a.Is, kBRows, kTileK, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  return launch<1>(a, maps, num_sms, s);
}

}  // namespace moe
