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

constexpr int kThreads = 480;          // 15 warps
constexpr int kPkWarp = 0;             // TMA producer of packed weights
constexpr int kBWarp = 1;              // TMA producer of activation rows
constexpr int kMmaWarp = 2;            // MMA issuer
constexpr int kEpiWarp0 = 3;           // warps 3..6: epilogue
constexpr int kDqWarp0 = 7;            // warps 7..14: dequantisation
constexpr int kDqWarps = 8;
constexpr int kStageK = 2;             // 64-wide K-blocks per activation stage
constexpr int kBStages = 3;            // activation ring (smem)
constexpr int kBRows = 32;             // TMA box height of activation rows
constexpr int kBAtomBytes = kTileN * 128;          // 128 rows x 64 fp16
constexpr int kBStageBytes = kStageK * kBAtomBytes;
constexpr int kSuperK = 4;             // K-blocks per packed stage (128-byte rows of words)
constexpr int kPkTileBytes = kTileM * 128;         // 128 rows x 32 words
constexpr int kAccCols = kTileN;       // fp32 accumulator columns per matrix
constexpr int kAColsPerMat = 32;       // TMEM columns of one matrix in one A stage (one 64-wide K-block)

template <int NMAT>
struct Cfg {
  static constexpr int kPkStages = NMAT == 2 ? 3 : 4;
  static constexpr int kAccStages = NMAT == 2 ? 1 : 2;  // TMEM: accumulators then A stages
  static constexpr int kAStages = NMAT == 2 ? 4 : 8;    // dequantised weights (TMEM), one K-block each
  static constexpr int kACol0 = kAccStages * NMAT * kAccCols;
  static constexpr int kTmemCols = 512;
  static_assert(kACol0 + kAStages * NMAT * kAColsPerMat <= kTmemCols, "TMEM budget");
  static constexpr int kOffPk = 0;
  static constexpr int kOffB = kOffPk + kPkStages * NMAT * kPkTileBytes;
  static constexpr int kOffStage = kOffB + kBStages * kBStageBytes;  // epilogue staging, 8 KB per warp
  static constexpr int kStageBytes = kTileN * 32 * 2;
  static constexpr int kOffBar = kOffStage + 4 * kStageBytes;
  static constexpr int kNumBars = 2 * kPkStages + 2 * kBStages + 2 * kAStages + 2 * kAccStages + 1;
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

// Wait (bounded, ignoring the abort flag) for the copies of the stages this
// thread issued, before the CTA may exit.
template <int N>
__device__ __forceinline__ void drain_stages(uint64_t *full, uint32_t issued, uint32_t issued_ph) {
  for (int t = 0; t < N; ++t) {
    if (!(issued >> t & 1u)) continue;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(&full[t], issued_ph >> t & 1u) && global_ns() - t0 < kWaitBudgetNs) {
    }
  }
}

// 2^e as a float for |e| <= 126, built from its exponent bits
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

template <int NMAT>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const GemmArgs a,
                                                                    const __grid_constant__ TmaMaps maps) {
  using C = Cfg<NMAT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sPk = smem + C::kOffPk;
  uint8_t *sB = smem + C::kOffB;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kOffBar);
  uint64_t *pk_full = bars;
  uint64_t *pk_empty = pk_full + C::kPkStages;
  uint64_t *b_full = pk_empty + C::kPkStages;
  uint64_t *b_empty = b_full + kBStages;
  uint64_t *a_full = b_empty + kBStages;
  uint64_t *a_empty = a_full + C::kAStages;
  uint64_t *acc_full = a_empty + C::kAStages;
  uint64_t *acc_empty = acc_full + C::kAccStages;
  uint64_t *mma_done = acc_empty + C::kAccStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::kOffMisc);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool gate_up = NMAT == 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kPkStages; ++s) {
      mbar_init(&pk_full[s], 1);
      mbar_init(&pk_empty[s], kDqWarps);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < C::kAStages; ++s) {
      mbar_init(&a_full[s], kDqWarps);
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
  if (warp == kPkWarp && lane == 0) {
    tma_prefetch_desc(&maps.w);
    tma_prefetch_desc(&maps.w_sh);
  }
  if (warp == kBWarp && lane == 0) {
    tma_prefetch_desc(&maps.b);
    if (!gate_up) tma_prefetch_desc(&maps.b_sh);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int nitems = min(*a.item_count, a.max_items);
  const int H = a.H;

  if (warp == kPkWarp) {
    // ------------------------------------------------ producer: packed weights
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_ph = 0;
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
          wrow[NMAT - 1] = base + Ig + wi.mblk * kTileM;
        } else {
          K = Ig;
          wrow[0] = (sh ? 0 : wi.group * 3 * H) + 2 * H + wi.mblk * kTileM;
        }
        const CUtensorMap *mw = sh ? &maps.w_sh : &maps.w;
        const int nsb = (K / kTileK + kSuperK - 1) / kSuperK;
        for (int sb = 0; sb < nsb; ++sb) {
          if (!mbar_wait(&pk_empty[s], ph ^ 1u, abort, a.status, 100)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&pk_full[s], NMAT * kPkTileBytes);
          issued |= 1u << s;
          issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
#pragma unroll
          for (int m = 0; m < NMAT; ++m)
            tma_load_2d(sPk + (s * NMAT + m) * kPkTileBytes, mw, &pk_full[s], sb * kSuperK * 8, wrow[m]);
          if (++s == C::kPkStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) drain_stages<C::kPkStages>(pk_full, issued, issued_ph);
    }
  } else if (warp == kBWarp) {
    // ------------------------------------------------ producer: activation rows
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_ph = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
        const WorkItem wi = a.items[it];
        const bool sh = wi.group == a.E;
        const int K = gate_up ? H : (sh ? a.Is : a.I);
        const CUtensorMap *mb = (!gate_up && sh) ? &maps.b_sh : &maps.b;
        const int brow0 = (!gate_up && sh) ? wi.row0 - a.R : wi.row0;
        const int nb = (wi.nrows + kBRows - 1) / kBRows;
        for (int ks = 0; ks < K / (kTileK * kStageK); ++ks) {
          if (!mbar_wait(&b_empty[s], ph ^ 1u, abort, a.status, 101)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&b_full[s], kStageK * nb * kBRows * 128);
          issued |= 1u << s;
          issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
#pragma unroll
          for (int kh = 0; kh < kStageK; ++kh)
            for (int j = 0; j < nb; ++j)
              tma_load_2d(sB + s * kBStageBytes + kh * kBAtomBytes + j * kBRows * 128, mb, &b_full[s],
                          (ks * kStageK + kh) * kTileK, brow0 + j * kBRows);
          if (++s == kBStages) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) drain_stages<kBStages>(b_full, issued, issued_ph);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer (whole warp, one elected lane issues)
    int sb = 0, sa = 0;
    uint32_t phb = 0, pha = 0;
    bool ok = true;
    int li = 0;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
      const WorkItem wi = a.items[it];
      const bool sh = wi.group == a.E;
      const int K = gate_up ? H : (sh ? a.Is : a.I);
      const int st = li % C::kAccStages;
      const uint32_t acc_ph = (li / C::kAccStages) & 1;
      if (!warp_wait(&acc_empty[st], acc_ph ^ 1u, abort, a.status, 110)) break;
      tc_fence_after();
      const int n16 = (wi.nrows + 15) & ~15;
      const uint32_t idesc = idesc_f16_f32(kTileM, n16);
      const uint32_t d0 = tmem_base + st * NMAT * kAccCols;
      for (int ks = 0; ks < K / (kTileK * kStageK); ++ks) {
        if (!warp_wait(&b_full[sb], phb, abort, a.status, 112)) {
          ok = false;
          break;
        }
        const uint32_t b_addr = smem_u32(sB + sb * kBStageBytes);
        for (int kh = 0; kh < kStageK; ++kh) {
          if (!warp_wait(&a_full[sa], pha, abort, a.status, 111)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (elect_one()) {
            const uint32_t a_col = tmem_base + C::kACol0 + sa * NMAT * kAColsPerMat;
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(b_addr + kh * kBAtomBytes + kk * 32);
#pragma unroll
              for (int m = 0; m < NMAT; ++m)
                tc_mma_f16_ts(d0 + m * kAccCols, a_col + m * kAColsPerMat + kk * 8, bdesc, idesc,
                              (ks | kh | kk) != 0 ? 1u : 0u);
            }
            tc_commit(&a_empty[sa]);
            if (kh == kStageK - 1) tc_commit(&b_empty[sb]);
          }
          __syncwarp();
          if (++sa == C::kAStages) {
            sa = 0;
            pha ^= 1u;
          }
        }
        if (!ok) break;
        if (++sb == kBStages) {
          sb = 0;
          phb ^= 1u;
        }
      }
      if (ok && elect_one()) tc_commit(&acc_full[st]);
      __syncwarp();
    }
    // all issued MMAs finish before tensor memory is released
    if (elect_one()) tc_commit(mma_done);
    __syncwarp();
    if (lane == 0) {
      const unsigned long long t0 = global_ns();
      while (!mbar_try_wait(mma_done, 0) && global_ns() - t0 < kWaitBudgetNs) {
      }
    }
    __syncwarp();
  } else if (warp < kDqWarp0) {
    // ------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    int li = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
      const WorkItem wi = a.items[it];
      const bool sh = wi.group == a.E;
      const int st = li % C::kAccStages;
      const uint32_t acc_ph = (li / C::kAccStages) & 1;
      if (!warp_wait(&acc_full[st], acc_ph, abort, a.status, 120)) break;
      tc_fence_after();
      const int mrow = wi.mblk * kTileM + q * 32 + lane;  // weight row of this thread
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + st * NMAT * kAccCols;
      // This warp's 32 output columns of the tile's rows: staged in shared memory
      // as [row][32] fp16, then written out as 16-byte chunks. Output row j of
      // the tile starts at obase + j * pitch (elements).
      __half *stg = reinterpret_cast<__half *>(smem + C::kOffStage + (warp - kEpiWarp0) * C::kStageBytes);
      __half *obase;
      int pitch;
      int scol;  // this lane's column inside the 32-wide slab
      if (gate_up) {
        pitch = sh ? a.Is : a.I;
        obase = (sh ? a.h + a.h_shared_off + static_cast<int64_t>(wi.row0 - a.R) * a.Is
                    : a.h + static_cast<int64_t>(wi.row0) * a.I) +
                wi.mblk * kTileM + q * 32;
        scol = (lane & ~7) + kperm_dst(lane & 7);  // K-permuted order of the down GEMM's operand
      } else {
        pitch = H;
        obase = a.y + static_cast<int64_t>(wi.row0) * H + wi.mblk * kTileM + q * 32;
        scol = lane;
      }
      (void)mrow;
      for (int c0 = 0; c0 < wi.nrows; c0 += 32) {
        const bool last = c0 + 32 >= wi.nrows;
        // per-column factor, one column per lane, broadcast by shuffles
        const int jl = c0 + lane;
        float fl = 0.f;
        if (jl < wi.nrows)
          fl = gate_up ? __int_as_float(a.row_exp[wi.row0 + jl]) : a.row_w[wi.row0 + jl];
        if (gate_up) {
          // two 16-column halves keep the live registers down
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t g16[16], u16[16];
            tmem_ld_32x32b_x16(tq + c0 + 16 * hh, g16);
            tmem_ld_32x32b_x16(tq + kAccCols + c0 + 16 * hh, u16);
            tmem_ld_wait();
            if (last && hh == 1) {  // accumulators fully read: the next tile's MMAs may start
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[st]);
            }
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int e = __float_as_int(__shfl_sync(0xffffffffu, fl, 16 * hh + jj));
              // silu(gate) * up with gate = g 2^e, up = u 2^e, result scaled by 2^-2e
              const float gt = __uint_as_float(g16[jj]) * pow2i(e);
              const float sg = __fdividef(gt, 1.0f + __expf(-gt));
              stg[(c0 + 16 * hh + jj) * 32 + scol] = __float2half_rn(sg * pow2i(-e) * __uint_as_float(u16[jj]));
            }
          }
        } else {
          uint32_t r0[32];
          tmem_ld_32x32b_x32(tq + c0, r0);
          tmem_ld_wait();
          if (last) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[st]);
          }
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const float f = __shfl_sync(0xffffffffu, fl, jj);
            stg[(c0 + jj) * 32 + scol] = __float2half_rn(f * __uint_as_float(r0[jj]));
          }
        }
      }
      __syncwarp();
      // write out: 4 chunks of 16 bytes per row, 8 rows per warp instruction
      for (int j = lane >> 2; j < wi.nrows; j += 8) {
        const int c = lane & 3;
        const uint4 v = *reinterpret_cast<const uint4 *>(stg + j * 32 + c * 8);
        *reinterpret_cast<uint4 *>(obase + static_cast<int64_t>(j) * pitch + c * 8) = v;
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------ dequantisation
    // Warp w owns TMEM lane quarter w % 4, i.e. weight rows 32*(w%4) + lane.
    // gate/up: warps 7..10 dequantise the gate rows, 11..14 the up rows, eight
    // words per row and K-block; down: the two warps of a quarter take four
    // words each. Each row's fp16 values go straight to TMEM (tcgen05.st),
    // where the MMA reads its A operand; a row's scale and bias are loaded one
    // K-block ahead.
    const int dw = warp - kDqWarp0;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int m = gate_up ? dw >> 2 : 0;
    const int half = gate_up ? 0 : dw >> 2;  // down: words 4*half .. 4*half+3
    int sp = 0, sa = 0;
    uint32_t php = 0, pha = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
      const WorkItem wi = a.items[it];
      const bool sh = wi.group == a.E;
      const int Ig = sh ? a.Is : a.I;
      const uint16_t *S, *B;
      int K;
      if (gate_up) {
        K = H;
        const size_t off = (sh ? 0 : static_cast<size_t>(wi.group) * 3 * a.I * H / kGroup) +
                           static_cast<size_t>(m * Ig + wi.mblk * kTileM + r) * (H / kGroup);
        S = (sh ? a.w.sh_scales : a.w.scales) + off;
        B = (sh ? a.w.sh_biases : a.w.biases) + off;
      } else {
        K = Ig;
        const size_t off = (sh ? 0 : static_cast<size_t>(wi.group) * 3 * a.I * H / kGroup) +
                           static_cast<size_t>(2) * Ig * H / kGroup +
                           static_cast<size_t>(wi.mblk * kTileM + r) * (Ig / kGroup);
        S = (sh ? a.w.sh_scales : a.w.scales) + off;
        B = (sh ? a.w.sh_biases : a.w.biases) + off;
      }
      const int nkb = K / kTileK;  // one scale/bias group per K-block
      uint16_t s_next = __ldg(S), b_next = __ldg(B);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!warp_wait(&a_empty[sa], pha ^ 1u, abort, a.status, 131)) {
          ok = false;
          break;
        }
        const uint32_t ta =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + C::kACol0 + sa * NMAT * kAColsPerMat + m * kAColsPerMat;
        const __half2 s2 = bf16_to_half2_bcast(s_next), b2 = bf16_to_half2_bcast(b_next);
        if (kb + 1 < nkb) {
          s_next = __ldg(S + kb + 1);
          b_next = __ldg(B + kb + 1);
        }
        const int j = kb % kSuperK;
        if (j == 0 && !warp_wait(&pk_full[sp], php, abort, a.status, 130)) {
          ok = false;
          break;
        }
        // row r of the packed stage: 128 bytes = 4 K-blocks of 8 words, in
        // 16-byte chunks placed at chunk ^ (r & 7) by the TMA's 128-byte swizzle
        const uint8_t *prow = sPk + (sp * NMAT + m) * kPkTileBytes + r * 128;
        if (gate_up) {
          const uint4 v0 = *reinterpret_cast<const uint4 *>(prow + (((2 * j) ^ (r & 7)) << 4));
          const uint4 v1 = *reinterpret_cast<const uint4 *>(prow + (((2 * j + 1) ^ (r & 7)) << 4));
          if (j == kSuperK - 1 || kb == nkb - 1) {  // words in registers: release the packed stage
            __syncwarp();
            if (lane == 0) mbar_arrive(&pk_empty[sp]);
            if (++sp == C::kPkStages) {
              sp = 0;
              php ^= 1u;
            }
          }
          const uint32_t wv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          uint32_t d[32];
#pragma unroll
          for (int cw = 0; cw < 8; ++cw) {
            const uint4 v = dequant_word(wv[cw], s2, b2);
            d[4 * cw + 0] = v.x;
            d[4 * cw + 1] = v.y;
            d[4 * cw + 2] = v.z;
            d[4 * cw + 3] = v.w;
          }
          tmem_st_32x32b_x32(ta, d);
        } else {
          const uint4 v0 = *reinterpret_cast<const uint4 *>(prow + (((2 * j + half) ^ (r & 7)) << 4));
          if (j == kSuperK - 1 || kb == nkb - 1) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&pk_empty[sp]);
            if (++sp == C::kPkStages) {
              sp = 0;
              php ^= 1u;
            }
          }
          const uint32_t wv[4] = {v0.x, v0.y, v0.z, v0.w};
          uint32_t d[16];
#pragma unroll
          for (int cw = 0; cw < 4; ++cw) {
            const uint4 v = dequant_word(wv[cw], s2, b2);
            d[4 * cw + 0] = v.x;
            d[4 * cw + 1] = v.y;
            d[4 * cw + 2] = v.z;
            d[4 * cw + 3] = v.w;
          }
          tmem_st_32x32b_x16(ta + 16 * half, d);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[sa]);
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
                     static_cast<uint64_t>(a.E) * 3 * a.I, H / 8, kTileM, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.w_sh, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.sh_packed,
                      static_cast<uint64_t>(3) * a.Is, H / 8, kTileM, 32, CU_TENSOR_MAP_SWIZZLE_128B);
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
                     static_cast<uint64_t>(a.E) * 3 * H, a.I / 8, kTileM, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.w_sh, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.sh_packed,
                      static_cast<uint64_t>(3) * H, a.Is / 8, kTileM, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.h, static_cast<uint64_t>(a.h_rows), a.I,
                      kBRows, kTileK, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.b_sh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.h + a.h_shared_off,
                      static_cast<uint64_t>(a.hs_rows), a.Is, kBRows, kTileK, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  return launch<1>(a, maps, num_sms, s);
}

}  // namespace moe
