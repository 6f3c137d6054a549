// gemm_down.cu -- down projection of the grouped expert GEMM on the
// 5th-generation tensor cores: Y = w_routing * (h W_down^T), per routed row.
//
// Same scheme as the gate/up GEMM: the 4-bit weights are rebuilt one tile at a
// time on chip and the products accumulate in fp32 ("Perplexity open sources
// Lily...", section "Measurements"; aioga.com record, article body paragraph
// 4). The weights are the MMA's M side (128 rows of W_down) and the expert's
// rows of h the N side (up to 128), so uneven expert groups, some with a
// handful of tokens (aioga.com record, paragraph 3), only shrink N.
//
//   TMA: packed int4 rows (128-byte swizzle), fp16 h rows (32-row boxes)
//   8 dequant warps (two per TMEM lane quarter, four words of each K-block
//        row each): q*scale + bias -> fp16 -> TMEM (tcgen05.st), the MMA's A
//   1 thread: tcgen05.mma (A from TMEM, B = h rows from shared memory)
//   8 epilogue warps (two per lane quarter, alternate 16-row groups):
//        tcgen05.ld, scale by the row's routing weight, fp16 rows of Y staged
//        in shared memory and written out in 16-byte pieces.
//
// TMEM: two 128-column accumulator stages (a tile's epilogue overlaps the next
// tile's main loop) and four weight stages of two K-blocks (64 columns) each,
// so every wait and commit covers 128 elements of K.
// Warp roles (640 threads): 0 weight TMA, 1 activation TMA, 2 MMA issue,
// 4-11 epilogue, 12-19 dequantisation (warp 3 idle, so that every role's warps
// see the tensor-memory lane quarter warp % 4). Every wait is bounded.
#include <algorithm>

#include "gemm_common.cuh"

namespace moe {

namespace {

using namespace sm100;
using namespace gemm;

constexpr int kPkWarp = 0;
constexpr int kBWarp = 1;
constexpr int kMmaWarp = 2;
constexpr int kEpiPerQ = 2;                    // epilogue warps per TMEM lane quarter
constexpr int kDqPerQ = 2;                     // dequantisation warps per lane quarter
constexpr int kEpiWarp0 = 4;
constexpr int kEpiWarps = 4 * kEpiPerQ;
constexpr int kDqWarp0 = kEpiWarp0 + kEpiWarps;
constexpr int kDqWarps = 4 * kDqPerQ;
constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
constexpr int kDqWords = 8 / kDqPerQ;          // words of a K-block row per dequantisation warp
static_assert(kThreads <= 1024, "one CTA");
static_assert(kDqWords == 2 || kDqWords == 4, "a warp takes 8 or 16 bytes of a K-block row");

constexpr int kN = kTileN;                     // activation rows per tile
constexpr int kStageK = 2;                     // K-blocks per activation stage
constexpr int kBStages = 3;
constexpr int kBAtomBytes = kN * 128;          // one K-block of kN activation rows
constexpr int kBStageBytes = kStageK * kBAtomBytes;
constexpr int kSuperK = 4;                     // K-blocks per packed stage
constexpr int kPkStages = 6;
constexpr int kPkStageBytes = kTileM * 128;    // 128 weight rows x 32 words
constexpr int kAKB = 2;                        // K-blocks per TMEM weight stage (= per activation stage)
constexpr int kAStages = 4;                    // TMEM weight stages of two K-blocks (2 x 32 columns) each
static_assert(kAKB == kStageK, "one weight stage per activation stage");
constexpr int kAccStages = 2;
constexpr int kACol0 = kAccStages * kN;
constexpr int kTmemCols = 512;
static_assert(kACol0 + kAStages * kAKB * 32 <= kTmemCols, "TMEM budget");
static_assert(kEpiWarp0 % 4 == 0 && kDqWarp0 % 4 == 0, "warp w of a role reaches TMEM lane quarter w % 4");
constexpr int kStgBytes = kN * 32 * 2;         // per lane quarter: kN rows x 32 columns fp16

constexpr int kOffPk = 0;
constexpr int kOffB = kOffPk + kPkStages * kPkStageBytes;
constexpr int kOffStg = kOffB + kBStages * kBStageBytes;
constexpr int kOffBar = kOffStg + 4 * kStgBytes;
constexpr int kNumBars = 2 * kPkStages + 2 * kBStages + 2 * kAStages + 2 * kAccStages + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmem = kOffMisc + 64 + 1024;  // + slack for aligning the base
static_assert(kOffB % 1024 == 0 && kBAtomBytes % 1024 == 0, "128-byte swizzle tiles need 1024-byte alignment");
static_assert(kSmem <= 227 * 1024, "shared memory budget");

// Scale/bias row of W_down row mblk*128 + r of item wi.
__device__ __forceinline__ SbRow sb_row_dn(const GemmArgs &a, const WorkItem &wi, int r) {
  const bool sh = wi.group == a.E;
  const int Ig = sh ? a.Is : a.I;
  const int H = a.H;
  const size_t off = (sh ? 0 : static_cast<size_t>(wi.group) * 3 * a.I * H / kGroup) +
                     static_cast<size_t>(2) * Ig * H / kGroup + static_cast<size_t>(wi.mblk * kTileM + r) * (Ig / kGroup);
  return SbRow{(sh ? a.w.sh_scales : a.w.scales) + off, (sh ? a.w.sh_biases : a.w.biases) + off, Ig};
}

__global__ void __launch_bounds__(kThreads, 1) gemm_down_kernel(const GemmArgs a,
                                                                const __grid_constant__ TmaMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sPk = smem + kOffPk;
  uint8_t *sB = smem + kOffB;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
  uint64_t *pk_full = bars;
  uint64_t *pk_empty = pk_full + kPkStages;
  uint64_t *b_full = pk_empty + kPkStages;
  uint64_t *b_empty = b_full + kBStages;
  uint64_t *a_full = b_empty + kBStages;
  uint64_t *a_empty = a_full + kAStages;
  uint64_t *acc_full = a_empty + kAStages;
  uint64_t *acc_empty = acc_full + kAccStages;
  uint64_t *mma_done = acc_empty + kAccStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kOffMisc);
  volatile int *abort = reinterpret_cast<volatile int *>(smem + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPkStages; ++s) {
      mbar_init(&pk_full[s], 1);
      mbar_init(&pk_empty[s], kDqWarps);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int s = 0; s < kAStages; ++s) {
      mbar_init(&a_full[s], kDqWarps);
      mbar_init(&a_empty[s], 1);
    }
    for (int s = 0; s < kAccStages; ++s) {
      mbar_init(&acc_full[s], 1);
      mbar_init(&acc_empty[s], kEpiWarps);
    }
    mbar_init(mma_done, 1);
    *abort = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kPkWarp && lane == 0) {
    tma_prefetch_desc(&maps.w);
    tma_prefetch_desc(&maps.w_sh);
  }
  if (warp == kBWarp && lane == 0) {
    tma_prefetch_desc(&maps.b);
    tma_prefetch_desc(&maps.b_sh);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the prologue above touched no global memory; the routing results, the
  // activation rows and the work list come from the kernels before this one
  pdl_wait();
  pdl_trigger();

  const int nitems = min(*a.item_count, a.max_items);
  const int H = a.H;

  if (warp == kPkWarp) {
    // ------------------------------------------------ producer: packed weights
    if (lane == 0) {
      TmaRing<kPkStages> ring;
      bool ok = true;
      for (int it = next_item(a, blockIdx.x, nitems, true, true); it < nitems && ok;
           it = next_item(a, it + gridDim.x, nitems, true, true)) {
        const WorkItem wi = a.items[it];
        const bool sh = wi.group == a.E;
        const int K = sh ? a.Is : a.I;
        // rows of K/8 words: an expert's block is 3H such rows, W_down its last H
        const int wrow = (sh ? 0 : wi.group * 3 * H) + 2 * H + wi.mblk * kTileM;
        const CUtensorMap *mw = sh ? &maps.w_sh : &maps.w;
        for (int sb = 0; sb < (K / kTileK + kSuperK - 1) / kSuperK; ++sb, ring.advance()) {
          if (!ring.claim(pk_empty, pk_full, kPkStageBytes, abort, a.status, 100)) {
            ok = false;
            break;
          }
          tma_load_2d(sPk + ring.s * kPkStageBytes, mw, &pk_full[ring.s], sb * kSuperK * 8, wrow);
        }
      }
      if (!ok) ring.drain(pk_full);
    }
  } else if (warp == kBWarp) {
    // ------------------------------------------------ producer: activation rows
    if (lane == 0) {
      TmaRing<kBStages> ring;
      bool ok = true;
      for (int it = next_item(a, blockIdx.x, nitems, true, false); it < nitems && ok;
           it = next_item(a, it + gridDim.x, nitems, true, false)) {
        const WorkItem wi = a.items[it];
        const bool sh = wi.group == a.E;
        const int K = sh ? a.Is : a.I;
        const CUtensorMap *mb = sh ? &maps.b_sh : &maps.b;
        const int brow0 = sh ? wi.row0 - a.R : wi.row0;
        const int nb = (wi.nrows + kBRows - 1) / kBRows;
        for (int ks = 0; ks < K / (kTileK * kStageK); ++ks, ring.advance()) {
          if (!ring.claim(b_empty, b_full, kStageK * nb * kBRows * 128, abort, a.status, 101)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int kh = 0; kh < kStageK; ++kh)
            for (int j = 0; j < nb; ++j)
              tma_load_2d(sB + ring.s * kBStageBytes + kh * kBAtomBytes + j * kBRows * 128, mb, &b_full[ring.s],
                          (ks * kStageK + kh) * kTileK, brow0 + j * kBRows);
        }
      }
      if (!ok) ring.drain(b_full);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------ MMA issuer (whole warp, one elected lane issues)
    RingCursor<kBStages> bs;
    RingCursor<kAStages> as;
    bool ok = true;
    int li = 0;
    for (int it = next_item(a, blockIdx.x, nitems, true, false); it < nitems && ok;
         it = next_item(a, it + gridDim.x, nitems, true, false), ++li) {
      const WorkItem wi = a.items[it];
      const int K = wi.group == a.E ? a.Is : a.I;
      const int st = li % kAccStages;
      const uint32_t acc_ph = (li / kAccStages) & 1;
      if (!warp_wait(&acc_empty[st], acc_ph ^ 1u, abort, a.status, 110)) break;
      tc_fence_after();
      const uint32_t idesc = idesc_f16_f32(kTileM, (wi.nrows + 15) & ~15);
      const uint32_t d = tmem_base + st * kN;
      for (int ks = 0; ks < K / (kTileK * kStageK); ++ks) {
        if (!warp_wait(&b_full[bs.s], bs.ph, abort, a.status, 112)) {
          ok = false;
          break;
        }
        const uint32_t b_addr = smem_u32(sB + bs.s * kBStageBytes);
        if (!warp_wait(&a_full[as.s], as.ph, abort, a.status, 111)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kh = 0; kh < kStageK; ++kh) {
            const uint32_t a_col = tmem_base + kACol0 + as.s * (kAKB * 32) + kh * 32;
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk)
              tc_mma_f16_ts(d, a_col + kk * 8, smem_desc_sw128(b_addr + kh * kBAtomBytes + kk * 32), idesc,
                            (ks | kh | kk) != 0 ? 1u : 0u);
          }
          tc_commit(&a_empty[as.s]);
          tc_commit(&b_empty[bs.s]);
        }
        __syncwarp();
        as.advance();
        bs.advance();
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
  } else if (warp < kEpiWarp0) {
    // warp 3: no role
  } else if (warp < kDqWarp0) {
    // ------------------------------------------------ epilogue
    // The kEpiPerQ warps of lane quarter q take the tile's 16-row groups in
    // turn: warp `sub` the groups g with g % kEpiPerQ == sub.
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int sub = (warp - kEpiWarp0) >> 2;
    // the quarter's 32 output columns of the tile's rows, staged as [row][32]
    // fp16; the quarter's warps write disjoint rows
    __half *stg = reinterpret_cast<__half *>(smem + kOffStg + q * kStgBytes);
    int li = 0;
    for (int it = next_item(a, blockIdx.x, nitems, true, false); it < nitems;
         it = next_item(a, it + gridDim.x, nitems, true, false), ++li) {
      const WorkItem wi = a.items[it];
      const int st = li % kAccStages;
      const uint32_t acc_ph = (li / kAccStages) & 1;
      const int ng = (wi.nrows + 15) >> 4;  // 16-row groups of the tile
      // routing weight of each row, lane l of chunk c holding row 32c + l,
      // loaded before the accumulators are ready
      static_assert(kN / 32 == 4, "four 32-row chunks per tile");
      float w_l[kN / 32];
#pragma unroll
      for (int c = 0; c < kN / 32; ++c) {
        const int jl = 32 * c + lane;
        w_l[c] = jl < wi.nrows ? a.row_w[wi.row0 + jl] : 0.f;
      }
      if (!warp_wait(&acc_full[st], acc_ph, abort, a.status, 120)) break;
      tc_fence_after();
      if (sub >= ng) {  // no group for this warp: the accumulators are not read
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[st]);
      }
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + st * kN;
      __half *obase = a.y + static_cast<int64_t>(wi.row0) * H + wi.mblk * kTileM + q * 32;
      for (int g = sub; g < ng; g += kEpiPerQ) {
        const int c16 = 16 * g;
        const int c = g >> 1;
        const float wl = c == 0 ? w_l[0] : c == 1 ? w_l[1] : c == 2 ? w_l[2] : w_l[3];
        uint32_t r0[16];
        tmem_ld_32x32b_x16(tq + c16, r0);
        tmem_ld_wait();
        if (g + kEpiPerQ >= ng) {  // this warp's last read of the accumulators
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[st]);
        }
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const float f = __shfl_sync(0xffffffffu, wl, 16 * (g & 1) + jj);
          stg[(c16 + jj) * 32 + lane] = __float2half_rn(f * __uint_as_float(r0[jj]));
        }
      }
      __syncwarp();
      // write out this warp's rows: 4 chunks of 16 bytes per row, 8 rows per warp instruction
      for (int g = sub; g < ng; g += kEpiPerQ) {
        const int jend = min(16 * g + 16, wi.nrows);
        for (int j = 16 * g + (lane >> 2); j < jend; j += 8) {
          const int c = lane & 3;
          const uint4 v = *reinterpret_cast<const uint4 *>(stg + j * 32 + c * 8);
          *reinterpret_cast<uint4 *>(obase + static_cast<int64_t>(j) * H + c * 8) = v;
        }
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------ dequantisation
    // Warp w owns TMEM lane quarter w % 4, i.e. weight rows 32*(w%4) + lane; the
    // kDqPerQ warps of a quarter take words kDqWords*pw .. kDqWords*pw +
    // kDqWords - 1 (pw = dw / 4) of each row and K-block. The fp16 values go
    // straight to TMEM (tcgen05.st), where the MMA reads its A operand.
    const int dw = warp - kDqWarp0;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int pw = dw >> 2;
    RingCursor<kPkStages> pk;
    RingCursor<kAStages> as;
    bool ok = true;
    static_assert(kSuperK == 4, "the scale/bias stream loads four K-blocks at a time");
    SbStream sb;
    const int first = next_item(a, blockIdx.x, nitems, true, false);
    if (first < nitems) sb.start(sb_row_dn(a, a.items[first], r));
    for (int it = first; it < nitems && ok; it = next_item(a, it + gridDim.x, nitems, true, false)) {
      const int nkb = sb.row.K / kTileK;
      for (int kb = 0; kb < nkb; kb += kAKB) {  // two K-blocks per TMEM stage
        const int j = kb % kSuperK;             // 0 or 2 within the packed stage
        if (j == 0)
          sb.step(kb, nkb, [&](SbRow &nr) {
            const int nx = next_item(a, it + gridDim.x, nitems, true, false);
            if (nx >= nitems) return false;
            nr = sb_row_dn(a, a.items[nx], r);
            return true;
          });
        const __half2 s2a = sb.scale(j), b2a = sb.bias(j), s2b = sb.scale(j + 1), b2b = sb.bias(j + 1);
        if (j == 0 && !warp_wait(&pk_full[pk.s], pk.ph, abort, a.status, 130)) {
          ok = false;
          break;
        }
        // row r of the packed stage: 128 bytes = 4 K-blocks of 8 words, in
        // 16-byte chunks placed at chunk ^ (r & 7) by the TMA's 128-byte swizzle
        const uint8_t *prow = sPk + pk.s * kPkStageBytes + r * 128;
        // this warp's words of K-block j + kk: 4 kDqWords bytes at byte
        // 4 kDqWords pw of the block's 32, i.e. in chunk 2 (j + kk) + byte / 16
        constexpr int kBytes = 4 * kDqWords;
        const int boff = kBytes * pw;
        uint32_t v[2][kDqWords];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint8_t *src = prow + (((2 * (j + kk) + (boff >> 4)) ^ (r & 7)) << 4) + (boff & 15);
          if constexpr (kDqWords == 4) {
            const uint4 t = *reinterpret_cast<const uint4 *>(src);
            v[kk][0] = t.x, v[kk][1] = t.y, v[kk][2] = t.z, v[kk][3] = t.w;
          } else {
            const uint2 t = *reinterpret_cast<const uint2 *>(src);
            v[kk][0] = t.x, v[kk][1] = t.y;
          }
        }
        if (j + kAKB == kSuperK || kb + kAKB >= nkb) {  // words in registers: release the packed stage
          __syncwarp();
          if (lane == 0) mbar_arrive(&pk_empty[pk.s]);
          pk.advance();
        }
        // each pair of words fills 8 columns; a store overlaps the next pair's
        // arithmetic, the first pair is computed before the stage is known
        // free; one wait
        const uint32_t ta =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kACol0 + as.s * (kAKB * 32) + 4 * kDqWords * pw;
        uint32_t d8[8];
        dequant2(v[0][0], v[0][1], s2a, b2a, d8);
        if (!warp_wait(&a_empty[as.s], as.ph ^ 1u, abort, a.status, 131)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int p = 0; p < kDqWords / 2; ++p) {
            if (kk | p) dequant2(v[kk][2 * p], v[kk][2 * p + 1], kk ? s2b : s2a, kk ? b2b : b2a, d8);
            tmem_st_32x32b_x8(ta + kk * 32 + 8 * p, d8);
          }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[as.s]);
        as.advance();
      }
      sb.end_item();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_down(const GemmArgs &a, int num_sms, cudaStream_t s, bool pdl) {
  if (a.max_items <= 0) return cudaSuccess;
  TmaMaps maps;
  const int H = a.H;
  bool ok = make_map(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.packed, static_cast<uint64_t>(a.E) * 3 * H,
                     a.I / 8, kTileM, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.w_sh, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.sh_packed, static_cast<uint64_t>(3) * H,
                      a.Is / 8, kTileM, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.h, static_cast<uint64_t>(a.h_rows), a.I, kBRows,
                      kTileK, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.b_sh, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.h + a.h_shared_off,
                      static_cast<uint64_t>(a.hs_rows), a.Is, kBRows, kTileK, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e = ensure_smem_limit(gemm_down_kernel, kSmem, smem_set);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, std::min(num_sms, a.max_items));
  return launch_k(gemm_down_kernel, dim3(grid), dim3(kThreads), kSmem, s, pdl, a, maps);
}

}  // namespace moe
