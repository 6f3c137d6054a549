// gemm_gu.cu -- gate/up projection of the grouped expert GEMM, with the SwiGLU
// epilogue, on the 5th-generation tensor cores.
//
// The pages' engine rebuilds the 4-bit weights one tile at a time inside the
// grouped GEMM and accumulates in fp32, so the expanded weights never reach
// memory ("Perplexity open sources Lily...", section "Measurements"; aioga.com
// record, article body paragraph 4). The expert computes
// h = silu(x W_gate^T) * (x W_up^T), then h W_down^T (the gated feed-forward
// of each expert, same pages).
//
// Tile: 128 output rows of h for up to 128 activation rows (tokens): the same
// 128 rows of W_gate and of W_up are dequantised into two A operands that
// share one activation tile, so each activation byte brought on chip feeds 256
// weight rows. A single accumulator stage holds gate and up (2 x 128 TMEM
// columns); two weight stages of two K-blocks each (2 x 128 columns) fill the
// rest, so every wait and commit covers 128 elements of K.
//
//   TMA: packed int4 rows (a gate box and an up box, 128-byte swizzle) and
//        fp16 activation rows (32-row boxes)
//   8 dequant warps (one per TMEM lane quarter and matrix): q*scale + bias
//        -> fp16 -> TMEM (tcgen05.st)
//   1 thread: tcgen05.mma, two per 16-wide K step (gate, up), B shared
//   8 epilogue warps (two per lane quarter, alternate 16-token groups):
//        tcgen05.ld of gate and up for the same rows (same TMEM lanes),
//        h = silu(g) * u, fp16 in the K order the down GEMM's operand uses,
//        staged in shared memory and written out in 16-byte pieces.
//
// Warp roles (128-row tiles, 640 threads): 0 weight TMA, 1 activation TMA,
// 2 MMA issue, 4-11 epilogue, 12-19 dequantisation (warp 3 idle, so that every
// role's warps see the tensor-memory lane quarter warp % 4); 32-row tiles
// (small expert groups): 4-7 epilogue, 8-23 dequantisation. The single
// accumulator stage is the large tile's serial step: two epilogue warps per
// lane quarter empty it sooner than one; more epilogue or dequantisation
// warps only took issue slots from each other (measured). Every wait is
// bounded.
#include <algorithm>

#include "gemm_common.cuh"

namespace moe {

namespace {

using namespace sm100;
using namespace gemm;

constexpr int kPkWarp = 0;
constexpr int kBWarp = 1;
constexpr int kMmaWarp = 2;
constexpr int kEpiWarp0 = 4;

constexpr int kRows = kGuTileM;                // output rows per tile (rows of each of W_gate, W_up)
constexpr int kStageK = 2;                     // K-blocks per activation stage
constexpr int kSuperK = 4;                     // K-blocks per packed stage
constexpr int kPkTileBytes = kRows * 128;      // one matrix: kRows rows x 32 words
constexpr int kPkStageBytes = 2 * kPkTileBytes;
constexpr int kAKB = 2;                        // K-blocks per TMEM weight stage (= per activation stage)
constexpr int kAStageCols = kAKB * 2 * 32;     // [K-block 0: gate, up | K-block 1: gate, up]
static_assert(kAKB == kStageK, "one weight stage per activation stage");
constexpr int kTmemCols = 512;
static_assert(kRows == 128, "one TMEM lane per weight row");

// Tile shapes. N = 128 activation rows per tile for large groups; N = 32 when
// the groups are small (a few dozen tokens per expert): the single
// accumulator stage then takes 64 TMEM columns instead of 256, which leaves
// room for a third weight stage, so the dequantisation runs two stages ahead
// of the MMA instead of one; the smaller activation stages allow deeper
// rings, and with little epilogue work the warps go to dequantisation
// (16 dequantisation and 4 epilogue warps instead of 8 and 8: measured
// faster at T = 512).
template <int N>
struct GuTile {
  static constexpr int kEpiPerQ = N == 128 ? 2 : 1;          // epilogue warps per TMEM lane quarter
  static constexpr int kDqPerQ = N == 128 ? 1 : 2;           // dequantisation warps per lane quarter and matrix
  static constexpr int kEpiWarps = 4 * kEpiPerQ;
  static constexpr int kDqWarp0 = kEpiWarp0 + kEpiWarps;
  static constexpr int kDqWarps = 8 * kDqPerQ;
  static constexpr int kThreads = (kDqWarp0 + kDqWarps) * 32;
  static_assert(kThreads <= 1024, "one CTA");
  static_assert(kDqPerQ == 1 || kDqPerQ == 2, "a dequantisation warp takes a whole or half a K-block row");
  static_assert(kEpiWarp0 % 4 == 0 && kDqWarp0 % 4 == 0, "warp w of a role reaches TMEM lane quarter w % 4");
  static constexpr int kN = N;                               // activation rows per tile
  static constexpr int kBStages = N == 128 ? 3 : 6;
  static constexpr int kPkStages = N == 128 ? 3 : 4;
  static constexpr int kAStages = N == 128 ? 2 : 3;          // TMEM weight stages
  static constexpr int kBAtomBytes = kN * 128;               // one K-block of kN activation rows
  static constexpr int kBStageBytes = kStageK * kBAtomBytes;
  static constexpr int kAccCols = kN;                        // fp32 accumulator columns per matrix
  static constexpr int kACol0 = 2 * kAccCols;                // one accumulator stage: gate, then up
  static constexpr int kStgBytes = kN * 32 * 2;              // per lane quarter: kN tokens x 32 columns fp16
  static constexpr int kOffPk = 0;
  static constexpr int kOffB = kOffPk + kPkStages * kPkStageBytes;
  static constexpr int kOffStg = kOffB + kBStages * kBStageBytes;
  static constexpr int kOffBar = kOffStg + 4 * kStgBytes;
  static constexpr int kNumBars = 2 * kPkStages + 2 * kBStages + 2 * kAStages + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 64 + 1024;        // + slack for aligning the base
  static_assert(kN % 32 == 0 && kN <= 128, "whole 32-row activation boxes");
  static_assert(kACol0 + kAStages * kAStageCols <= kTmemCols, "TMEM budget");
  static_assert(kOffB % 1024 == 0 && kBAtomBytes % 1024 == 0, "128-byte swizzle tiles need 1024-byte alignment");
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

// Scale/bias row of row mblk*128 + r of W_gate (m = 0) or W_up (m = 1) of item wi.
__device__ __forceinline__ SbRow sb_row_gu(const GemmArgs &a, const WorkItem &wi, int m, int r) {
  const bool sh = wi.group == a.E;
  const int Ig = sh ? a.Is : a.I;
  const int H = a.H;
  const size_t off = (sh ? 0 : static_cast<size_t>(wi.group) * 3 * a.I * H / kGroup) +
                     static_cast<size_t>(m * Ig + wi.mblk * kRows + r) * (H / kGroup);
  return SbRow{(sh ? a.w.sh_scales : a.w.scales) + off, (sh ? a.w.sh_biases : a.w.biases) + off, H};
}

template <int N>
__global__ void __launch_bounds__(GuTile<N>::kThreads, 1) gemm_gate_up_kernel(const GemmArgs a,
                                                                              const __grid_constant__ TmaMaps maps) {
  using C = GuTile<N>;
  constexpr int kEpiPerQ = C::kEpiPerQ, kDqPerQ = C::kDqPerQ, kEpiWarps = C::kEpiWarps;
  constexpr int kDqWarp0 = C::kDqWarp0, kDqWarps = C::kDqWarps;
  constexpr int kN = C::kN, kBStages = C::kBStages, kPkStages = C::kPkStages, kAStages = C::kAStages;
  constexpr int kBAtomBytes = C::kBAtomBytes, kBStageBytes = C::kBStageBytes, kAccCols = C::kAccCols;
  constexpr int kACol0 = C::kACol0, kStgBytes = C::kStgBytes;
  constexpr int kOffPk = C::kOffPk, kOffB = C::kOffB, kOffStg = C::kOffStg, kOffBar = C::kOffBar;
  constexpr int kOffMisc = C::kOffMisc;
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
  uint64_t *acc_empty = acc_full + 1;
  uint64_t *mma_done = acc_empty + 1;
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
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kEpiWarps);
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
  if (warp == kBWarp && lane == 0) tma_prefetch_desc(&maps.b);
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
  const int nkb = H / kTileK;

  if (warp == kPkWarp) {
    // ------------------------------------------------ producer: packed weights
    if (lane == 0) {
      TmaRing<kPkStages> ring;
      bool ok = true;
      for (int it = next_item(a, blockIdx.x, nitems, false, true); it < nitems && ok;
           it = next_item(a, it + gridDim.x, nitems, false, true)) {
        const WorkItem wi = a.items[it];
        const bool sh = wi.group == a.E;
        const int base = sh ? 0 : wi.group * 3 * a.I;  // rows of H/8 words
        const int row_g = base + wi.mblk * kRows;
        const int row_u = base + (sh ? a.Is : a.I) + wi.mblk * kRows;
        const CUtensorMap *mw = sh ? &maps.w_sh : &maps.w;
        for (int sb = 0; sb < (nkb + kSuperK - 1) / kSuperK; ++sb, ring.advance()) {
          if (!ring.claim(pk_empty, pk_full, kPkStageBytes, abort, a.status, 200)) {
            ok = false;
            break;
          }
          uint8_t *dst = sPk + ring.s * kPkStageBytes;
          tma_load_2d(dst, mw, &pk_full[ring.s], sb * kSuperK * 8, row_g);
          tma_load_2d(dst + kPkTileBytes, mw, &pk_full[ring.s], sb * kSuperK * 8, row_u);
        }
      }
      if (!ok) ring.drain(pk_full);
    }
  } else if (warp == kBWarp) {
    // ------------------------------------------------ producer: activation rows
    if (lane == 0) {
      TmaRing<kBStages> ring;
      bool ok = true;
      for (int it = next_item(a, blockIdx.x, nitems, false, false); it < nitems && ok;
           it = next_item(a, it + gridDim.x, nitems, false, false)) {
        const WorkItem wi = a.items[it];
        const int nb = (wi.nrows + kBRows - 1) / kBRows;
        for (int ks = 0; ks < nkb / kStageK; ++ks, ring.advance()) {
          if (!ring.claim(b_empty, b_full, kStageK * nb * kBRows * 128, abort, a.status, 201)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int kh = 0; kh < kStageK; ++kh)
            for (int j = 0; j < nb; ++j)
              tma_load_2d(sB + ring.s * kBStageBytes + kh * kBAtomBytes + j * kBRows * 128, &maps.b, &b_full[ring.s],
                          (ks * kStageK + kh) * kTileK, wi.row0 + j * kBRows);
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
    for (int it = next_item(a, blockIdx.x, nitems, false, false); it < nitems && ok;
         it = next_item(a, it + gridDim.x, nitems, false, false), ++li) {
      const WorkItem wi = a.items[it];
      if (!warp_wait(acc_empty, (li & 1) ^ 1u, abort, a.status, 210)) break;
      tc_fence_after();
      const uint32_t idesc = idesc_f16_f32(kRows, (wi.nrows + 15) & ~15);
      for (int ks = 0; ks < nkb / kStageK; ++ks) {
        if (!warp_wait(&b_full[bs.s], bs.ph, abort, a.status, 212)) {
          ok = false;
          break;
        }
        const uint32_t b_addr = smem_u32(sB + bs.s * kBStageBytes);
        if (!warp_wait(&a_full[as.s], as.ph, abort, a.status, 211)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kh = 0; kh < kStageK; ++kh) {
            const uint32_t a_col = tmem_base + kACol0 + as.s * kAStageCols + kh * 64;
#pragma unroll
            for (int kk = 0; kk < kTileK / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(b_addr + kh * kBAtomBytes + kk * 32);
              const uint32_t acc = (ks | kh | kk) != 0 ? 1u : 0u;
              tc_mma_f16_ts(tmem_base, a_col + kk * 8, bdesc, idesc, acc);
              tc_mma_f16_ts(tmem_base + kAccCols, a_col + 32 + kk * 8, bdesc, idesc, acc);
            }
          }
          tc_commit(&a_empty[as.s]);
          tc_commit(&b_empty[bs.s]);
        }
        __syncwarp();
        as.advance();
        bs.advance();
      }
      if (ok && elect_one()) tc_commit(acc_full);
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
    // The kEpiPerQ warps of lane quarter q (rows 32q..32q+31 of both matrices)
    // take the tile's 16-token groups in turn: warp `sub` the groups g with
    // g % kEpiPerQ == sub, from tensor memory to shared memory to global.
    const int q = warp & 3;
    const int sub = (warp - kEpiWarp0) >> 2;
    // the quarter's 32 output columns of the tile's tokens, staged as [token][32]
    // fp16; the quarter's warps write disjoint tokens
    __half *stg = reinterpret_cast<__half *>(smem + kOffStg + q * kStgBytes);
    const int scol = (lane & ~7) + kperm_dst(lane & 7);  // K-permuted order of the down GEMM's operand
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    constexpr int kER = kN / 32;  // exponent registers per lane: token 32c + lane in register c
    int li = 0;
    for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
      const WorkItem wi = a.items[it];
      const bool sh = wi.group == a.E;
      const int ng = (wi.nrows + 15) >> 4;  // 16-token groups of the tile
      // exponent of each token's scaling (lane l of register c: token 32c + l),
      // loaded while the accumulators are still being computed
      int e_l[kER];
#pragma unroll
      for (int c = 0; c < kER; ++c) {
        const int jl = 32 * c + lane;
        e_l[c] = jl < wi.nrows ? a.row_exp[wi.row0 + jl] : 0;
      }
      if (!warp_wait(acc_full, li & 1, abort, a.status, 220)) break;
      tc_fence_after();
      if (sub >= ng) {  // no group for this warp: the accumulators are not read
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
      }
      const int pitch = sh ? a.Is : a.I;
      __half *obase = (sh ? a.h + a.h_shared_off + static_cast<int64_t>(wi.row0 - a.R) * a.Is
                          : a.h + static_cast<int64_t>(wi.row0) * a.I) +
                      wi.mblk * kRows + q * 32;
      for (int g = sub; g < ng; g += kEpiPerQ) {
        const int c16 = 16 * g;
        uint32_t g16[16], u16[16];
        tmem_ld_32x32b_x16(tq + c16, g16);
        tmem_ld_32x32b_x16(tq + kAccCols + c16, u16);
        tmem_ld_wait();
        if (g + kEpiPerQ >= ng) {  // this warp's last read of the accumulators
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(acc_empty);
        }
        const int ec = g >> 1;
        int e_g = e_l[0];
#pragma unroll
        for (int c = 1; c < kER; ++c)
          if (ec == c) e_g = e_l[c];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int e = __shfl_sync(0xffffffffu, e_g, 16 * (g & 1) + jj);
          // silu(gate) * up with gate = g 2^e, up = u 2^e, result scaled by 2^-2e
          const float gt = __uint_as_float(g16[jj]) * pow2i(e);
          const float sg = __fdividef(gt, 1.0f + __expf(-gt));
          stg[(c16 + jj) * 32 + scol] = __float2half_rn(sg * pow2i(-e) * __uint_as_float(u16[jj]));
        }
      }
      __syncwarp();
      // write out this warp's tokens: 4 chunks of 16 bytes per token row, 8 rows per warp instruction
      for (int g = sub; g < ng; g += kEpiPerQ) {
        const int jend = min(16 * g + 16, wi.nrows);
        for (int j = 16 * g + (lane >> 2); j < jend; j += 8) {
          const int c = lane & 3;
          const uint4 v = *reinterpret_cast<const uint4 *>(stg + j * 32 + c * 8);
          *reinterpret_cast<uint4 *>(obase + static_cast<int64_t>(j) * pitch + c * 8) = v;
        }
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------ dequantisation
    // Warp w owns TMEM lane quarter w % 4, i.e. weight rows 32*(w%4) + lane,
    // of W_gate ((dw / 4) % 2 == 0) or W_up, and the 16-byte chunks ch of each
    // K-block with ch % kDqPerQ == dw / 8 (a K-block row is two such chunks).
    // The fp16 values go straight to TMEM (tcgen05.st), where the MMA reads its
    // A operand.
    {
    constexpr int kCh = 2 / kDqPerQ;  // chunks per K-block row for this warp
    const int dw = warp - kDqWarp0;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int m = (dw >> 2) & 1;  // 0: gate, 1: up
    const int half = dw >> 3;     // 0 unless kDqPerQ == 2
    RingCursor<kPkStages> pk;
    RingCursor<kAStages> as;
    bool ok = true;
    static_assert(kSuperK == 4, "the scale/bias stream loads four K-blocks at a time");
    SbStream sb;
    const int first = next_item(a, blockIdx.x, nitems, false, false);
    if (first < nitems) sb.start(sb_row_gu(a, a.items[first], m, r));
    for (int it = first; it < nitems && ok; it = next_item(a, it + gridDim.x, nitems, false, false)) {
      for (int kb = 0; kb < nkb; kb += kAKB) {  // two K-blocks per TMEM stage
        const int j = kb % kSuperK;             // 0 or 2 within the packed stage
        if (j == 0)
          sb.step(kb, nkb, [&](SbRow &nr) {
            const int nx = next_item(a, it + gridDim.x, nitems, false, false);
            if (nx >= nitems) return false;
            nr = sb_row_gu(a, a.items[nx], m, r);
            return true;
          });
        const __half2 s2a = sb.scale(j), b2a = sb.bias(j), s2b = sb.scale(j + 1), b2b = sb.bias(j + 1);
        if (j == 0 && !warp_wait(&pk_full[pk.s], pk.ph, abort, a.status, 230)) {
          ok = false;
          break;
        }
        // row r of the packed tile: 128 bytes = 4 K-blocks of 8 words, in
        // 16-byte chunks placed at chunk ^ (r & 7) by the TMA's 128-byte swizzle;
        // chunk c of K-block j + kk is 2 (j + kk) + c
        const uint8_t *prow = sPk + pk.s * kPkStageBytes + m * kPkTileBytes + r * 128;
        uint4 v[2][kCh];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int c = 0; c < kCh; ++c)
            v[kk][c] = *reinterpret_cast<const uint4 *>(prow + (((2 * (j + kk) + c * kDqPerQ + half) ^ (r & 7)) << 4));
        if (j + kAKB == kSuperK || kb + kAKB >= nkb) {  // words in registers: release the packed stage
          __syncwarp();
          if (lane == 0) mbar_arrive(&pk_empty[pk.s]);
          pk.advance();
        }
        // pieces of 8 columns whose stores overlap the next piece's
        // arithmetic; the first is computed before the stage is known free;
        // one wait. Chunk c of a K-block fills columns 16 c .. 16 c + 15 of
        // the matrix's 32 in that K-block's 64.
        const uint32_t ta = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + kACol0 + as.s * kAStageCols + m * 32;
        uint32_t d8[8];
        dequant2(v[0][0].x, v[0][0].y, s2a, b2a, d8);
        if (!warp_wait(&a_empty[as.s], as.ph ^ 1u, abort, a.status, 231)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int c = 0; c < kCh; ++c) {
            const uint32_t tc = ta + kk * 64 + (c * kDqPerQ + half) * 16;
            if (kk | c) dequant2(v[kk][c].x, v[kk][c].y, kk ? s2b : s2a, kk ? b2b : b2a, d8);
            tmem_st_32x32b_x8(tc, d8);
            dequant2(v[kk][c].z, v[kk][c].w, kk ? s2b : s2a, kk ? b2b : b2a, d8);
            tmem_st_32x32b_x8(tc + 8, d8);
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
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_gemm_gate_up(const GemmArgs &a, int num_sms, cudaStream_t s, bool pdl) {
  if (a.max_items <= 0) return cudaSuccess;
  TmaMaps maps;
  const int H = a.H;
  bool ok = make_map(&maps.w, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.packed, static_cast<uint64_t>(a.E) * 3 * a.I,
                     H / 8, kRows, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.w_sh, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, a.w.sh_packed, static_cast<uint64_t>(3) * a.Is,
                      H / 8, kRows, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && make_map(&maps.b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, a.xt, static_cast<uint64_t>(a.xt_rows), H, kBRows,
                      kTileK, CU_TENSOR_MAP_SWIZZLE_128B);
  maps.b_sh = maps.b;
  if (!ok) return cudaErrorInvalidValue;
  const int grid = std::max(1, std::min(num_sms, a.max_items));
  if (a.gu_tile == GuTile<32>::kN) {
    static std::atomic<uint64_t> smem_set{0};
    const cudaError_t e = ensure_smem_limit(gemm_gate_up_kernel<32>, GuTile<32>::kSmem, smem_set);
    if (e != cudaSuccess) return e;
    return launch_k(gemm_gate_up_kernel<32>, dim3(grid), dim3(GuTile<32>::kThreads), GuTile<32>::kSmem, s, pdl, a, maps);
  }
  if (a.gu_tile != GuTile<128>::kN) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> smem_set{0};
  const cudaError_t e = ensure_smem_limit(gemm_gate_up_kernel<128>, GuTile<128>::kSmem, smem_set);
  if (e != cudaSuccess) return e;
  return launch_k(gemm_gate_up_kernel<128>, dim3(grid), dim3(GuTile<128>::kThreads), GuTile<128>::kSmem, s, pdl, a, maps);
}

}  // namespace moe
