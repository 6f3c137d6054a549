// gemm_common.cuh -- pieces shared by the tensor-core kernels (the gate/up and
// down grouped expert GEMMs, the router): bounded warp waits, the teardown
// drain of in-flight copies, work-item range checks, the scale/bias row loads
// and dequantisation of the weight warps, and TMA descriptor set-up.
#pragma once

#include <cuda.h>

#include <atomic>

#include "kernels.cuh"
#include "sm100.cuh"

namespace moe {
namespace gemm {

using namespace sm100;

constexpr int kBRows = 32;  // TMA box height of activation rows

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

// The producer side of an N-stage TMA ring, run by one thread: claim() waits
// (bounded) for the next stage to be free and arms its full barrier with the
// bytes about to land; advance() steps to the following stage; drain() waits
// for the copies still in flight, so that a CTA that gave up can exit safely.
template <int N>
struct TmaRing {
  int s = 0;
  uint32_t ph = 0, issued = 0, issued_ph = 0;

  __device__ __forceinline__ bool claim(uint64_t *empty, uint64_t *full, uint32_t bytes, volatile int *abort,
                                        DevStatus *st, uint32_t site) {
    if (!mbar_wait(&empty[s], ph ^ 1u, abort, st, site)) return false;
    mbar_arrive_expect_tx(&full[s], bytes);
    issued |= 1u << s;
    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
    return true;
  }
  __device__ __forceinline__ void advance() {
    if (++s == N) {
      s = 0;
      ph ^= 1u;
    }
  }
  __device__ __forceinline__ void drain(uint64_t *full) const { drain_stages<N>(full, issued, issued_ph); }
};

// The consumer side of an N-stage ring: the stage index and the parity of its
// current phase.
template <int N>
struct RingCursor {
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void advance() {
    if (++s == N) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// Whether a work item lies inside the buffers it addresses: its expert, its
// 128-row weight block and its activation rows (routed rows in [0, R), the
// shared expert's rows in [R, R + T)); every TMA coordinate of the item
// derives from these. dn: the down GEMM (weight rows H) or gate/up (I or Is).
__device__ __forceinline__ bool item_in_range(const GemmArgs &a, const WorkItem &wi, bool dn) {
  if (wi.group < 0 || wi.group > a.E) return false;
  const bool sh = wi.group == a.E;
  const int mrows = dn ? a.H : (sh ? a.Is : a.I);
  if (wi.mblk < 0 || wi.mblk >= mrows / kTileM) return false;
  if (wi.nrows < 1 || wi.nrows > (dn ? kTileN : a.gu_tile) || wi.row0 < 0) return false;
  const int64_t end = static_cast<int64_t>(wi.row0) + wi.nrows;
  if (sh) return wi.row0 >= a.R && end <= static_cast<int64_t>(a.R) + a.T;
  return end <= a.R;
}

// The first work item at or after `it` (stepping by the grid) that this CTA
// processes. Without MOE_FLAG_DEBUG that is `it`; with it, items out of range
// are skipped by every warp role alike (so the pipelines stay in step), and
// the role that passes report = true records each one in the status word.
__device__ __forceinline__ int next_item(const GemmArgs &a, int it, int nitems, bool dn, bool report) {
  if (!a.debug) return it;
  while (it < nitems && !item_in_range(a, a.items[it], dn)) {
    if (report) report_error(a.status, kDevBounds, dn ? 150u : 250u, static_cast<uint32_t>(it));
    it += gridDim.x;
  }
  return it;
}

// 2^e as a float for |e| <= 126, built from its exponent bits
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

// The scale and bias row of one weight row, and its K extent.
struct SbRow {
  const uint16_t *S, *B;
  int K;
};

// The scales and biases of K-blocks kb .. kb+3 of one row (bf16 bits, K-block
// kb in the low half of .x); one 8-byte load each where the row allows it.
__device__ __forceinline__ void load_sb4(const SbRow &w, int kb, uint2 &s, uint2 &b) {
  const int nkb = w.K / kTileK;
  if ((nkb & 3) == 0 && ((reinterpret_cast<uintptr_t>(w.S) | reinterpret_cast<uintptr_t>(w.B)) & 7) == 0) {
    s = __ldg(reinterpret_cast<const uint2 *>(w.S + kb));
    b = __ldg(reinterpret_cast<const uint2 *>(w.B + kb));
  } else {
    uint32_t sv[4], bv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      sv[i] = kb + i < nkb ? __ldg(w.S + kb + i) : 0u;
      bv[i] = kb + i < nkb ? __ldg(w.B + kb + i) : 0u;
    }
    s = make_uint2(sv[0] | sv[1] << 16, sv[2] | sv[3] << 16);
    b = make_uint2(bv[0] | bv[1] << 16, bv[2] | bv[3] << 16);
  }
}

__device__ __forceinline__ uint16_t pick_bf16(uint2 v, int j) {
  const uint32_t w = (j & 2) ? v.y : v.x;
  return static_cast<uint16_t>((j & 1) ? w >> 16 : w);
}

// The scales and biases of one weight row as the dequantisation walks its
// K-blocks: four K-blocks per load, one packed stage ahead, and during the
// last packed stage of an item the first four of the next item's row.
struct SbStream {
  SbRow row{}, next{};
  uint2 s_cur{}, b_cur{}, s_nxt{}, b_nxt{};

  __device__ __forceinline__ void start(const SbRow &r) {
    row = next = r;
    load_sb4(row, 0, s_nxt, b_nxt);
  }
  // At K-block kb (a multiple of 4) of a row of nkb K-blocks: K-blocks kb ..
  // kb + 3 become current and the next four are requested; next_row(r) gives
  // the next item's row (returns false if there is none).
  template <class NextRow>
  __device__ __forceinline__ void step(int kb, int nkb, NextRow next_row) {
    s_cur = s_nxt;
    b_cur = b_nxt;
    if (kb + 4 < nkb) {
      load_sb4(row, kb + 4, s_nxt, b_nxt);
    } else if (next_row(next)) {
      load_sb4(next, 0, s_nxt, b_nxt);
    }
  }
  __device__ __forceinline__ void end_item() { row = next; }
  __device__ __forceinline__ __half2 scale(int j) const { return bf16_to_half2_bcast(pick_bf16(s_cur, j)); }
  __device__ __forceinline__ __half2 bias(int j) const { return bf16_to_half2_bcast(pick_bf16(b_cur, j)); }
};

// Dequantise two packed words (16 weights of one row) into 8 fp16 pairs.
__device__ __forceinline__ void dequant2(uint32_t w0, uint32_t w1, __half2 s2, __half2 b2, uint32_t (&d)[8]) {
  const uint4 o0 = dequant_word(w0, s2, b2), o1 = dequant_word(w1, s2, b2);
  d[0] = o0.x;
  d[1] = o0.y;
  d[2] = o0.z;
  d[3] = o0.w;
  d[4] = o1.x;
  d[5] = o1.y;
  d[6] = o1.z;
  d[7] = o1.w;
}

// ---------------------------------------------------------------------------
// host: tensor maps
// ---------------------------------------------------------------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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

// Raises a kernel's dynamic shared-memory limit on the current device, once
// per device (the attribute belongs to the device's context, not the process).
template <typename Kernel>
inline cudaError_t ensure_smem_limit(Kernel kernel, int bytes, std::atomic<uint64_t> &done_devices) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
  if (bit && (done_devices.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit) done_devices.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// rows x cols matrix, row-major; box = box_rows x box_cols elements
inline bool make_map(CUtensorMap *m, CUtensorMapDataType dt, size_t elem, const void *base, uint64_t rows,
                     uint64_t cols, uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * elem};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gemm
}  // namespace moe
