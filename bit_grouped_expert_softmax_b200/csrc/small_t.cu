// small_t.cu -- fused MoE layer for batches of up to 8 tokens.
//
// Batch-1 decode has almost no weight reuse, so memory bandwidth sets the
// ceiling (aioga.com record of the Lily report, article body paragraph 6).
// One persistent cooperative kernel, one CTA per SM, does the whole layer and
// requests every weight byte it needs as early as the data dependences allow:
//
//   entry    the shared expert needs no routing: each CTA requests, with bulk
//            asynchronous copies into shared memory, its shared-expert gate/up
//            row block and the shared expert's down rows of its output slice,
//            before it waits for the kernel ahead on the stream (programmatic
//            dependent launch) and before it looks at a logit
//   routing  every CTA routes the (<= 8) tokens itself (same result in every
//            CTA) with all its warps: each warp ranks the logits of one
//            32-expert slice of one token by shuffles and keeps that slice's
//            top k, then one thread per candidate counts the candidates that
//            precede it; the distinct experts are listed and their gate/up
//            row blocks requested from several warps at once, their down rows
//            right after
//   gate/up  each 16-row block of an expert is split along K over several
//            warps; tensor-core mma.sync m16n8k16 with A = dequantised weights
//            (fp16 q*scale+bias, as in the grouped GEMM) and B = the tokens
//            (N = 8 covers every token at once); the partial sums are reduced
//            in a fixed order by up to four warps, each of which stores its
//            part of h = silu(gate) * up to a small scratch as tagged words
//            (two fp16 values and the launch tag in one 8-byte store)
//   down     each CTA owns 16 output features; warp w takes the used experts
//            u = w, w + 16, ...; it reads expert u's h (bounded polling, until
//            every word carries this launch's tag), then multiplies it by the
//            down rows already in shared memory and weights each token's
//            result by its routing weight; the warps' results are summed in a
//            fixed order and rounded once
//   exit     every CTA adds itself to an exit count (release increment) once it
//            has read the launch tag; a warp of CTA 0 waits for the full count,
//            clears the counters and records the tag for the next launch on
//            the stream. A CTA that gave up on a wait waits for its own copies
//            still in flight before it leaves
//
// There is no grid-wide barrier and no readiness counter: an expert's down
// product starts as soon as that expert's h words have all arrived, while
// other experts' gate/up blocks finish.
//
// Operand order along K: packed word W holds elements 8W..8W+7; the fp16
// operands store them at positions 8W + s in the pair order (0,4),(1,5),(2,6),
// (3,7) that the int4 conversion produces. Within each block of 16 words,
// thread c of an mma quad takes words 4c..4c+3, one per mma pair; both
// operands index the same word, so the products are those of the plain dot
// product.
#include <algorithm>

#include "gemm_common.cuh"
#include "kernels.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace moe {

namespace {

using namespace sm100;

constexpr int kSTWarps = 16;
constexpr int kSTThreads = kSTWarps * 32;
constexpr int kRowBlock = 16;  // weight rows per mma tile
constexpr int kXPad = 32;      // fp16 padding per staged token row (bank spread)
constexpr int kSlices = kMaxExperts / 32;  // 32-expert slices of a token's logits
constexpr int kCandPerToken = kSlices * kMaxTopK;  // routing candidates of one token, at most
static_assert(kSmallTMaxU == kSmallT * kMaxTopK + 1, "one shared plus at most T*k routed experts");
constexpr int kMaxU = kSmallTMaxU;
constexpr int kPairsPerLane = 4;  // staged poll of tagged h words: at most 128 pairs per expert

struct SmallTShared {
  int ids[kSmallT][kMaxTopK];
  uint32_t wkey[kSmallT][kMaxTopK];     // order keys of the chosen experts' logits
  float wt[kSmallT][kMaxTopK];
  int xexp[kSmallT];                   // max |x| bits, then the token's exponent
  uint32_t bitmap[kMaxExperts / 32];   // experts used by any token
  int ulist[kMaxU];                    // [0] the shared expert (E), then the distinct experts ascending
  uint32_t umask[kMaxU];               // tokens routed to each
  int8_t uslot[kMaxU][kSmallT];        // slot j of expert u in token t (-1: none; k: shared)
  int b_iss[4];                        // copies issued into each phase-1 stage
  int d_iss[kMaxU];                    // copies issued into each phase-2 stage
  int nU;
  uint32_t tag;  // this launch's tag of the SwiGLU output words
  int abort;
};

// Per-launch layout of the dynamic shared memory.
struct StLayout {
  int Imax, kw, ks;   // max intermediate, K per warp and warps per row block in phase 1
  int nb, nd;         // stages of the phase-1 and phase-2 rings
  size_t x_off, red_off, b_off, d_off, bar_off, bytes;
  size_t b_stage, d_stage;
};

constexpr size_t kStBudget = 220 * 1024;

__host__ __device__ inline StLayout st_layout(int H, int I, int Is, int T, int k) {
  StLayout L;
  L.Imax = I > Is ? I : Is;
  // K is split over ks warps per 16-row block, each walking its slice in
  // 16-word (128-element) blocks: ks is the largest power of two <= 8 (so the
  // 16 warps form whole groups) whose slices are whole 128-element blocks.
  L.ks = 8;
  while (L.ks > 1 && (H / 128) % L.ks != 0) L.ks >>= 1;
  L.kw = H / L.ks;
  L.b_stage = static_cast<size_t>(2) * kRowBlock * (H / 2) + static_cast<size_t>(4) * kRowBlock * (H / kGroup) * 2;
  L.d_stage = static_cast<size_t>(kRowBlock) * (L.Imax / 2) + static_cast<size_t>(2) * kRowBlock * (L.Imax / kGroup) * 2;
  L.x_off = 0;
  const size_t x_bytes = static_cast<size_t>(kSmallT) * (H + kXPad) * 2;
  L.red_off = (x_bytes + 127) / 128 * 128;
  // partial sums of the K slices; during routing, the top-k candidates
  const size_t red_bytes = static_cast<size_t>(kSTThreads) * 8 * 4;
  L.b_off = L.red_off + red_bytes;
  // phase-1 ring: the most stages (up to 4) that still leave the down ring one
  // stage per used expert (or at least 8)
  const int want_d = T * k + 1;
  L.nb = 0;
  L.nd = 0;
  for (int nb = 4; nb >= 2; --nb) {
    const size_t used = L.b_off + nb * L.b_stage + 512;
    if (used >= kStBudget) continue;
    int nd = static_cast<int>((kStBudget - used) / L.d_stage);
    nd = nd < want_d ? nd : want_d;
    if (nd >= (want_d < 8 ? want_d : 8) || nb == 2) {
      L.nb = nb;
      L.nd = nd;
      break;
    }
  }
  L.d_off = L.b_off + L.nb * L.b_stage;
  L.bar_off = L.d_off + L.nd * L.d_stage;
  L.bytes = L.bar_off + 2 * (L.nb + L.nd) * 8 + 16;
  return L;
}

// Bounded wait on an mbarrier phase; on timeout or abort returns false.
__device__ __forceinline__ bool st_wait(uint64_t *bar, uint32_t parity, volatile int *abort, DevStatus *st,
                                        uint32_t site, unsigned long long budget) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > budget) {
      *abort = 1;
      report_error(st, kDevTimeout, site, blockIdx.x);
      return false;
    }
  }
}

// Whole warp: bounded wait until *cnt >= need, with acquire ordering for every
// lane's later loads. Gives up on the CTA's abort flag or after the budget
// (then records a timeout with the expert index and sets the abort flag).
__device__ __forceinline__ bool wait_count(const uint32_t *cnt, uint32_t need, volatile int *abort, DevStatus *st,
                                           uint32_t site, uint32_t detail, unsigned long long budget) {
  unsigned long long t0 = 0;
  for (unsigned it = 0;; ++it) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
    if (__all_sync(0xffffffffu, v >= need)) return true;
    if (__any_sync(0xffffffffu, *abort != 0)) return false;
    if (it == 0) t0 = global_ns();
    __nanosleep(64);
    int late = 0;
    if ((it & 15u) == 15u) late = global_ns() - t0 > budget ? 1 : 0;
    if (__shfl_sync(0xffffffffu, late, 0)) {
      if ((threadIdx.x & 31) == 0) {
        *abort = 1;
        report_error(st, kDevTimeout, site, detail);
      }
      return false;
    }
  }
}

// One thread: wait (bounded) for the last phase issued into each stage of a
// ring, so that no copy into this CTA's shared memory is still in flight.
__device__ __forceinline__ void drain_ring(uint64_t *full, const int *issued, int n) {
  for (int s = 0; s < n; ++s) {
    if (issued[s] <= 0) continue;
    const uint32_t par = static_cast<uint32_t>(issued[s] - 1) & 1u;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(&full[s], par) && global_ns() - t0 < kWaitBudgetNs) {
    }
  }
}

// The SwiGLU outputs go from the CTAs that compute them to the CTAs that
// multiply them by the down rows as 8-byte words: two fp16 values (K positions
// 2w, 2w + 1) in the low half and the launch's tag in the high half. A naturally
// aligned 8-byte store or load is single-copy atomic, so a reader that sees
// the tag also sees the values stored with it: no fence, no counter and no
// second read are needed between the two sides. The tag changes every launch
// and is never 0 (the value the scratch is cleared to).
__device__ __forceinline__ void st_tagged(uint64_t *p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ ulonglong2 ld_tagged2(const uint64_t *p) {
  ulonglong2 r;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(r.x), "=l"(r.y) : "l"(p) : "memory");
  return r;
}
__device__ __forceinline__ bool tag_ok(const ulonglong2 &v, uint32_t tag) {
  return static_cast<uint32_t>(v.x >> 32) == tag && static_cast<uint32_t>(v.y >> 32) == tag;
}
// the four fp16 values of a word pair
__device__ __forceinline__ uint2 tagged_values(const ulonglong2 &v) {
  return make_uint2(static_cast<uint32_t>(v.x), static_cast<uint32_t>(v.y));
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Weight pointers of one expert id (E = the shared expert).
struct ExpertPtrs {
  const uint32_t *packed;
  const uint16_t *scales, *biases;
  int Iu;
};

__device__ __forceinline__ ExpertPtrs expert_ptrs(const SmallTArgs &a, int e) {
  ExpertPtrs p;
  if (e == a.E) {
    p.packed = a.w.sh_packed;
    p.scales = a.w.sh_scales;
    p.biases = a.w.sh_biases;
    p.Iu = a.Is;
  } else {
    p.packed = a.w.packed + static_cast<size_t>(e) * 3 * a.I * a.H / 8;
    p.scales = a.w.scales + static_cast<size_t>(e) * 3 * a.I * a.H / kGroup;
    p.biases = a.w.biases + static_cast<size_t>(e) * 3 * a.I * a.H / kGroup;
    p.Iu = a.I;
  }
  return p;
}

// 8 bf16 values -> 8 fp16 values scaled by 2^-ex, in operand order
__device__ __forceinline__ uint4 x_scaled_fp16(uint4 v, int ex) {
  const float scale = __int_as_float((127 - ex) << 23);  // 2^-ex, |ex| <= 100
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  __half hv[8];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    hv[2 * q] = __float2half_rn(__uint_as_float(w4[q] << 16) * scale);
    hv[2 * q + 1] = __float2half_rn(__uint_as_float(w4[q] & 0xffff0000u) * scale);
  }
  uint4 o;
  uint32_t *op = reinterpret_cast<uint32_t *>(&o);
#pragma unroll
  for (int s2 = 0; s2 < 8; s2 += 2) op[s2 / 2] = pack_half2(hv[kperm_src(s2)], hv[kperm_src(s2 + 1)]);
  return o;
}

__device__ __forceinline__ float bf16x8_absmax(uint4 v) {
  const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    m = fmaxf(m, fmaxf(fabsf(__uint_as_float(w4[q] << 16)), fabsf(__uint_as_float(w4[q] & 0xffff0000u))));
  return m;
}

}  // namespace

int small_t_grid(int num_sms) { return num_sms; }

size_t small_t_smem_bytes(int T, int H, int k, int I, int Is) {
  const StLayout L = st_layout(H, I, Is, T, k);
  if (L.nb < 2 || L.nd < 2) return static_cast<size_t>(1) << 30;  // does not fit: not eligible
  return L.bytes;
}

bool small_t_fits(int T, int H, int k, int I, int Is, int num_sms) {
  return T >= 1 && T <= kSmallT && H % 256 == 0 && H / kRowBlock <= small_t_grid(num_sms) &&
         small_t_smem_bytes(T, H, k, I, Is) <= kStBudget;
}

__global__ void __launch_bounds__(kSTThreads, 1) small_t_kernel(const SmallTArgs a) {
  extern __shared__ __align__(1024) uint8_t dyn[];
  __shared__ SmallTShared sh;
  const StLayout L = st_layout(a.H, a.I, a.Is, a.T, a.k);
  const int T = a.T, E = a.E, k = a.k, H = a.H;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;  // mma fragment coordinates
  __half *xs = reinterpret_cast<__half *>(dyn + L.x_off);  // [8][H + kXPad]
  float *red = reinterpret_cast<float *>(dyn + L.red_off); // [512 threads][8]
  uint32_t *cand_key = reinterpret_cast<uint32_t *>(red);  // routing: [T][kCandPerToken]
  int *cand_id = reinterpret_cast<int *>(red) + kSmallT * kCandPerToken;
  uint8_t *bring = dyn + L.b_off;
  uint8_t *dring = dyn + L.d_off;
  uint64_t *b_full = reinterpret_cast<uint64_t *>(dyn + L.bar_off);
  uint64_t *d_full = b_full + L.nb;
  volatile int *abort = &sh.abort;
  uint64_t *hb = a.hbuf;                             // [T][k+1][Imax/2] tagged words, operand order
  uint32_t *exit_count = a.sync + kSmallTExitWord;
  uint32_t *router_count = a.sync + kSmallTRouterWord;  // CTAs whose router scores are published
  const unsigned long long budget = a.wait_ns;
  const int Imax = L.Imax;
  const int nrb_sh = a.Is / kRowBlock;               // the shared expert's row blocks: the first units
  const int nrb = a.I / kRowBlock;                   // row blocks of a routed expert
  const int n_dblk = H / kRowBlock;                  // phase-2 output blocks (one per CTA)
  const int hw = H / 8;                              // packed words per gate/up row
  const bool has_dblk = blockIdx.x < n_dblk;

  // ---- set-up --------------------------------------------------------------------
  if (threadIdx.x == 0) {
    for (int s = 0; s < L.nb + L.nd; ++s) mbar_init(&b_full[s], 1);
    sh.abort = 0;
    sh.ulist[0] = E;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (threadIdx.x < kSmallT) sh.xexp[threadIdx.x] = 0;
  if (threadIdx.x < kMaxExperts / 32) sh.bitmap[threadIdx.x] = 0;
  if (threadIdx.x < 4) sh.b_iss[threadIdx.x] = 0;
  for (int i = threadIdx.x; i < kMaxU; i += kSTThreads) {
    sh.umask[i] = 0;
    sh.d_iss[i] = 0;
#pragma unroll
    for (int t = 0; t < kSmallT; ++t) sh.uslot[i][t] = -1;
  }
  __syncthreads();

  // Phase-1 units are (expert, 16-row block), the shared expert's blocks first;
  // unit q of this CTA is global unit blockIdx.x + q * gridDim.x and uses ring
  // stage q % nb. A unit is six bulk copies (gate rows, up rows, their scales
  // and biases) from lanes 0..5 of the calling warp.
  // a round takes at most one unit per ring stage: every unit of a round has
  // its copies issued before the round starts (the refill follows the round)
  const int units_per_round = min(kSTWarps / L.ks, L.nb);
  auto issue_b = [&](int q) {  // all lanes of one warp
    const int unit = blockIdx.x + q * gridDim.x;
    int e, rb;
    if (unit < nrb_sh) {
      e = E;
      rb = unit;
    } else {
      e = sh.ulist[1 + (unit - nrb_sh) / nrb];
      rb = (unit - nrb_sh) % nrb;
    }
    const ExpertPtrs p = expert_ptrs(a, e);
    const int s = q % L.nb;
    uint8_t *st = bring + s * L.b_stage;
    const uint32_t pk = kRowBlock * (H / 2), sb = kRowBlock * (H / kGroup) * 2;
    uint64_t *bar = &b_full[s];
    // the stage's only arrival is this expect-tx, so it cannot complete before
    // it, whatever order the copies land in
    if (lane == 0) {
      mbar_arrive_expect_tx(bar, 2 * pk + 4 * sb);
      sh.b_iss[s] += 1;
    }
    __syncwarp();
    if (lane < 2) {
      const size_t row0 = static_cast<size_t>(lane) * p.Iu + rb * kRowBlock;
      bulk_g2s(st + lane * pk, p.packed + row0 * hw, pk, bar);
    } else if (lane < 6) {  // scales / biases, gate then up
      const int m = (lane - 2) >> 1;
      const size_t row0 = static_cast<size_t>(m) * p.Iu + rb * kRowBlock;
      const uint16_t *src = ((lane & 1) ? p.biases : p.scales) + row0 * (H / kGroup);
      bulk_g2s(st + 2 * pk + (lane - 2) * sb, src, sb, bar);
    }
    __syncwarp();
  };
  // Phase-2 stage u % nd holds expert u's down rows [n0, n0 + 16): three copies,
  // ten experts per warp-wide step.
  auto issue_d_range = [&](int u0, int u1) {  // all lanes of one warp
    const int n0 = blockIdx.x * kRowBlock;
    for (int ub = u0; ub < u1; ub += 10) {
      const int sub = lane / 3, l = lane % 3, u = ub + sub;
      if (sub < 10 && u < u1) {
        const ExpertPtrs p = expert_ptrs(a, sh.ulist[u]);
        const int s = u % L.nd;
        uint8_t *st = dring + s * L.d_stage;
        const uint32_t pk = kRowBlock * (p.Iu / 2);
        const uint32_t sb = kRowBlock * (p.Iu / kGroup) * 2;
        uint64_t *bar = &d_full[s];
        if (l == 0) {
          mbar_arrive_expect_tx(bar, pk + 2 * sb);
          sh.d_iss[s] += 1;
          bulk_g2s(st, p.packed + static_cast<size_t>(2) * p.Iu * H / 8 + static_cast<size_t>(n0) * (p.Iu / 8), pk,
                   bar);
        } else {
          const size_t g0 = static_cast<size_t>(2) * p.Iu * H / kGroup + static_cast<size_t>(n0) * (p.Iu / kGroup);
          bulk_g2s(st + kRowBlock * (Imax / 2) + (l - 1) * sb, ((l == 2) ? p.biases : p.scales) + g0, sb, bar);
        }
      }
      __syncwarp();
    }
  };

  // ---- entry: the shared expert's copies need no routing -----------------------------
  // They read only the weights, so they are issued before the wait for the
  // kernel ahead on the stream (programmatic dependent launch): x, the
  // logits, the counters and the scratch are touched only after it.
  const bool shared_first = blockIdx.x < nrb_sh;  // unit 0 is a shared-expert block
  if (warp == 0 && shared_first) issue_b(0);
  if (warp == 1 && has_dblk) issue_d_range(0, 1);  // expert u = 0 is the shared one
  pdl_wait();
  // this launch's tag: one more than the last launch's (0 skipped); the word is
  // written only by the last step of a launch, once every CTA has read it
  if (threadIdx.x == 0) {
    uint32_t e;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(e) : "l"(a.sync + kSmallTEpochWord) : "memory");
    sh.tag = e + 1 == 0 ? 1u : e + 1;
  }
  // every CTA of this grid is resident once all have passed here, so the next
  // launch's CTAs, which take SMs only as this grid's leave, cannot keep one
  // of them waiting
  pdl_trigger();

  // tokens: every thread loads its chunks of x now (kept in registers) so the
  // loads overlap the logits loads of the routing below; a warp's 32 chunks of
  // 8 values belong to one token since H / 8 is a multiple of 32
  constexpr int kXPer = kSmallT * 2048 / 8 / kSTThreads;  // cached chunks per thread (H <= 2048)
  const int nxc = T * hw;                                   // 8-value chunks of x
  uint4 xv[kXPer];
#pragma unroll
  for (int i = 0; i < kXPer; ++i) {
    const int idx = threadIdx.x + i * kSTThreads;
    xv[i] = idx < nxc ? __ldg(reinterpret_cast<const uint4 *>(a.x) + idx) : make_uint4(0, 0, 0, 0);
  }

  // ---- router scores, when they are computed here ---------------------------------------
  // CTA b scores experts b, b + G, ... for every token: each (expert, token)
  // dot product over H is split into 256-element slices over warps (fp32
  // products of the bf16 operands), the slices summed in a fixed order. The
  // scores go to global memory and are published with a release increment;
  // every CTA then waits (bounded, acquire) until all scoring CTAs are done.
  if (a.router_w) {
    float *lw = const_cast<float *>(a.logits);
    const int n_mine = blockIdx.x < static_cast<unsigned>(E) ? (E - 1 - blockIdx.x) / gridDim.x + 1 : 0;
    const int nks = H / 256;
    const int n_part = n_mine * T * nks;  // (expert, token, slice) partial sums of this CTA
    for (int pw = warp; pw < n_part; pw += kSTWarps) {
      const int pair = pw / nks, ks = pw % nks;
      const int e = blockIdx.x + (pair / T) * gridDim.x, t = pair % T;
      const uint4 xv8 = __ldg(reinterpret_cast<const uint4 *>(a.x + static_cast<size_t>(t) * H + ks * 256) + lane);
      const uint4 wv8 = __ldg(reinterpret_cast<const uint4 *>(a.router_w + static_cast<size_t>(e) * H + ks * 256) + lane);
      const uint32_t xs[4] = {xv8.x, xv8.y, xv8.z, xv8.w}, ws[4] = {wv8.x, wv8.y, wv8.z, wv8.w};
      float acc = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc = fmaf(__uint_as_float(xs[q] << 16), __uint_as_float(ws[q] << 16), acc);
        acc = fmaf(__uint_as_float(xs[q] & 0xffff0000u), __uint_as_float(ws[q] & 0xffff0000u), acc);
      }
      acc = warp_sum(acc);
      if (lane == 0) red[pw] = acc;
    }
    __syncthreads();
    for (int pair = threadIdx.x; pair < n_mine * T; pair += kSTThreads) {
      float sum = 0.f;
      for (int ks = 0; ks < nks; ++ks) sum += red[pair * nks + ks];
      const int e = blockIdx.x + (pair / T) * gridDim.x, t = pair % T;
      lw[static_cast<size_t>(t) * E + e] = sum;
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0 && n_mine > 0)
      asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(router_count) : "memory");
    const uint32_t n_scoring = static_cast<uint32_t>(min(E, static_cast<int>(gridDim.x)));
    if (warp == 0) wait_count(router_count, n_scoring, abort, a.status, 43, 0, budget);
    __syncthreads();
  }

  // ---- routing, step 1: the top k of each 32-expert slice of each token ----------------
  // Order: larger float32 logit first, equal logits lower expert id first (a
  // strict total order, since ids differ). One key per lane; a lane's rank in
  // its slice is the number of lanes that precede it in that order, counted
  // with shuffles. Lanes of rank < k write their candidate to position
  // slice * k + rank of the token's candidate list (key 0: no expert there;
  // it precedes nothing valid and is never among a token's top k, as k <= E).
  const int nsl = (E + 31) / 32;
  {  // empty entries (key 0) pad each token's list to a multiple of four
    const int npad = ((nsl * k + 3) & ~3) - nsl * k;
    if (threadIdx.x < T * npad) {
      const int t = threadIdx.x / npad, m = nsl * k + threadIdx.x % npad;
      cand_key[t * kCandPerToken + m] = 0u;
      cand_id[t * kCandPerToken + m] = 0x7fffffff;
    }
  }
  for (int un = warp; un < T * nsl; un += kSTWarps) {
    const int t = un / nsl, sl = un % nsl, e = sl * 32 + lane;
    // coherent load: with the router in this kernel, other CTAs wrote the scores
    const uint32_t key = e < E ? float_key(__ldcg(a.logits + static_cast<size_t>(t) * E + e)) : 0u;
    int rank = 0;
#pragma unroll 8
    for (int m = 0; m < 32; ++m) {
      const uint32_t km = __shfl_sync(0xffffffffu, key, m);
      rank += (km > key || (km == key && m < lane)) ? 1 : 0;
    }
    if (rank < k) {
      cand_key[t * kCandPerToken + sl * k + rank] = key;
      cand_id[t * kCandPerToken + sl * k + rank] = e;
    }
  }
  // max |x| of each token (the power-of-two scale of its fp16 copy)
#pragma unroll
  for (int i = 0; i < kXPer; ++i) {
    const int idx0 = (threadIdx.x & ~31) + i * kSTThreads;
    const float m = warp_max(bf16x8_absmax(xv[i]));
    if (lane == 0 && idx0 < nxc && m > 0.f) atomicMax(&sh.xexp[idx0 / hw], __float_as_int(m));
  }
  for (int i0 = kXPer * kSTThreads; i0 < nxc; i0 += kSTThreads) {  // H > 2048
    const int idx = threadIdx.x + i0, idx0 = (threadIdx.x & ~31) + i0;
    float m = 0.f;
    if (idx < nxc) m = bf16x8_absmax(__ldg(reinterpret_cast<const uint4 *>(a.x) + idx));
    m = warp_max(m);
    if (lane == 0 && idx0 < nxc && m > 0.f) atomicMax(&sh.xexp[idx0 / hw], __float_as_int(m));
  }
  __syncthreads();
  // this CTA has read the launch tag and is past the router-score wait: it
  // reads neither counter again (the release orders the tag read before it)
  if (threadIdx.x == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(exit_count) : "memory");

  // ---- routing, step 2: the token's top k among its slices' candidates --------------------
  // The token's top k lie among the slices' top k. One thread per candidate
  // counts the candidates that precede it (16-byte reads of the token's list,
  // four independent counts: no long dependent chain); the candidate with
  // count j < k is the token's j-th expert. The list is padded to a multiple
  // of four with empty entries (key 0), which precede nothing.
  const int nc = nsl * k, nc4 = (nc + 3) & ~3;
  {
    for (int gi = threadIdx.x; gi < T * nc; gi += kSTThreads) {
      const int t = gi / nc, i = gi - t * nc;
      const uint32_t *kl = cand_key + t * kCandPerToken;
      const int *il = cand_id + t * kCandPerToken;
      const uint32_t ck = kl[i];
      const int ci = il[i];
      int r0 = 0, r1 = 0, r2 = 0, r3 = 0;
#pragma unroll 4
      for (int m = 0; m < nc4; m += 4) {
        const uint4 kq = *reinterpret_cast<const uint4 *>(kl + m);
        const int4 iq = *reinterpret_cast<const int4 *>(il + m);
        r0 += (kq.x > ck || (kq.x == ck && iq.x < ci)) ? 1 : 0;
        r1 += (kq.y > ck || (kq.y == ck && iq.y < ci)) ? 1 : 0;
        r2 += (kq.z > ck || (kq.z == ck && iq.z < ci)) ? 1 : 0;
        r3 += (kq.w > ck || (kq.w == ck && iq.w < ci)) ? 1 : 0;
      }
      const int rank = r0 + r1 + r2 + r3;
      if (ck != 0u && rank < k) {
        sh.ids[t][rank] = ci;
        sh.wkey[t][rank] = ck;
        atomicOr(&sh.bitmap[ci >> 5], 1u << (ci & 31));
      }
    }
  }
  __syncthreads();
  // in parallel: the distinct experts (warp 0), each token's renormalised
  // weights (warps 1..T), each (token, slot)'s expert index (warps 9, 10) and
  // each token's power-of-two scale (warp 11)
  if (warp == 0) {
    // u = 1 + the rank of each set bit of the bitmap; u = 0 is the shared expert
    int before = 0;
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
      const uint32_t wbits = sh.bitmap[i];
      if ((wbits >> lane) & 1u) sh.ulist[1 + before + __popc(wbits & ((1u << lane) - 1u))] = 32 * i + lane;
      before += __popc(wbits);
    }
    if (lane == 0) sh.nU = before + 1;
    if (lane < T) sh.uslot[0][lane] = static_cast<int8_t>(k);
    if (lane == 0) sh.umask[0] = (1u << T) - 1u;
  } else if (warp <= T) {
    // the softmax over all E restricted to the chosen k and renormalised is
    // exp(l_j - l_max) over the sum of those k terms (l_max: the first chosen)
    const int t = warp - 1;
    const float ex = lane < k ? expf(key_float(sh.wkey[t][lane]) - key_float(sh.wkey[t][0])) : 0.f;
    const float z = warp_sum(ex);
    if (lane < k) sh.wt[t][lane] = ex / z;
  } else if (warp == 9 || warp == 10) {
    const int f = (warp - 9) * 32 + lane;  // (token, slot) pairs, T * k <= 128: two passes of 64
    for (int ff = f; ff < T * k; ff += 64) {
      const int t = ff / k, j = ff % k, e = sh.ids[t][j];
      int u = 1 + __popc(sh.bitmap[e >> 5] & ((1u << (e & 31)) - 1u));
      for (int i = 0; i < (e >> 5); ++i) u += __popc(sh.bitmap[i]);
      atomicOr(&sh.umask[u], 1u << t);
      sh.uslot[u][t] = static_cast<int8_t>(j);
    }
  } else if (warp == 11 && lane < kSmallT) {  // per-token power-of-two scale: max |x| in [2, 4) after scaling
    const float amax = __int_as_float(sh.xexp[lane]);
    int ex = 0;
    if (amax > 0.f && amax <= 3.0e38f) ex = min(max(ilogbf(amax) - 1, -100), 100);
    sh.xexp[lane] = ex;
  }
  __syncthreads();
  const int nU = sh.nU;
  const int n_units = nrb_sh + (nU - 1) * nrb;
  const int my_units = blockIdx.x < n_units ? (n_units - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  // the requests block their warp while many copies are outstanding, so each
  // phase-1 unit goes out from its own warp (2, 3, ...); the routed experts'
  // down rows, needed only after gate/up, follow them (below)
  if (warp >= 2) {
    const int q = (shared_first ? 1 : 0) + warp - 2;
    if (q < min(my_units, L.nb)) issue_b(q);
  }
  // stage the tokens: fp16 scaled by 2^-e in operand order
#pragma unroll
  for (int i = 0; i < kXPer; ++i) {
    const int idx = threadIdx.x + i * kSTThreads;
    if (idx < nxc)
      *reinterpret_cast<uint4 *>(xs + static_cast<size_t>(idx / hw) * (H + kXPad) + (idx % hw) * 8) =
          x_scaled_fp16(xv[i], sh.xexp[idx / hw]);
  }
  for (int idx = threadIdx.x + kXPer * kSTThreads; idx < nxc; idx += kSTThreads)
    *reinterpret_cast<uint4 *>(xs + static_cast<size_t>(idx / hw) * (H + kXPad) + (idx % hw) * 8) =
        x_scaled_fp16(__ldg(reinterpret_cast<const uint4 *>(a.x) + idx), sh.xexp[idx / hw]);
  // rows t >= T are left as they are: an mma output column depends only on its
  // own token column, and the columns of rows t >= T are never read
  __syncthreads();
  // the down rows go out after every gate/up request of this CTA, so the
  // memory system serves the gate/up rows first
  if (warp == 1 && has_dblk) issue_d_range(1, min(nU, L.nd));

  // ---- gate/up ---------------------------------------------------------------------
  const int slot = warp / L.ks, kq = warp % L.ks;  // unit slot in a round, K slice of this warp
  const int rounds = (my_units + units_per_round - 1) / units_per_round;
  const bool slot_used = slot < units_per_round;  // warps of an unused slot only join the barriers
  const int ng = H / kGroup;
  const int n_pub = min(L.ks, 4);  // warps per unit that reduce its K slices and store its h
  for (int r = 0; r < rounds; ++r) {
    const int q = slot_used ? r * units_per_round + slot : my_units;
    // two accumulator sets per matrix (even and odd words): shorter dependent chains
    float accg[4] = {0.f, 0.f, 0.f, 0.f}, accu[4] = {0.f, 0.f, 0.f, 0.f};
    float accg2[4] = {0.f, 0.f, 0.f, 0.f}, accu2[4] = {0.f, 0.f, 0.f, 0.f};
    int u = 0, rb = 0, unit = 0;
    if (q < my_units) {
      unit = blockIdx.x + q * gridDim.x;
      if (unit < nrb_sh) {
        u = 0;
        rb = unit;
      } else {
        u = 1 + (unit - nrb_sh) / nrb;
        rb = (unit - nrb_sh) % nrb;
      }
      const int s = q % L.nb;
      int ok = 1;
      if (lane == 0) ok = st_wait(&b_full[s], (q / L.nb) & 1u, abort, a.status, 40, budget) ? 1 : 0;
      if (__shfl_sync(0xffffffffu, ok, 0)) {
        const uint8_t *st = bring + s * L.b_stage;
        const uint32_t *pg = reinterpret_cast<const uint32_t *>(st);
        const uint32_t *pu = pg + kRowBlock * hw;
        const uint16_t *sbp = reinterpret_cast<const uint16_t *>(st + 2 * kRowBlock * (H / 2));
        const uint16_t *sg = sbp, *bg = sbp + kRowBlock * ng, *su = sbp + 2 * kRowBlock * ng,
                       *bu = sbp + 3 * kRowBlock * ng;
        const __half *xrow = xs + static_cast<size_t>(g) * (H + kXPad);
        for (int wb = kq * L.kw / 8; wb < (kq + 1) * L.kw / 8; wb += 16) {  // blocks of 16 words
          const int w0 = wb + 4 * c;  // this thread's four words (one scale group)
          const int grp = w0 / 8;
          const __half2 sg0 = bf16_to_half2_bcast(sg[g * ng + grp]), bg0 = bf16_to_half2_bcast(bg[g * ng + grp]);
          const __half2 sg1 = bf16_to_half2_bcast(sg[(g + 8) * ng + grp]),
                        bg1 = bf16_to_half2_bcast(bg[(g + 8) * ng + grp]);
          const __half2 su0 = bf16_to_half2_bcast(su[g * ng + grp]), bu0 = bf16_to_half2_bcast(bu[g * ng + grp]);
          const __half2 su1 = bf16_to_half2_bcast(su[(g + 8) * ng + grp]),
                        bu1 = bf16_to_half2_bcast(bu[(g + 8) * ng + grp]);
          const uint4 wg0 = *reinterpret_cast<const uint4 *>(pg + g * hw + w0);
          const uint4 wg1 = *reinterpret_cast<const uint4 *>(pg + (g + 8) * hw + w0);
          const uint4 wu0 = *reinterpret_cast<const uint4 *>(pu + g * hw + w0);
          const uint4 wu1 = *reinterpret_cast<const uint4 *>(pu + (g + 8) * hw + w0);
          const uint32_t ag0[4] = {wg0.x, wg0.y, wg0.z, wg0.w}, ag1[4] = {wg1.x, wg1.y, wg1.z, wg1.w};
          const uint32_t au0[4] = {wu0.x, wu0.y, wu0.z, wu0.w}, au1[4] = {wu1.x, wu1.y, wu1.z, wu1.w};
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const uint4 xb = *reinterpret_cast<const uint4 *>(xrow + (w0 + p) * 8);
            const uint4 g0 = dequant_word(ag0[p], sg0, bg0), g1 = dequant_word(ag1[p], sg1, bg1);
            const uint4 u0 = dequant_word(au0[p], su0, bu0), u1 = dequant_word(au1[p], su1, bu1);
            float(&ag)[4] = (p & 1) ? accg2 : accg;
            float(&au)[4] = (p & 1) ? accu2 : accu;
            mma16816(ag, g0.x, g1.x, g0.y, g1.y, xb.x, xb.y);
            mma16816(ag, g0.z, g1.z, g0.w, g1.w, xb.z, xb.w);
            mma16816(au, u0.x, u1.x, u0.y, u1.y, xb.x, xb.y);
            mma16816(au, u0.z, u1.z, u0.w, u1.w, xb.z, xb.w);
          }
        }
      }
    }
    // partial sums of the K slices, reduced in slice order by the unit's first warp
    float *rp = red + static_cast<size_t>(threadIdx.x) * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      rp[i] = accg[i] + accg2[i];
      rp[4 + i] = accu[i] + accu2[i];
    }
    __syncthreads();
    const bool live = __all_sync(0xffffffffu, *abort == 0);  // warp-uniform: the block below syncs the warp
    // The unit's first n_pub warps each reduce the C-fragment elements i = kq,
    // kq + n_pub, ... over the K slices (slice order) and store their h as
    // tagged words (the warp is shuffled so that one lane stores each pair).
    if (q < my_units && kq < n_pub && live) {
      // C fragment: rows g (i = 0, 1) and g + 8 (i = 2, 3), token columns 2c, 2c + 1
      for (int i = kq; i < 4; i += n_pub) {
        float G = 0.f, U = 0.f;
        for (int zz = 0; zz < L.ks; ++zz) {
          const float *zp = red + static_cast<size_t>((warp - kq + zz) * 32 + lane) * 8;
          G += zp[i];
          U += zp[4 + i];
        }
        const int t = 2 * c + (i & 1);
        const int row0 = rb * kRowBlock + (i >> 1) * 8;  // this element's 8-row group; the lane's row is row0 + g
        const bool mine = t < T && ((sh.umask[u] >> t) & 1u);
        const uint32_t hbits = mine ? __half_as_ushort(__float2half_rn(swiglu_scaled(G, U, sh.xexp[t]))) : 0u;
        // K positions 2g and 2g + 1 of the group hold rows g and g + 4 (the
        // operand order), which lanes g and g + 4 of the same column computed
        const uint32_t hi = __shfl_xor_sync(0xffffffffu, hbits, 16);
        if (g < 4 && mine && !(a.test_fault && unit == 0)) {
          const int j = sh.uslot[u][t];
          st_tagged(hb + (static_cast<size_t>(t) * (k + 1) + j) * (Imax / 2) + row0 / 2 + g,
                    (static_cast<uint64_t>(sh.tag) << 32) | (hi << 16) | hbits);
        }
      }
    }
    __syncthreads();
    // the stages this round used are free: refill them with the units nb ahead
    if (warp == 0 && __all_sync(0xffffffffu, *abort == 0))
      for (int zz = 0; zz < units_per_round; ++zz) {
        const int qn = r * units_per_round + zz + L.nb;
        if (qn < my_units) issue_b(qn);
      }
  }

  // ---- down + combine ----------------------------------------------------------------
  // Every CTA counted itself out (exit count) once it had read the launch tag
  // and was past the router-score wait. The last warp of CTA 0 waits
  // (bounded, acquire) for the whole grid's count, clears the two counters and
  // records the tag for the next launch, which no CTA of this one reads any
  // more: off the critical path when that warp has no expert of its own,
  // otherwise after its down products. The tag is recorded even when the wait
  // runs out, so the next launch never reuses it.
  const bool clears = blockIdx.x == 0 && warp == kSTWarps - 1;
  auto clear_counters = [&]() {  // whole warp (CTA 0's last)
    if (wait_count(exit_count, gridDim.x, abort, a.status, 44, 0, budget)) {
      if (lane == kSmallTExitWord || lane == kSmallTRouterWord) a.sync[lane] = 0u;
    }
    if (lane == 0) asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(a.sync + kSmallTEpochWord), "r"(sh.tag)
                                : "memory");
    __syncwarp();
  };
  if (!has_dblk && clears) clear_counters();
  if (has_dblk) {
    const int n0 = blockIdx.x * kRowBlock;
    const uint32_t tag = sh.tag;
    // each warp's share of the token staging area, for the values of h rows
    const size_t h_slice_bytes = (L.red_off / kSTWarps) & ~static_cast<size_t>(15);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};  // rows g, g+8; tokens 2c, 2c+1 (this warp's experts, ascending)
    bool ok2 = __all_sync(0xffffffffu, *abort == 0);
    // Bounded wait of the whole warp, between polls of tagged words: false
    // (recording a timeout with the expert) once the budget is spent or the
    // CTA gave up.
    unsigned long long poll_t0 = 0;
    auto poll_more = [&](int it, int u) {
      if (__any_sync(0xffffffffu, *abort != 0)) return false;
      if (it == 0) poll_t0 = global_ns();
      __nanosleep(32);
      int late = 0;
      if ((it & 15) == 15) late = global_ns() - poll_t0 > budget ? 1 : 0;
      if (__shfl_sync(0xffffffffu, late, 0)) {
        if (lane == 0) {
          *abort = 1;
          report_error(a.status, kDevTimeout, 42, u);
        }
        return false;
      }
      return true;
    };
    // pass p (base p * nd) gives warp w the experts base + w, base + w + 16, ...
    // below min(nU, base + nd): a warp at or past min(nU, nd) has none at all
    bool cleared = false;
    if (warp >= min(nU, L.nd) && clears && nU <= L.nd) {  // one pass: no block barrier ahead that this wait could hold up
      clear_counters();
      cleared = true;
    }
    for (int base = 0; base < nU; base += L.nd) {
      const uint32_t par = (base / L.nd) & 1u;
      if (base > 0) {  // next pass: the ring's stages are free once every warp is done
        __syncthreads();
        if (warp == 0 && __all_sync(0xffffffffu, *abort == 0)) issue_d_range(base, min(nU, base + L.nd));
      }
      for (int u = base + warp; u < min(nU, base + L.nd); u += kSTWarps) {
        if (!ok2) break;
        const int s = u % L.nd;
        int okw = 1;
        if (lane == 0) okw = st_wait(&d_full[s], par, abort, a.status, 41, budget) ? 1 : 0;
        ok2 = __shfl_sync(0xffffffffu, okw, 0) != 0;
        if (!ok2) break;
        const int Iu = u == 0 ? a.Is : a.I;
        const int iw = Iu / 8;  // packed words per down row
        const uint8_t *st = dring + s * L.d_stage;
        const uint32_t *pd = reinterpret_cast<const uint32_t *>(st);
        const int ngd = Iu / kGroup;
        const uint16_t *sd = reinterpret_cast<const uint16_t *>(st + kRowBlock * (Imax / 2));
        const uint16_t *bd = sd + kRowBlock * ngd;
        // B fragments: token g's h for this expert (zeros if g is not routed to
        // it), written as tagged words by other CTAs of this launch and read
        // through L2 until every word carries this launch's tag. Where the
        // warp's share of the token staging area (free once this CTA's gate/up
        // is done) holds the expert's rows for all T tokens, the whole warp
        // polls them together (one round trip once they are there) and keeps
        // the values there; otherwise each lane polls its token's words as the
        // products need them.
        const int jg = (g < T) ? sh.uslot[u][g] : -1;
        const int cpr = Iu / 4;  // word pairs (16 bytes, four values) per row
        const bool staged = static_cast<size_t>(T) * Iu * 2 <= h_slice_bytes && T * cpr <= 32 * kPairsPerLane;
        __half *hw = reinterpret_cast<__half *>(dyn + L.x_off + warp * h_slice_bytes);
        if (staged) {
          const int nch = T * cpr;
          uint32_t pending = 0;  // bit i: pair lane + 32 i is awaited
#pragma unroll
          for (int i = 0; i < kPairsPerLane; ++i) {
            const int idx = lane + 32 * i;
            if (idx < nch && sh.uslot[u][idx / cpr] >= 0) pending |= 1u << i;
          }
          for (int it = 0;; ++it) {
            ulonglong2 v[kPairsPerLane];
#pragma unroll
            for (int i = 0; i < kPairsPerLane; ++i) {
              const int idx = lane + 32 * i, t = idx / cpr, cc = idx - t * cpr;
              if ((pending >> i) & 1u)
                v[i] = ld_tagged2(hb + (static_cast<size_t>(t) * (k + 1) + sh.uslot[u][t]) * (Imax / 2) + 2 * cc);
            }
#pragma unroll
            for (int i = 0; i < kPairsPerLane; ++i) {
              const int idx = lane + 32 * i, t = idx / cpr, cc = idx - t * cpr;
              if (((pending >> i) & 1u) && tag_ok(v[i], tag)) {
                *reinterpret_cast<uint2 *>(hw + t * Iu + 4 * cc) = tagged_values(v[i]);
                pending &= ~(1u << i);
              }
            }
            if (__all_sync(0xffffffffu, pending == 0)) break;
            if (!poll_more(it, u)) {
              ok2 = false;
              break;
            }
          }
          if (!ok2) break;
          __syncwarp();
        }
        const __half *hrow = hw + (g < T ? g : 0) * Iu;  // staged values
        const uint64_t *trow = hb + (static_cast<size_t>(g) * (k + 1) + (jg < 0 ? 0 : jg)) * (Imax / 2);
        float y[4] = {0.f, 0.f, 0.f, 0.f}, y2[4] = {0.f, 0.f, 0.f, 0.f};  // even / odd words
        for (int w0 = 4 * c; w0 < iw; w0 += 16) {  // 16-word blocks; this thread's words w0 .. w0 + 3
          uint4 hv[4];
#pragma unroll
          for (int p = 0; p < 4; ++p)
            hv[p] = (staged && jg >= 0) ? *reinterpret_cast<const uint4 *>(hrow + (w0 + p) * 8) : make_uint4(0, 0, 0, 0);
          if (!staged) {  // the 8 values of word w0 + p are the tagged pairs 2 (w0 + p) and 2 (w0 + p) + 1
            uint32_t pending = jg >= 0 ? 0xffu : 0u;
            for (int it = 0;; ++it) {
              ulonglong2 v[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                if ((pending >> i) & 1u) v[i] = ld_tagged2(trow + 2 * (2 * (w0 + i / 2) + (i & 1)));
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                if (((pending >> i) & 1u) && tag_ok(v[i], tag)) {
                  const uint2 q2 = tagged_values(v[i]);
                  if (i & 1) {
                    hv[i / 2].z = q2.x;
                    hv[i / 2].w = q2.y;
                  } else {
                    hv[i / 2].x = q2.x;
                    hv[i / 2].y = q2.y;
                  }
                  pending &= ~(1u << i);
                }
              }
              if (__all_sync(0xffffffffu, pending == 0)) break;
              if (!poll_more(it, u)) {
                ok2 = false;
                break;
              }
            }
            if (!ok2) break;
          }
          const int grp = w0 / 8;
          const __half2 s0 = bf16_to_half2_bcast(sd[g * ngd + grp]), b0 = bf16_to_half2_bcast(bd[g * ngd + grp]);
          const __half2 s1 = bf16_to_half2_bcast(sd[(g + 8) * ngd + grp]),
                        b1 = bf16_to_half2_bcast(bd[(g + 8) * ngd + grp]);
          const uint4 wd0 = *reinterpret_cast<const uint4 *>(pd + g * iw + w0);
          const uint4 wd1 = *reinterpret_cast<const uint4 *>(pd + (g + 8) * iw + w0);
          const uint32_t ad0[4] = {wd0.x, wd0.y, wd0.z, wd0.w}, ad1[4] = {wd1.x, wd1.y, wd1.z, wd1.w};
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            const uint4 d0 = dequant_word(ad0[p], s0, b0), d1 = dequant_word(ad1[p], s1, b1);
            float(&yy)[4] = (p & 1) ? y2 : y;
            mma16816(yy, d0.x, d1.x, d0.y, d1.y, hv[p].x, hv[p].y);
            mma16816(yy, d0.z, d1.z, d0.w, d1.w, hv[p].z, hv[p].w);
          }
        }
        if (!ok2) break;
        // weight each token's column by its routing weight (1 for the shared expert) and 2^(2e)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int t = 2 * c + (i & 1);
          if (t < T && ((sh.umask[u] >> t) & 1u)) {
            const int j = sh.uslot[u][t];
            const float wgt = (j == k) ? 1.0f : sh.wt[t][j];
            acc[i] += wgt * ldexpf(y[i] + y2[i], 2 * sh.xexp[t]);
          }
        }
      }
    }
    if (clears && !cleared) clear_counters();
    float *rp = red + static_cast<size_t>(threadIdx.x) * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) rp[i] = acc[i];
    __syncthreads();
    // warps' contributions summed in warp order, one rounding; 16 rows x T tokens
    if (warp == 0) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 2 * c + (i & 1);
        const int n = n0 + g + (i >> 1) * 8;
        if (t < T) {
          float o = 0.f;
          for (int zz = 0; zz < kSTWarps; ++zz) o += red[static_cast<size_t>(zz * 32 + lane) * 8 + i];
          if (a.residual) o += bf16_bits_to_float(a.residual[static_cast<size_t>(t) * H + n]);
          a.out[static_cast<size_t>(t) * H + n] = float_to_bf16_bits(o);
        }
      }
    }
  }

  // ---- exit ----------------------------------------------------------------------------
  __syncthreads();
  if (threadIdx.x == 0) {
    // after a wait gave up, copies may still be in flight: they land before the
    // CTA leaves (without one, every issued stage has been waited on)
    if (*abort) {
      drain_ring(b_full, sh.b_iss, L.nb);
      drain_ring(d_full, sh.d_iss, L.nd);
    }
  }
}

cudaError_t launch_small_t(const SmallTArgs &a, int num_sms, cudaStream_t s, bool pdl) {
  const StLayout L = st_layout(a.H, a.I, a.Is, a.T, a.k);
  const size_t smem = L.bytes;
  // the limit is raised to the most any layout takes, once per device
  static std::atomic<uint64_t> smem_set{0};
  cudaError_t err = gemm::ensure_smem_limit(small_t_kernel, static_cast<int>(kStBudget), smem_set);
  if (err != cudaSuccess) return err;
  // cooperative: every CTA resident at once (they wait on one another's
  // SwiGLU outputs); with pdl, also allowed to start while the kernel
  // ahead on the stream finishes
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(small_t_grid(num_sms));
  cfg.blockDim = dim3(kSTThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, small_t_kernel, a);
}

}  // namespace moe
