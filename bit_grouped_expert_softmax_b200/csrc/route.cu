// route.cu -- routing on the device, one stream, no host synchronisation.
//
// The report lists the routing histogram, prefix scan, scatter and block map
// as work kept inside one GPU command buffer (aioga.com record, article body
// paragraph 5); the router itself scores every expert and keeps the top k
// ("Perplexity open sources Lily...", section "Requirements and model layout").
// Four kernels:
//   route_topk_kernel    softmax over E, warp top-k, renormalised weights,
//                        per-chunk expert histogram
//   route_scan_kernel    per-expert totals and per-chunk prefixes (one warp per
//                        expert)
//   route_scatter_kernel the exclusive scan of the totals (offsets) and the
//                        grouped-GEMM work lists (block map), each block
//                        computing the scan itself and writing its share of
//                        the lists; the stable permutation (experts
//                        ascending, tokens ascending within an expert) and its
//                        inverse
//   gather_kernel        each token's row, fp16 scaled by a power of two, copied
//                        to its k routed rows and its shared-expert row (expert-
//                        contiguous, the gate/up GEMM's activation operand), and
//                        the per-row exponents and weights the epilogues use
#include "kernels.cuh"
#include "topk.cuh"

namespace moe {

__global__ void __launch_bounds__(256) route_topk_kernel(int T, int E, int k, int chunk,
                                                         const float *__restrict__ logits,
                                                         int32_t *__restrict__ ids,
                                                         float *__restrict__ wts,
                                                         int32_t *__restrict__ chunk_cnt) {
  // one warp per token; the per-chunk expert histogram is built with integer
  // atomics (order-independent) into chunk_cnt, which starts zeroed
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= T) return;
  int id;
  float w;
  warp_topk(logits + static_cast<size_t>(t) * E, E, k, lane, id, w);
  if (lane < k) {
    ids[static_cast<size_t>(t) * k + lane] = id;
    wts[static_cast<size_t>(t) * k + lane] = w;
    atomicAdd(&chunk_cnt[static_cast<size_t>(t / chunk) * E + id], 1);
  }
}

// One warp per expert (8 per block). Each warp turns its expert's column of
// per-chunk counts into exclusive prefix sums over the chunks (in place: the
// rows each chunk's first entry lands at, relative to the expert's first row)
// and leaves the expert's total in totals[e].
__global__ void __launch_bounds__(256) route_scan_kernel(RouteScanArgs a) {
  pdl_wait();
  pdl_trigger();
  const int E = a.E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  if (e >= E) return;
  int run = 0;
  for (int c0 = 0; c0 < a.nchunk; c0 += 128) {
    int v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // four loads in flight per lane
      const int c = c0 + 32 * u + lane;
      v[u] = c < a.nchunk ? __ldcg(a.chunk_cnt + static_cast<size_t>(c) * E + e) : 0;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + 32 * u + lane;
      const int incl = warp_incl_scan(v[u]);
      if (c < a.nchunk) a.chunk_cnt[static_cast<size_t>(c) * E + e] = run + incl - v[u];
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (lane == 0) a.totals[e] = run;
}

// Stable scatter and the block map. One block per routing chunk of 32 tokens.
// Every block scans the experts' totals into their first rows (offsets) and
// the groups' work-item counts into list positions itself (257 values, in
// shared memory: no block waits for another); block 0 stores the offsets and
// the item counts, and each block writes the work items of every
// gridDim.x-th group. Warp 0 then ranks the chunk's entries; the chunk's row
// of bases is reset to zero afterwards, ready for the next routing's
// histogram. Work items of group g are (n-tile, m-block) with the m-block
// fastest, so neighbouring CTAs share the activation tile of one n-tile.
__global__ void __launch_bounds__(256) route_scatter_kernel(RouteScatterArgs a) {
  __shared__ int cnt[kMaxExperts];
  __shared__ int sid[kRouteChunk * kMaxTopK];  // the chunk's expert ids, flat order
  __shared__ int tot[kMaxExperts + 1];
  __shared__ int off[kMaxExperts + 2], gu_off[kMaxExperts + 2], dn_off[kMaxExperts + 2];
  __shared__ int totals3[3];
  pdl_wait();
  pdl_trigger();
  const int chunk = blockIdx.x, E = a.E, k = a.k, T = a.T;
  const int G = E + 1;  // routed experts plus the shared one
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t *row = a.chunk_base + static_cast<size_t>(chunk) * E;
  const int t0 = chunk * a.chunk, t1 = min(T, t0 + a.chunk);
  const int f0 = t0 * k, f1 = t1 * k;
  // the experts' totals, the chunk's per-expert prefix and the chunk's ids,
  // all loaded by the whole block at once
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    tot[e] = __ldcg(a.totals + e);
    cnt[e] = __ldcg(row + e);
  }
  for (int f = f0 + threadIdx.x; f < f1; f += blockDim.x) sid[f - f0] = a.ids[f];
  __syncthreads();
  // exclusive scans over the groups, done by warp 0 with 9 values per lane (G <= 257)
  if (warp == 0) {
    constexpr int PER = (kMaxExperts + 1 + 31) / 32;
    int c3[PER], gu[PER], dn[PER];
    int sc = 0, sg = 0, sd = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int g = lane * PER + i;
      int n = 0, gi = 0, di = 0;
      if (g < G) {
        n = (g < E) ? tot[g] : T;
        gi = ((n + a.gu_tile - 1) / a.gu_tile) * ((g < E ? a.I : a.Is) / kGuTileM);
        di = ((n + kTileN - 1) / kTileN) * (a.H / kTileM);
      }
      c3[i] = (g < E) ? n : 0;
      gu[i] = gi;
      dn[i] = di;
      sc += c3[i];
      sg += gi;
      sd += di;
    }
    const int ic = warp_incl_scan(sc), ig = warp_incl_scan(sg), id = warp_incl_scan(sd);
    int bc = ic - sc, bg = ig - sg, bd = id - sd;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int g = lane * PER + i;
      if (g <= G) {
        off[g] = bc;
        gu_off[g] = bg;
        dn_off[g] = bd;
      }
      bc += c3[i];
      bg += gu[i];
      bd += dn[i];
    }
    if (lane == 31) {
      totals3[0] = ic;
      totals3[1] = ig;
      totals3[2] = id;
    }
  }
  __syncthreads();
  // the chunk's first row of each expert: the expert's offset plus the
  // entries of earlier chunks (the scan's per-chunk prefix)
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    cnt[e] += off[e];
    row[e] = 0;
  }
  const int R = T * k;
  if (blockIdx.x == 0) {
    for (int g = threadIdx.x; g <= E; g += blockDim.x) a.offsets[g] = (g < E) ? off[g] : R;
    if (threadIdx.x == 0) {
      const int gu_total = totals3[1], dn_total = totals3[2];
      if (gu_total > a.max_gu || dn_total > a.max_dn)
        report_error(a.status, kDevBounds, 10, static_cast<uint32_t>(max(gu_total, dn_total)));
      a.item_counts[0] = min(gu_total, a.max_gu);
      a.item_counts[1] = min(dn_total, a.max_dn);
    }
  }
  __syncthreads();
  if (warp != 0) {
    // work items: warps 1..7 of block b take groups b + gridDim.x * j. The
    // (n-tile, m-block) of item i is (i / m, i % m); lane l starts at item l
    // and steps by 32 items, carrying quotient and remainder along.
    for (int g = blockIdx.x + gridDim.x * (warp - 1); g < G; g += gridDim.x * ((blockDim.x >> 5) - 1)) {
      const int n = (g < E) ? tot[g] : T;
      const int row0 = (g < E) ? off[g] : R;
      const int ntg = (n + a.gu_tile - 1) / a.gu_tile, ntile = (n + kTileN - 1) / kTileN;
      const int mg = (g < E ? a.I : a.Is) / kGuTileM, md = a.H / kTileM;
      {
        int nt = lane / mg, mb = lane % mg;
        const int qs = 32 / mg, rs = 32 % mg;
        for (int i = lane; i < ntg * mg; i += 32) {
          const int slot = gu_off[g] + i;
          if (slot < a.max_gu)
            a.gu_items[slot] = WorkItem{g, row0 + nt * a.gu_tile, min(a.gu_tile, n - nt * a.gu_tile), mb};
          nt += qs;
          mb += rs;
          if (mb >= mg) {
            mb -= mg;
            ++nt;
          }
        }
      }
      {
        int nt = lane / md, mb = lane % md;
        const int qs = 32 / md, rs = 32 % md;
        for (int i = lane; i < ntile * md; i += 32) {
          const int slot = dn_off[g] + i;
          if (slot < a.max_dn) a.dn_items[slot] = WorkItem{g, row0 + nt * kTileN, min(kTileN, n - nt * kTileN), mb};
          nt += qs;
          mb += rs;
          if (mb >= md) {
            mb -= md;
            ++nt;
          }
        }
      }
    }
    return;
  }
  // flat order f = t*k + j is token-ascending; within a batch of 32 entries the
  // rank among equal experts comes from match/popc, across batches from cnt[]
  for (int fb = f0; fb < f1; fb += 32) {
    const int f = fb + lane;
    const bool valid = f < f1;
    const unsigned active = __ballot_sync(0xffffffffu, valid);
    if (valid) {
      const int e = sid[f - f0];
      const unsigned peers = __match_any_sync(active, e);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      const int base = cnt[e];
      __syncwarp(active);
      if (rank == 0) cnt[e] = base + __popc(peers);
      const int pos = base + rank;
      if (pos < 0 || pos >= T * k) {
        report_error(a.status, kDevBounds, 20, static_cast<uint32_t>(pos));
      } else {
        a.perm[pos] = f;
        a.inv[f] = pos;
        a.row_w[pos] = a.wts[f];
      }
    }
    __syncwarp();
  }
}

// Gather: one warp per token. The row is scaled by a power of two 2^-e chosen
// from its max |x| (exact in fp16 unless the row spans more than fp16's
// range), converted to fp16 and written, in the K-permuted operand order, to
// the token's k routed rows (positions from the scatter) and its shared-expert
// row R + t. (Gathering the GEMM's operand rows from one compact fp16 row per
// token instead, by TMA tile::gather4 or by cp.async, made the gate/up GEMM
// 1.6-2x slower at T = 4096.)
__global__ void __launch_bounds__(256) gather_kernel(RouteScatterArgs a) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + warp;
  if (t >= a.T) return;
  const int H = a.H, k = a.k, R = a.T * k;
  __shared__ int srows[8][kMaxTopK];  // each warp's token's routed rows
  int *rows = srows[warp];
  if (lane < k) rows[lane] = a.inv[static_cast<size_t>(t) * k + lane];
  __syncwarp();
  const uint4 *src = reinterpret_cast<const uint4 *>(a.x + static_cast<size_t>(t) * H);
  const int nchunk8 = H / 8;
  // the first 256 chunks (H <= 2048: the whole row) are loaded at once and
  // kept in registers for the conversion; the rest are read twice
  constexpr int kHeld = 8;
  uint4 held[kHeld];
#pragma unroll
  for (int i = 0; i < kHeld; ++i) {
    const int c = lane + 32 * i;
    held[i] = c < nchunk8 ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
  }
  auto absmax8 = [](uint4 v, float m) {
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      m = fmaxf(m, fabsf(__uint_as_float(w4[q] << 16)));
      m = fmaxf(m, fabsf(__uint_as_float(w4[q] & 0xffff0000u)));
    }
    return m;
  };
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < kHeld; ++i) amax = absmax8(held[i], amax);
  for (int c = lane + 32 * kHeld; c < nchunk8; c += 32) amax = absmax8(__ldg(src + c), amax);
  amax = warp_max(amax);
  int ex = 0;
  if (amax > 0.f && amax <= 3.0e38f) ex = min(max(ilogbf(amax) - 1, -100), 100);  // scaled max in [2, 4)
  const float scale = exp2f(static_cast<float>(-ex));
  if (lane == 0) a.xexp[t] = ex;
  // per-row epilogue factors of the token's k + 1 rows
  if (lane < k && rows[lane] >= 0 && rows[lane] < R) a.row_exp[rows[lane]] = ex;
  if (lane == 0) {
    a.row_exp[R + t] = ex;
    a.row_w[R + t] = 1.0f;
  }
  auto to_fp16 = [&](uint4 v) {
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
    for (int s = 0; s < 8; s += 2) op[s / 2] = pack_half2(hv[kperm_src(s)], hv[kperm_src(s + 1)]);
    return o;
  };
  // each converted chunk goes to the token's k routed rows and its shared row
  auto put = [&](int c, uint4 o) {
    for (int j = 0; j < k; ++j) {
      const int row = rows[j];
      if (row >= 0 && row < R) reinterpret_cast<uint4 *>(a.xt + static_cast<size_t>(row) * H)[c] = o;
    }
    reinterpret_cast<uint4 *>(a.xt + static_cast<size_t>(R + t) * H)[c] = o;
  };
#pragma unroll
  for (int i = 0; i < kHeld; ++i) {
    const int c = lane + 32 * i;
    if (c < nchunk8) put(c, to_fp16(held[i]));
  }
  for (int c = lane + 32 * kHeld; c < nchunk8; c += 32) put(c, to_fp16(__ldg(src + c)));
}

}  // namespace moe
