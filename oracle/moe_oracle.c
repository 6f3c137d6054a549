/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of the routed int4 MoE layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes, and where the pages say so ("Perplexity open sources
 * Lily, a Rust and Metal inference engine for Apple Silicon", section
 * "Requirements and model layout"; the aioga.com record of the same report,
 * article body paragraphs 3 and 4):
 *
 *  - the router scores all experts of a token and picks eight (top_k of E);
 *  - one shared expert sees every token;
 *  - weights are groupwise-affine 4-bit: every group of 64 weights shares one
 *    bfloat16 scale and one bfloat16 bias, w = q * scale + bias, q in 0..15.
 *
 * Readings taken where the pages are silent (each one listed in the design
 * notes of the repository):
 *
 *  - router: p = softmax(logits) over all E experts (fp64, max-subtracted);
 *    the k experts are chosen by comparing the raw float32 logits, largest
 *    first, equal logits going to the lower expert id; their probabilities
 *    are renormalised to sum to one;
 *  - expert MLP: SwiGLU, y = W_down (silu(W_gate x) * (W_up x)), with
 *    silu(z) = z / (1 + exp(-z));
 *  - shared expert: weight 1, no gate;
 *  - out_t = sum_{j=0}^{k-1} w_{t,j} y_{ids[t,j]}(x_t) + y_shared(x_t),
 *    accumulated in fp64 in that order, with no intermediate rounding;
 *  - layout: per expert [gate I x H | up I x H | down H x I], rows with K
 *    contiguous, 8 codes per uint32 with element 8w+j in bits 4j..4j+3;
 *    scale/bias group g of a row covers K in [64g, 64g+64);
 *  - expert offsets and the permutation: experts in ascending order, and
 *    within one expert the (token, slot) pairs in ascending token order;
 *    perm holds the flat index t*k + j.
 *
 * Every function is written for a reader to check by eye, not for speed.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_GROUP 64

/* bfloat16 bit pattern -> exact double */
double oracle_bf16_value(uint16_t bits) {
  uint32_t u = (uint32_t)bits << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* 4-bit code of element kk of a row stored as K/8 words, low nibble first */
int oracle_code(const uint32_t *row_words, int kk) {
  return (int)((row_words[kk / 8] >> (4 * (kk % 8))) & 0xFu);
}

/* weight (n, kk) of an N x K matrix: q * scale + bias in fp64 */
double oracle_weight(const uint32_t *words, const uint16_t *scales,
                     const uint16_t *biases, int K, int n, int kk) {
  const uint32_t *row = words + (size_t)n * (K / 8);
  size_t g = (size_t)n * (K / ORACLE_GROUP) + (size_t)(kk / ORACLE_GROUP);
  double q = (double)oracle_code(row, kk);
  return q * oracle_bf16_value(scales[g]) + oracle_bf16_value(biases[g]);
}

/* dequantise a whole N x K matrix into out[N*K] (fp64); rows in parallel */
void oracle_dequant_matrix(const uint32_t *words, const uint16_t *scales,
                           const uint16_t *biases, int N, int K, double *out) {
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int n = 0; n < N; ++n)
    for (int kk = 0; kk < K; ++kk)
      out[(size_t)n * K + kk] = oracle_weight(words, scales, biases, K, n, kk);
}

/*
 * Router for T tokens over E experts, top k.
 *   ids [T*k]   chosen experts, largest logit first (ties: lower id first)
 *   w   [T*k]   renormalised softmax probabilities of the chosen experts
 *   counts [E]  number of (token, slot) pairs per expert
 *   offsets [E+1] exclusive prefix sum of counts
 *   perm [T*k]  flat indices t*k+j sorted by (expert, token)
 * Any output pointer may be NULL. Returns 0, or -1 on bad sizes.
 */
int oracle_route(int T, int E, int k, const float *logits, int32_t *ids,
                 double *w, int32_t *counts, int32_t *offsets, int32_t *perm) {
  if (T < 0 || E <= 0 || k <= 0 || k > E) return -1;
  int32_t *sel = (int32_t *)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1) * k);
  double *wt = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * k);
  char *taken = (char *)malloc((size_t)E);
  double *p = (double *)malloc(sizeof(double) * (size_t)E);
  if (!sel || !wt || !taken || !p) {
    free(sel); free(wt); free(taken); free(p);
    return -1;
  }
  for (int t = 0; t < T; ++t) {
    const float *l = logits + (size_t)t * E;
    /* softmax over all E experts in fp64 */
    double m = (double)l[0];
    for (int e = 1; e < E; ++e)
      if ((double)l[e] > m) m = (double)l[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp((double)l[e] - m);
      z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= z;
    /* top-k by the float32 logits: repeated selection of the largest
       remaining one, scanning ids upwards so equal values keep the lower id */
    memset(taken, 0, (size_t)E);
    double psum = 0.0;
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        if (best < 0 || l[e] > l[best]) best = e;
      }
      taken[best] = 1;
      sel[(size_t)t * k + j] = best;
      psum += p[best];
    }
    /* renormalise the k chosen probabilities to sum to one */
    for (int j = 0; j < k; ++j)
      wt[(size_t)t * k + j] = p[sel[(size_t)t * k + j]] / psum;
  }
  if (ids) memcpy(ids, sel, sizeof(int32_t) * (size_t)T * k);
  if (w) memcpy(w, wt, sizeof(double) * (size_t)T * k);
  if (counts || offsets || perm) {
    int32_t *cnt = (int32_t *)calloc((size_t)E, sizeof(int32_t));
    int32_t *off = (int32_t *)calloc((size_t)E + 1, sizeof(int32_t));
    if (!cnt || !off) {
      free(cnt); free(off); free(sel); free(wt); free(taken); free(p);
      return -1;
    }
    /* histogram */
    for (size_t i = 0; i < (size_t)T * k; ++i) cnt[sel[i]] += 1;
    /* exclusive prefix sum */
    off[0] = 0;
    for (int e = 0; e < E; ++e) off[e + 1] = off[e] + cnt[e];
    /* stable scatter: experts ascending, tokens ascending within an expert */
    if (perm) {
      int32_t pos = 0;
      for (int e = 0; e < E; ++e)
        for (int t = 0; t < T; ++t)
          for (int j = 0; j < k; ++j)
            if (sel[(size_t)t * k + j] == e) perm[pos++] = t * k + j;
    }
    if (counts) memcpy(counts, cnt, sizeof(int32_t) * (size_t)E);
    if (offsets) memcpy(offsets, off, sizeof(int32_t) * ((size_t)E + 1));
    free(cnt);
    free(off);
  }
  free(sel); free(wt); free(taken); free(p);
  return 0;
}

/*
 * Router scores ("Perplexity open sources Lily...", section "Requirements and
 * model layout": the router scores every expert of a token):
 *   logits[t*E + e] = sum_h x[t, h] * w[e, h], in fp64 from the bfloat16 bit
 * patterns of x [T, H] and the router weight w [E, H] (rows K-contiguous).
 */
void oracle_router_logits(int T, int E, int H, const uint16_t *x_bf16, const uint16_t *w_bf16,
                          double *logits) {
#ifdef _OPENMP
#pragma omp parallel for schedule(static)
#endif
  for (int t = 0; t < T; ++t)
    for (int e = 0; e < E; ++e) {
      double acc = 0.0;
      for (int h = 0; h < H; ++h)
        acc += oracle_bf16_value(x_bf16[(size_t)t * H + h]) * oracle_bf16_value(w_bf16[(size_t)e * H + h]);
      logits[(size_t)t * E + e] = acc;
    }
}

/*
 * One SwiGLU expert on one token, fp64 throughout.
 *   words/scales/biases: the expert's three matrices in the packed layout
 *   x [H] input, y [H] output, a [I] scratch.
 */
void oracle_expert(int H, int I, const uint32_t *words, const uint16_t *scales,
                   const uint16_t *biases, const double *x, double *y, double *a) {
  const uint32_t *wg = words;
  const uint32_t *wu = words + (size_t)I * H / 8;
  const uint32_t *wd = words + (size_t)2 * I * H / 8;
  const uint16_t *sg = scales, *su = scales + (size_t)I * H / ORACLE_GROUP;
  const uint16_t *sd = scales + (size_t)2 * I * H / ORACLE_GROUP;
  const uint16_t *bg = biases, *bu = biases + (size_t)I * H / ORACLE_GROUP;
  const uint16_t *bd = biases + (size_t)2 * I * H / ORACLE_GROUP;
  for (int i = 0; i < I; ++i) {
    double g = 0.0, u = 0.0;
    for (int h = 0; h < H; ++h) {
      g += oracle_weight(wg, sg, bg, H, i, h) * x[h];
      u += oracle_weight(wu, su, bu, H, i, h) * x[h];
    }
    a[i] = g / (1.0 + exp(-g)) * u; /* silu(gate) * up */
  }
  for (int n = 0; n < H; ++n) {
    double acc = 0.0;
    for (int i = 0; i < I; ++i) acc += oracle_weight(wd, sd, bd, I, n, i) * a[i];
    y[n] = acc;
  }
}

/*
 * The whole layer for T tokens. x_bf16 [T,H] bfloat16 bits, logits [T,E],
 * packed [E][3*I*H/8], scales/biases [E][3*I*H/64], sh_* the shared expert
 * with intermediate Is. out [T,H] fp64. nthreads <= 0 uses the OpenMP default.
 * Returns 0, or -1 on bad sizes or allocation failure.
 */
int oracle_moe_forward(int T, int H, int E, int k, int I, int Is,
                       const uint16_t *x_bf16, const float *logits,
                       const uint32_t *packed, const uint16_t *scales,
                       const uint16_t *biases, const uint32_t *sh_packed,
                       const uint16_t *sh_scales, const uint16_t *sh_biases,
                       double *out, int nthreads) {
  if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E || I <= 0 || Is <= 0) return -1;
  if (H % ORACLE_GROUP || I % ORACLE_GROUP || Is % ORACLE_GROUP) return -1;
  if (T == 0) return 0;
  int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)T * k);
  double *w = (double *)malloc(sizeof(double) * (size_t)T * k);
  if (!ids || !w) { free(ids); free(w); return -1; }
  if (oracle_route(T, E, k, logits, ids, w, NULL, NULL, NULL)) {
    free(ids); free(w);
    return -1;
  }
  const size_t wpe = (size_t)3 * I * H / 8, gpe = (size_t)3 * I * H / ORACLE_GROUP;
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
  {
    int imax = I > Is ? I : Is;
    double *xd = (double *)malloc(sizeof(double) * (size_t)H);
    double *y = (double *)malloc(sizeof(double) * (size_t)H);
    double *a = (double *)malloc(sizeof(double) * (size_t)imax);
    if (!xd || !y || !a) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      failed = 1;
    }
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int t = 0; t < T; ++t) {
      if (!xd || !y || !a) continue;
      double *o = out + (size_t)t * H;
      for (int h = 0; h < H; ++h) {
        xd[h] = oracle_bf16_value(x_bf16[(size_t)t * H + h]);
        o[h] = 0.0;
      }
      for (int j = 0; j < k; ++j) {
        int e = ids[(size_t)t * k + j];
        oracle_expert(H, I, packed + (size_t)e * wpe, scales + (size_t)e * gpe,
                      biases + (size_t)e * gpe, xd, y, a);
        double wj = w[(size_t)t * k + j];
        for (int h = 0; h < H; ++h) o[h] += wj * y[h];
      }
      oracle_expert(H, Is, sh_packed, sh_scales, sh_biases, xd, y, a);
      for (int h = 0; h < H; ++h) o[h] += y[h]; /* shared expert, weight 1 */
    }
    free(xd); free(y); free(a);
  }
  free(ids); free(w);
  return failed ? -1 : 0;
}

/* number of threads the OpenMP runtime would use (1 without OpenMP) */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
