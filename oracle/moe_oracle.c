/*
 * moe_oracle.c -- fp64 CPU oracle for the decode pass of one Mixture-of-Experts
 * block.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, obviously-correct
 * reference that the CUDA library is checked against.  Only the tests, the
 * smoke check and the CPU-baseline leg of the benchmark load it; the library
 * (moe_decode_block_b200) never links, imports or calls it, and the two share
 * no code, header, table or helper.
 *
 * Source.  The pages ("Hyper Optimizing Kimi K3 in vLLM: Moving Fast and
 * Responsibly", commentary, section "Recovering time between operators"; and
 * "vLLM Hyper-Optimizes Kimi K3 on NVIDIA GB300", section "What's Optimized")
 * name the steps of the block -- router scores, selected experts, a shared
 * expert that runs beside them, residual processing -- but print no formula.
 * This file takes the plainest standard reading of those steps:
 *
 *   for every token b, independently:
 *   1. logit[e] = sum_h x[b,h] * R[h,e]  (+ bias[e] when a bias is given)
 *   2. p = softmax(logit) over all E experts
 *   3. S = the k experts with the largest logits, ordered by logit
 *      descending; equal logits go to the smaller expert id first
 *   4. w_j = p[S_j] / sum_{i in S} p[i]                (renormalised top-k)
 *   5. for j < k: g = x_b . W13[S_j][:, 0:I], u = x_b . W13[S_j][:, I:2I],
 *      a = silu(g) * u with silu(z) = z / (1 + exp(-z)), y_j = a . W2[S_j]
 *   6. s = (silu(x_b . Ws13[:, 0:Is]) * (x_b . Ws13[:, Is:2Is])) . Ws2
 *   7. out_b = x_b + sum_j w_j y_j + s       (shared expert weight is 1)
 *
 * Layouts: x [B,H], R [H,E], W13[e] [H,2I], W2[e] [I,H], Ws13 [H,2Is],
 * Ws2 [Is,H]; all row-major bf16 given as raw 16-bit patterns, widened
 * exactly to fp64.  All arithmetic is fp64.  Every output element is summed
 * in index order by a single thread, so results do not depend on the number
 * of OpenMP threads.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG (-1)
#define ORACLE_MISSING_EXPERT (-2)
#define ORACLE_NO_MEMORY (-3)

/* bf16 -> fp64: a bf16 value is the top 16 bits of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t bits) {
  uint32_t u = ((uint32_t)bits) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* y[c] = sum_{r < nrows} v[r] * W[r, col0 + c] for c < ncols, with W a
 * row-major bf16 matrix of leading dimension ld.  Columns are split across
 * threads; each y[c] is accumulated in r order by one thread. */
static void vec_times_matrix(const double* v, const uint16_t* W, int nrows,
                             int ld, int col0, int ncols, double* y) {
  const int blk = 64;
  const int nblk = (ncols + blk - 1) / blk;
#pragma omp parallel for schedule(static)
  for (int ib = 0; ib < nblk; ++ib) {
    const int c0 = ib * blk;
    const int c1 = (c0 + blk < ncols) ? c0 + blk : ncols;
    double acc[64];
    for (int c = c0; c < c1; ++c) acc[c - c0] = 0.0;
    for (int r = 0; r < nrows; ++r) {
      const double vr = v[r];
      const uint16_t* row = W + (size_t)r * (size_t)ld + (size_t)col0;
      for (int c = c0; c < c1; ++c) acc[c - c0] += vr * bf16_bits_to_double(row[c]);
    }
    for (int c = c0; c < c1; ++c) y[c] = acc[c - c0];
  }
}

static double silu(double z) { return z / (1.0 + exp(-z)); }

/* Steps 5/6 for one token and one expert: y = (silu(g) * u) . W2. */
static void swiglu_mlp(const double* xb, const uint16_t* W13, const uint16_t* W2,
                       int H, int I, double* gu, double* a, double* y) {
  vec_times_matrix(xb, W13, H, 2 * I, 0, 2 * I, gu);
  for (int c = 0; c < I; ++c) a[c] = silu(gu[c]) * gu[I + c];
  vec_times_matrix(a, W2, I, H, 0, H, y);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* Steps 1-4.  logits [B,E] (bias included), ids [B,k], w [B,k]. */
int oracle_router(const uint16_t* x, const uint16_t* router_w, const float* bias,
                  int B, int H, int E, int k, double* logits, int32_t* ids,
                  double* w) {
  if (B < 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return ORACLE_BAD_ARG;
  if (B == 0) return ORACLE_OK;
  if (!x || !router_w || !logits || !ids || !w) return ORACLE_BAD_ARG;
  double* xb = (double*)malloc(sizeof(double) * (size_t)H);
  double* p = (double*)malloc(sizeof(double) * (size_t)E);
  char* taken = (char*)malloc((size_t)E);
  if (!xb || !p || !taken) {
    free(xb); free(p); free(taken);
    return ORACLE_NO_MEMORY;
  }
  for (int b = 0; b < B; ++b) {
    double* lg = logits + (size_t)b * E;
    for (int h = 0; h < H; ++h) xb[h] = bf16_bits_to_double(x[(size_t)b * H + h]);
    vec_times_matrix(xb, router_w, H, E, 0, E, lg);                 /* step 1 */
    if (bias)
      for (int e = 0; e < E; ++e) lg[e] += (double)bias[e];
    double m = lg[0];                                                /* step 2 */
    for (int e = 1; e < E; ++e) m = lg[e] > m ? lg[e] : m;
    double z = 0.0;
    for (int e = 0; e < E; ++e) {
      p[e] = exp(lg[e] - m);
      z += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= z;
    memset(taken, 0, (size_t)E);                                     /* step 3 */
    for (int j = 0; j < k; ++j) {
      int best = -1;
      for (int e = 0; e < E; ++e) {
        if (taken[e]) continue;
        /* strict '>' while e ascends keeps the smaller id on equal logits */
        if (best < 0 || lg[e] > lg[best]) best = e;
      }
      taken[best] = 1;
      ids[(size_t)b * k + j] = best;
    }
    double ps = 0.0;                                                 /* step 4 */
    for (int j = 0; j < k; ++j) ps += p[ids[(size_t)b * k + j]];
    for (int j = 0; j < k; ++j)
      w[(size_t)b * k + j] = p[ids[(size_t)b * k + j]] / ps;
  }
  free(xb); free(p); free(taken);
  return ORACLE_OK;
}

/* Steps 5-7 for a given routing (ids, w).  w13/w2 are arrays of E host
 * pointers; only the selected experts are dereferenced and a NULL selected
 * expert returns ORACLE_MISSING_EXPERT.  n_shared is 0 or 1. */
int oracle_block(const uint16_t* x, const int32_t* ids, const double* w,
                 const uint16_t* const* w13, const uint16_t* const* w2,
                 const uint16_t* sw13, const uint16_t* sw2, int B, int H, int E,
                 int k, int I, int Is, int n_shared, double* out) {
  if (B < 0 || H <= 0 || E <= 0 || k < 0 || k > E || I <= 0) return ORACLE_BAD_ARG;
  if (n_shared != 0 && n_shared != 1) return ORACLE_BAD_ARG;
  if (B == 0) return ORACLE_OK;
  if (!x || !out || (k > 0 && (!ids || !w || !w13 || !w2))) return ORACLE_BAD_ARG;
  if (n_shared && (!sw13 || !sw2 || Is <= 0)) return ORACLE_BAD_ARG;
  const int imax = (n_shared && Is > I) ? Is : I;
  double* xb = (double*)malloc(sizeof(double) * (size_t)H);
  double* gu = (double*)malloc(sizeof(double) * 2 * (size_t)imax);
  double* a = (double*)malloc(sizeof(double) * (size_t)imax);
  double* y = (double*)malloc(sizeof(double) * (size_t)H);
  int rc = ORACLE_OK;
  if (!xb || !gu || !a || !y) {
    rc = ORACLE_NO_MEMORY;
    goto done;
  }
  for (int b = 0; b < B; ++b) {
    double* ob = out + (size_t)b * H;
    for (int h = 0; h < H; ++h) {
      xb[h] = bf16_bits_to_double(x[(size_t)b * H + h]);
      ob[h] = xb[h];                                          /* residual */
    }
    for (int j = 0; j < k; ++j) {                                    /* step 5 */
      const int e = ids[(size_t)b * k + j];
      if (e < 0 || e >= E) { rc = ORACLE_BAD_ARG; goto done; }
      if (!w13[e] || !w2[e]) { rc = ORACLE_MISSING_EXPERT; goto done; }
      swiglu_mlp(xb, w13[e], w2[e], H, I, gu, a, y);
      const double wj = w[(size_t)b * k + j];
      for (int h = 0; h < H; ++h) ob[h] += wj * y[h];
    }
    if (n_shared) {                                                  /* step 6 */
      swiglu_mlp(xb, sw13, sw2, H, Is, gu, a, y);
      for (int h = 0; h < H; ++h) ob[h] += y[h];                     /* step 7 */
    }
  }
done:
  free(xb); free(gu); free(a); free(y);
  return rc;
}

/* Step 5 (or 6) for one expert and a list of tokens, the building block of
 * the expert-at-a-time driver: y[i, :] = (silu(g) * u) . W2 for token
 * rows[i] of x, with W13 [H,2I], W2 [I,H] that expert's weights. */
int oracle_expert_outputs(const uint16_t* x, int B, int H, const uint16_t* W13,
                          const uint16_t* W2, int I, int n, const int32_t* rows,
                          double* y) {
  if (B < 0 || H <= 0 || I <= 0 || n < 0) return ORACLE_BAD_ARG;
  if (n == 0) return ORACLE_OK;
  if (!x || !W13 || !W2 || !rows || !y) return ORACLE_BAD_ARG;
  double* xb = (double*)malloc(sizeof(double) * (size_t)H);
  double* gu = (double*)malloc(sizeof(double) * 2 * (size_t)I);
  double* a = (double*)malloc(sizeof(double) * (size_t)I);
  int rc = ORACLE_OK;
  if (!xb || !gu || !a) {
    rc = ORACLE_NO_MEMORY;
    goto done;
  }
  for (int i = 0; i < n; ++i) {
    const int b = rows[i];
    if (b < 0 || b >= B) { rc = ORACLE_BAD_ARG; goto done; }
    for (int h = 0; h < H; ++h) xb[h] = bf16_bits_to_double(x[(size_t)b * H + h]);
    swiglu_mlp(xb, W13, W2, H, I, gu, a, y + (size_t)i * H);
  }
done:
  free(xb); free(gu); free(a);
  return rc;
}

/* ---- FP8 expert weights (an extension the pages do not cover) ----------
 * Weights stored as 8-bit e4m3 codes (1 sign bit, 4 exponent bits with bias
 * 7, 3 mantissa bits; exponent 0 is subnormal: m / 8 * 2^-6; the all-ones
 * code is NaN, there is no infinity) in [out, in] layout, with one fp32 scale
 * per block of 128 outputs x 128 inputs, scales row-major over
 * [ceil(out / 128), ceil(in / 128)].  The weight of (output o, input i) is
 * decode(q[o, i]) * scale[o / 128, i / 128], in fp64. */
static double e4m3_to_double(uint8_t q) {
  const int s = q >> 7, e = (q >> 3) & 15, m = q & 7;
  if (e == 15 && m == 7) return NAN;
  const double v = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return s ? -v : v;
}

double oracle_e4m3_value(uint8_t q) { return e4m3_to_double(q); }

/* y[o] = sum_i v[i] * W[o, i] for o < nout, W the block-scaled e4m3 matrix
 * [nout, nin] (row o contiguous); each y[o] is summed in i order by one
 * thread. */
static void vec_times_fp8(const double* v, const uint8_t* q, const float* sc, int nout, int nin, double* y) {
  const int nb = (nin + 127) / 128;
#pragma omp parallel for schedule(static)
  for (int o = 0; o < nout; ++o) {
    const uint8_t* row = q + (size_t)o * nin;
    const float* srow = sc + (size_t)(o / 128) * nb;
    double acc = 0.0;
    for (int i = 0; i < nin; ++i) acc += v[i] * (e4m3_to_double(row[i]) * (double)srow[i / 128]);
    y[o] = acc;
  }
}

/* Step 5 for one expert with e4m3 weights: q13 [2I, H] (outputs 0..I-1 the
 * gate, I..2I-1 the up projection) with scales s13, q2 [H, I] with scales
 * s2; y[i, :] for token rows[i] of x. */
int oracle_expert_outputs_fp8(const uint16_t* x, int B, int H, const uint8_t* q13, const float* s13,
                              const uint8_t* q2, const float* s2, int I, int n, const int32_t* rows,
                              double* y) {
  if (B < 0 || H <= 0 || I <= 0 || n < 0) return ORACLE_BAD_ARG;
  if (n == 0) return ORACLE_OK;
  if (!x || !q13 || !s13 || !q2 || !s2 || !rows || !y) return ORACLE_BAD_ARG;
  double* xb = (double*)malloc(sizeof(double) * (size_t)H);
  double* gu = (double*)malloc(sizeof(double) * 2 * (size_t)I);
  double* a = (double*)malloc(sizeof(double) * (size_t)I);
  int rc = ORACLE_OK;
  if (!xb || !gu || !a) {
    rc = ORACLE_NO_MEMORY;
    goto done;
  }
  for (int i = 0; i < n; ++i) {
    const int b = rows[i];
    if (b < 0 || b >= B) { rc = ORACLE_BAD_ARG; goto done; }
    for (int h = 0; h < H; ++h) xb[h] = bf16_bits_to_double(x[(size_t)b * H + h]);
    vec_times_fp8(xb, q13, s13, 2 * I, H, gu);
    for (int c = 0; c < I; ++c) a[c] = silu(gu[c]) * gu[I + c];
    vec_times_fp8(a, q2, s2, H, I, y + (size_t)i * H);
  }
done:
  free(xb); free(gu); free(a);
  return rc;
}

/* Step 7 from per-assignment expert outputs: out_b = x_b + sum_j w_j y[b,j]
 * (+ s_b), with y [B,k,H] and s [B,H] (NULL: no shared expert) -- the same
 * additions, in the same order, as oracle_block. */
int oracle_combine(const uint16_t* x, const double* w, const double* y,
                   const double* s, int B, int H, int k, double* out) {
  if (B < 0 || H <= 0 || k < 0) return ORACLE_BAD_ARG;
  if (B == 0) return ORACLE_OK;
  if (!x || !out || (k > 0 && (!w || !y))) return ORACLE_BAD_ARG;
  for (int b = 0; b < B; ++b) {
    double* ob = out + (size_t)b * H;
    for (int h = 0; h < H; ++h) ob[h] = bf16_bits_to_double(x[(size_t)b * H + h]);
    for (int j = 0; j < k; ++j) {
      const double wj = w[(size_t)b * k + j];
      const double* yj = y + ((size_t)b * k + j) * H;
      for (int h = 0; h < H; ++h) ob[h] += wj * yj[h];
    }
    if (s)
      for (int h = 0; h < H; ++h) ob[h] += s[(size_t)b * H + h];
  }
  return ORACLE_OK;
}

/* Steps 1-7. */
int oracle_moe_forward(const uint16_t* x, const uint16_t* router_w, const float* bias,
                       const uint16_t* const* w13, const uint16_t* const* w2,
                       const uint16_t* sw13, const uint16_t* sw2, int B, int H,
                       int E, int k, int I, int Is, int n_shared, double* out,
                       int32_t* ids, double* w, double* logits) {
  int rc = oracle_router(x, router_w, bias, B, H, E, k, logits, ids, w);
  if (rc != ORACLE_OK) return rc;
  return oracle_block(x, ids, w, w13, w2, sw13, sw2, B, H, E, k, I, Is, n_shared, out);
}
