/*
 * moe_oracle.c - plain, slow fp64 CPU oracle of one MoE decode-layer step.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call this code:
 * only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * use it. It shares no code with the CUDA path.
 *
 * What it computes: one decode step of a sparse mixture-of-experts layer of
 * the kind the Kimi K3 decode pages describe (page "vLLM 合併 Kimi K3 專用解碼：
 * 官方稱 GB300 快 1.5 到 2 倍，423 tok/s 怎麼核對", section "Kimi K3 專用解碼路徑
 * 改了什麼": 896 routed experts, 16 active per token; page
 * post.smzdm.com/p/a6zppe4g, section "改了什么：每层 23 个 kernel 砍到 13 个":
 * router scores and a shared expert that runs beside the routing). The pages
 * give no formulas; the definition below is the plainest reading of the
 * workload description, written out directly, row by row, in fp64:
 *
 *   n      = bf16( x * rsqrt(mean(x^2) + eps) * gamma )          RMSNorm
 *   l[e]   = sum_h n[h] * W_r[e,h]  (+ bias[e])                   router logits
 *   S      = the k largest l[e], ties to the lower e              top-k
 *   w[j]   = exp(l[S_j]) / sum_i exp(l[S_i])                      renormalised
 *   E_e(n) = W_d[e] * bf16( silu(W_g[e] n) (.) (W_u[e] n) )        SwiGLU expert
 *   s      = W_sd  * bf16( silu(W_sg n)   (.) (W_su n) )           shared expert
 *   y      = bf16( x + s + sum_j w[j] * E_{S_j}(n) )              combine + residual
 *
 * bf16 rounding (round to nearest even) is applied exactly at the three
 * points the workload fixes as bf16 activations (n, the SwiGLU product h, and
 * the output y); every other quantity stays fp64. silu(v) = v / (1 + exp(-v)).
 * Rows are independent; parallelism (OpenMP) is over output features only.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "moe_oracle.h"

/* ---- bf16 helpers (fp64 <-> bf16) ---------------------------------------- */

double oracle_bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Round an fp64 value to the nearest bf16 value (ties to even), directly from
 * fp64 (no intermediate fp32 rounding). bf16: 8 significant bits, the fp32
 * exponent range, subnormals below 2^-126. */
double oracle_bf16_round(double v) {
  if (v == 0.0 || !isfinite(v)) return v;
  int e;
  (void)frexp(v, &e); /* |v| in [2^(e-1), 2^e) */
  int ulp_exp = e - 8;
  if (ulp_exp < -133) ulp_exp = -133; /* subnormal spacing 2^-133 */
  double r = ldexp(nearbyint(ldexp(v, -ulp_exp)), ulp_exp);
  const double max_bf16 = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
  if (fabs(r) > max_bf16) return v > 0 ? INFINITY : -INFINITY;
  return r;
}

uint16_t oracle_double_to_bf16_bits(double v) {
  float f = (float)oracle_bf16_round(v); /* exact: the value is a bf16 value */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if (isnan(v)) return 0x7FC0u;
  return (uint16_t)(u >> 16);
}

static inline double bf(uint16_t b) { return oracle_bf16_to_double(b); }

static double silu(double v) { return v / (1.0 + exp(-v)); }

/* Planted mistakes exist only in a second build of this file, compiled with
 * -DORACLE_MUTANTS for the test that proves the pins catch mistakes; there
 * oracle_set_mutant(m) swaps in one plausible error (ORACLE_MUT_* in
 * moe_oracle.h). In the oracle itself every MUT() is the constant 0. */
#ifdef ORACLE_MUTANTS
static int g_mutant = 0;
void oracle_set_mutant(int m) { g_mutant = m; }
#define MUT(m) (g_mutant == (m))
#else
#define MUT(m) 0
#endif

/* ---- stages ---------------------------------------------------------------- */

/* RMSNorm of one row: n = bf16(x * rsqrt(mean(x^2) + eps) * gamma). */
void oracle_rmsnorm(int H, double eps, const uint16_t* x, const uint16_t* gamma, double* n_out) {
  double ss = 0.0;
  for (int h = 0; h < H; ++h) ss += bf(x[h]) * bf(x[h]);
  double r = 1.0 / sqrt(ss / (double)H + eps);
  if (MUT(ORACLE_MUT_EPS_OUTSIDE)) r = 1.0 / (sqrt(ss / (double)H) + eps);
  for (int h = 0; h < H; ++h) {
    const double g = MUT(ORACLE_MUT_NO_GAMMA) ? 1.0 : bf(gamma[h]);
    const double v = bf(x[h]) * r * g;
    n_out[h] = MUT(ORACLE_MUT_NO_N_ROUND) ? v : oracle_bf16_round(v);
  }
}

/* y[m] = sum_k W[m,k] * v[k] for a row-major bf16 matrix W [M][K]. */
static void matvec(int M, int K, const uint16_t* W, const double* v, double* out) {
  int m;
#pragma omp parallel for schedule(static)
  for (m = 0; m < M; ++m) {
    const uint16_t* row = W + (size_t)m * (size_t)K;
    double acc = 0.0;
    for (int k = 0; k < K; ++k) acc += bf(row[k]) * v[k];
    out[m] = acc;
  }
}

/* Router logits of one row: l[e] = n . W_r[e] (+ bias[e]). */
void oracle_router(int H, int E, const double* n, const uint16_t* w_router, const float* bias,
                   double* logits) {
  matvec(E, H, w_router, n, logits);
  if (bias && !MUT(ORACLE_MUT_NO_BIAS))
    for (int e = 0; e < E; ++e) logits[e] += (double)bias[e];
}

/* The k largest values, ties to the lower index; idx_out in descending value
 * order. Returns -1 on a non-finite value or bad k. Plain O(k E) selection. */
int oracle_topk(int E, int k, const double* v, int32_t* idx_out) {
  if (E < 1 || k < 1 || k > E) return -1;
  for (int e = 0; e < E; ++e)
    if (!isfinite(v[e])) return -1;
  unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < E; ++e) {
      if (taken[e]) continue;
      if (best < 0 || v[e] > v[best]) best = e; /* strict: the lower index keeps a tie */
      else if (MUT(ORACLE_MUT_TIES_HIGH) && v[e] == v[best]) best = e;
    }
    taken[best] = 1;
    idx_out[j] = best;
  }
  free(taken);
  return 0;
}

/* Softmax over the selected logits (the full softmax renormalised over S). */
void oracle_softmax_selected(int k, const double* logits, const int32_t* idx, double* w_out) {
  double m = logits[idx[0]];
  for (int j = 1; j < k; ++j)
    if (logits[idx[j]] > m) m = logits[idx[j]];
  double z = 0.0;
  for (int j = 0; j < k; ++j) z += exp(logits[idx[j]] - m);
  for (int j = 0; j < k; ++j) w_out[j] = exp(logits[idx[j]] - m) / z;
  if (MUT(ORACLE_MUT_EQUAL_WEIGHTS))
    for (int j = 0; j < k; ++j) w_out[j] = 1.0 / (double)k;
}

/* SwiGLU expert: out = W_d * bf16(silu(W_g n) (.) (W_u n)); W_g,W_u [F][H], W_d [H][F]. */
void oracle_swiglu(int H, int F, const double* n, const uint16_t* wg, const uint16_t* wu,
                   const uint16_t* wd, double* out) {
  double* g = (double*)malloc(sizeof(double) * (size_t)F);
  double* u = (double*)malloc(sizeof(double) * (size_t)F);
  matvec(F, H, wg, n, g);
  matvec(F, H, wu, n, u);
  for (int i = 0; i < F; ++i) {
    double v = MUT(ORACLE_MUT_SILU_ON_UP) ? g[i] * silu(u[i]) : silu(g[i]) * u[i];
    g[i] = MUT(ORACLE_MUT_NO_H_ROUND) ? v : oracle_bf16_round(v);
  }
  if (MUT(ORACLE_MUT_DOWN_TRANSPOSED)) {
    for (int m = 0; m < H; ++m) {
      double acc = 0.0;
      for (int k = 0; k < F; ++k) acc += bf(wd[(size_t)k * H + m]) * g[k];
      out[m] = acc;
    }
  } else {
    matvec(H, F, wd, g, out);
  }
  free(g);
  free(u);
}

/* ---- FP8 expert weights ---------------------------------------------------------- */

/* The value of an FP8 E4M3 code (OCP FP8 "E4M3": 1 sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent field 0 is subnormal, m/8 * 2^-6; S.1111.111 is
 * NaN; there are no infinities). */
double oracle_e4m3_to_double(uint8_t code) {
  const int sgn = (code >> 7) & 1, ex = (code >> 3) & 15, m = code & 7;
  if (ex == 15 && m == 7) return NAN;
  const int bias = MUT(ORACLE_MUT_E4M3_BIAS) ? 8 : 7;
  const double mag = ex == 0 ? ldexp((double)m / 8.0, 1 - bias) : ldexp(1.0 + (double)m / 8.0, ex - bias);
  return sgn ? -mag : mag;
}

/* Dequantises a [rows][cols] matrix of E4M3 codes with one scale per 128 x 128 block
 * (scales [ceil(rows/128)][ceil(cols/128)]): w = value(code) * scale, returned as bf16
 * bits. The layer with FP8 expert weights is the bf16 layer evaluated on these weights,
 * so every w must be a bf16 value: ORACLE_EINVAL if one is not (or a code is NaN). */
int oracle_dequant_e4m3(int rows, int cols, const uint8_t* codes, const float* scales, uint16_t* out) {
  const int cb = (cols + 127) / 128;
  for (int r = 0; r < rows; ++r)
    for (int c = 0; c < cols; ++c) {
      const size_t blk = MUT(ORACLE_MUT_BLOCK_TRANSPOSED) ? (size_t)(c / 128) * ((rows + 127) / 128) + r / 128
                                                          : (size_t)(r / 128) * cb + c / 128;
      const double w = oracle_e4m3_to_double(codes[(size_t)r * cols + c]) * (double)scales[blk];
      if (!isfinite(w) || oracle_bf16_round(w) != w) return ORACLE_EINVAL;
      out[(size_t)r * cols + c] = oracle_double_to_bf16_bits(w);
    }
  return ORACLE_OK;
}

/* ---- whole layer ------------------------------------------------------------ */

/* The output of one row once its selection and weights are known:
 * y = bf16(x + s + sum_j w[j] E_{S_j}(n)), the shared expert first, then the
 * selected experts in the order given. Restricted to the experts e0 <= e < e1 and,
 * with_rs == 0, without x + s, it is the part of the row those experts contribute
 * (a part of an expert-parallel layer). Scratch: s, ex, acc (H each). */
static int combine_row(const oracle_dims* d, const oracle_weights* w, const uint16_t* xb,
                       const double* n, const int32_t* ib, const double* wb, int e0, int e1, int with_rs,
                       double* s, double* ex, double* acc, double* y_pre, uint16_t* y) {
  const int H = d->H, k = d->k, I = d->I, Is = d->Is;
  if (with_rs) oracle_swiglu(H, Is, n, w->ws_gate, w->ws_up, w->ws_down, s);
  for (int h = 0; h < H; ++h) {
    const double res = MUT(ORACLE_MUT_RESIDUAL_N) ? n[h] : bf(xb[h]);
    acc[h] = with_rs ? res + (MUT(ORACLE_MUT_NO_SHARED) ? 0.0 : s[h]) : 0.0;
  }
  for (int j = 0; j < k; ++j) {
    const int e = ib[j];
    if (e < e0 || e >= e1) continue;
    if (!w->w_gate[e] || !w->w_up[e] || !w->w_down[e]) return ORACLE_EMISSING;
    oracle_swiglu(H, I, n, w->w_gate[e], w->w_up[e], w->w_down[e], ex);
    for (int h = 0; h < H; ++h) acc[h] += wb[j] * ex[h];
  }
  for (int h = 0; h < H; ++h) {
    if (y_pre) y_pre[h] = acc[h];
    if (y) y[h] = oracle_double_to_bf16_bits(acc[h]);
  }
  return ORACLE_OK;
}

/* Both whole-layer entry points. sel == NULL: each row's selection is the top-k
 * of its logits. Otherwise sel [B][k] gives each row's selection (k distinct
 * experts); the weights are then the softmax of the row's own logits over it. */
static int layer_rows(const oracle_dims* d, const oracle_weights* w, int B, const uint16_t* x,
                      const int32_t* sel, int e0, int e1, int with_rs, double* logits, int32_t* topk_idx,
                      double* topk_w, double* y_pre, uint16_t* y) {
  const int H = d->H, E = d->E, k = d->k, I = d->I, Is = d->Is;
  if (B < 0 || H < 1 || E < 1 || k < 1 || k > E || I < 1 || Is < 1) return ORACLE_EINVAL;
  if (sel) {
    for (int b = 0; b < B; ++b)
      for (int j = 0; j < k; ++j) {
        const int e = sel[(size_t)b * k + j];
        if (e < 0 || e >= E) return ORACLE_EINVAL;
        for (int i = 0; i < j; ++i)
          if (sel[(size_t)b * k + i] == e) return ORACLE_EINVAL;
      }
  }
  double* n = (double*)malloc(sizeof(double) * (size_t)H);
  double* s = (double*)malloc(sizeof(double) * (size_t)H);
  double* ex = (double*)malloc(sizeof(double) * (size_t)H);
  double* acc = (double*)malloc(sizeof(double) * (size_t)H);
  int rc = ORACLE_OK;
  for (int b = 0; b < B && rc == ORACLE_OK; ++b) {
    const uint16_t* xb = x + (size_t)b * H;
    double* lb = logits + (size_t)b * E;
    int32_t* ib = topk_idx + (size_t)b * k;
    double* wb = topk_w + (size_t)b * k;

    oracle_rmsnorm(H, d->eps, xb, w->gamma, n);
    oracle_router(H, E, n, w->w_router, w->router_bias, lb);
    if (sel) {
      for (int e = 0; e < E; ++e)
        if (!isfinite(lb[e])) rc = ORACLE_ENONFINITE;
      if (rc != ORACLE_OK) break;
      memcpy(ib, sel + (size_t)b * k, sizeof(int32_t) * (size_t)k);
    } else if (oracle_topk(E, k, lb, ib) != 0) {
      rc = ORACLE_ENONFINITE;
      break;
    }
    oracle_softmax_selected(k, lb, ib, wb);
    rc = combine_row(d, w, xb, n, ib, wb, e0, e1, with_rs, s, ex, acc, y_pre ? y_pre + (size_t)b * H : NULL,
                     y ? y + (size_t)b * H : NULL);
  }
  free(n);
  free(s);
  free(ex);
  free(acc);
  return rc;
}

int oracle_layer(const oracle_dims* d, const oracle_weights* w, int B, const uint16_t* x,
                 double* logits, int32_t* topk_idx, double* topk_w, double* y_pre, uint16_t* y) {
  return layer_rows(d, w, B, x, NULL, 0, d->E, 1, logits, topk_idx, topk_w, y_pre, y);
}

int oracle_layer_selected(const oracle_dims* d, const oracle_weights* w, int B, const uint16_t* x,
                          const int32_t* sel, double* logits, int32_t* topk_idx, double* topk_w,
                          double* y_pre, uint16_t* y) {
  if (!sel) return ORACLE_EINVAL;
  return layer_rows(d, w, B, x, sel, 0, d->E, 1, logits, topk_idx, topk_w, y_pre, y);
}

int oracle_layer_partial(const oracle_dims* d, const oracle_weights* w, int B, const uint16_t* x,
                         const int32_t* sel, int e0, int e1, int with_rs, double* y_part) {
  if (!d || B < 0 || e0 < 0 || e1 < e0 || e1 > d->E || !y_part) return ORACLE_EINVAL;
  double* logits = (double*)malloc(sizeof(double) * (size_t)(B > 0 ? B : 1) * (size_t)d->E);
  int32_t* idx = (int32_t*)malloc(sizeof(int32_t) * (size_t)(B > 0 ? B : 1) * (size_t)d->k);
  double* wts = (double*)malloc(sizeof(double) * (size_t)(B > 0 ? B : 1) * (size_t)d->k);
  const int rc = layer_rows(d, w, B, x, sel, e0, e1, with_rs, logits, idx, wts, y_part, NULL);
  free(logits);
  free(idx);
  free(wts);
  return rc;
}
