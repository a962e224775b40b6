/*
 * synth_host.c - host-side fills of the seeded synthetic inputs (moe_synth.h).
 * Built with -ffp-contract=off so each fp32 step rounds exactly as on the
 * device. OpenMP parallel; every element is independent.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#include "moe_synth.h"

/* out[i] = bf16(mean + sigma * z(key(seed, tid), start + i)), i < n. */
void ms_fill_host(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, float sigma,
                  float mean, uint16_t* out) {
  const uint64_t key = ms_key(seed, tensor_id);
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < (int64_t)n; ++i) out[i] = ms_value_bf16(key, start + (uint64_t)i, sigma, mean);
}

/* Raw fp32 z values (used by the generator's own tests). */
void ms_z_host(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, float* out) {
  const uint64_t key = ms_key(seed, tensor_id);
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < (int64_t)n; ++i) out[i] = ms_z(key, start + (uint64_t)i);
}

/* Raw stream words word(key(seed, tid), c) for c in [start, start + n). */
void ms_words_host(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, uint64_t* out) {
  const uint64_t key = ms_key(seed, tensor_id);
  for (uint64_t i = 0; i < n; ++i) out[i] = ms_word(key, start + i);
}

uint64_t ms_mix64_host(uint64_t z) { return ms_mix64(z); }

/*
 * Correlated rows (speculative-verify shape): rows are grouped in sequences of
 * rows_per_seq; row r of sequence s is bf16(base_s + 0.1 * noise_r), with
 * base_s ~ z(ROW_BASE) and noise_r ~ z(ROW_NOISE), both over flat indices.
 */
void ms_fill_rows_correlated(uint64_t seed, uint32_t layer, int nseq, int rows_per_seq, int H,
                             uint16_t* out) {
  const uint64_t kb = ms_key(seed, ms_tensor_id(layer, MS_KIND_ROW_BASE));
  const uint64_t kn = ms_key(seed, ms_tensor_id(layer, MS_KIND_ROW_NOISE));
  const int rows = nseq * rows_per_seq;
  int r;
#pragma omp parallel for schedule(static)
  for (r = 0; r < rows; ++r) {
    const int s = r / rows_per_seq;
    for (int h = 0; h < H; ++h) {
      float base = ms_z(kb, (uint64_t)s * (uint64_t)H + (uint64_t)h);
      float noise = ms_z(kn, (uint64_t)r * (uint64_t)H + (uint64_t)h);
      out[(size_t)r * H + h] = ms_bf16_rne(ms_add_rn(base, ms_mul_rn(0.1f, noise)));
    }
  }
}

/*
 * Skewed router bias: a seeded Fisher-Yates permutation assigns ranks 1..E to
 * the experts; expert at rank r gets b = 2 * log(1 / r^1.1) = -2.2 * ln(r),
 * evaluated in double and rounded to fp32.
 */
void ms_router_bias(uint64_t seed, uint32_t layer, int E, float* out) {
  const uint64_t key = ms_key(seed, ms_tensor_id(layer, MS_KIND_BIAS_PERM));
  int* perm = (int*)malloc(sizeof(int) * (size_t)E);
  for (int i = 0; i < E; ++i) perm[i] = i;
  for (int i = E - 1; i >= 1; --i) {
    const int j = (int)(ms_word(key, (uint64_t)i) % (uint64_t)(i + 1));
    const int t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
  }
  for (int r = 0; r < E; ++r) out[perm[r]] = (float)(-2.2 * log((double)(r + 1)));
  free(perm);
}

/* out[i] = E4M3 code of element start + i of tensor tid (ms_code_e4m3), i < n. */
void ms_fill_e4m3_host(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, uint8_t* out) {
  const uint64_t key = ms_key(seed, tensor_id);
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < (int64_t)n; ++i) out[i] = ms_code_e4m3(key, start + (uint64_t)i);
}

/* The E4M3 code nearest to each fp32 value (the generator's encoder; tests only). */
void ms_e4m3_encode_host(const float* v, uint64_t n, uint8_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = ms_e4m3_rne(v[i]);
}

/* Scale exponents of blocks start .. start + n - 1 of tensor tid: s0 - 1, s0 or s0 + 1. */
void ms_block_exps_host(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, int s0, int32_t* out) {
  const uint64_t key = ms_key(seed, tensor_id);
  for (uint64_t i = 0; i < n; ++i) out[i] = ms_block_exp(key, start + i, s0);
}

/* Coverage codes of elements start .. start + n - 1 of an expert stack [E][rows][cols]. */
void ms_fill_e4m3_cover_host(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, uint64_t rows,
                             uint64_t cols, uint32_t phase, uint8_t* out) {
  const uint64_t key = ms_key(seed, tensor_id);
  int64_t i;
#pragma omp parallel for schedule(static)
  for (i = 0; i < (int64_t)n; ++i) out[i] = ms_code_e4m3_cover(key, start + (uint64_t)i, rows, cols, phase);
}

/* Scale exponents of coverage blocks start .. start + n - 1. */
void ms_block_exps_cover_host(uint64_t start, uint64_t n, uint32_t phase, int t, int32_t* out) {
  for (uint64_t i = 0; i < n; ++i) out[i] = ms_block_exp_cover(start + i, phase, t);
}
