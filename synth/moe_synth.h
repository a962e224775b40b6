/*
 * moe_synth.h - seeded synthetic inputs for the MoE decode-layer workloads.
 *
 * This header is the ONLY code shared by the CPU oracle side and the GPU side.
 * It holds input generation, nothing of the layer's arithmetic: every weight,
 * gamma and hidden-state value of the workloads is a pure function of
 * (seed, tensor id, flat element index), so any expert can be regenerated on
 * the host bit-identically to what the device generated.
 *
 * Definition (the same on host and device, integer ops plus exact or
 * correctly-rounded fp32 steps only):
 *   mix64(z)       SplitMix64 output finaliser (Steele, Lea & Flood, "Fast
 *                  splittable pseudorandom number generators", OOPSLA 2014).
 *   key            = mix64(mix64(seed) ^ tensor_id)
 *   word(key, c)   = mix64(key + (c + 1) * 0x9E3779B97F4A7C15)   (mod 2^64)
 *                  i.e. output c of a SplitMix64 stream whose state is key.
 *   z(key, i)      = (S - 6*65535) / 65536, S = sum of the twelve 16-bit
 *                  fields of word(key, 3i), word(key, 3i+1), word(key, 3i+2)
 *                  (Irwin-Hall sum of 12 uniforms: mean 0, variance ~1,
 *                  support [-6, 6]; exact in fp32).
 *   value          = bf16_rne(mean + sigma * z), both fp32 ops rounded to
 *                  nearest-even separately (no fused multiply-add).
 *
 * Tensor ids pack (layer, kind): id = (layer << 8) | kind.
 */
#ifndef MOE_SYNTH_H
#define MOE_SYNTH_H

#include <stdint.h>

#if defined(__CUDACC__)
#define MS_FN static __host__ __device__ __forceinline__
#else
#define MS_FN static inline
#endif

#define MS_GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL
#define MS_IRWIN_HALL_CENTRE 393210 /* 6 * 65535 */

enum ms_kind {
  MS_KIND_GAMMA = 1,
  MS_KIND_W_ROUTER = 2,
  MS_KIND_W_GATE = 3,
  MS_KIND_W_UP = 4,
  MS_KIND_W_DOWN = 5,
  MS_KIND_WS_GATE = 6,
  MS_KIND_WS_UP = 7,
  MS_KIND_WS_DOWN = 8,
  MS_KIND_X = 9,
  MS_KIND_BIAS_PERM = 10,
  MS_KIND_ROW_NOISE = 11,
  MS_KIND_ROW_BASE = 12,
  MS_KIND_WQ_GATE = 13, /* FP8 expert weights: e4m3 codes */
  MS_KIND_WQ_UP = 14,
  MS_KIND_WQ_DOWN = 15,
  MS_KIND_SQ_GATE = 16, /* FP8 expert weights: per-block scale exponents */
  MS_KIND_SQ_UP = 17,
  MS_KIND_SQ_DOWN = 18
};

MS_FN uint64_t ms_tensor_id(uint32_t layer, uint32_t kind) {
  return ((uint64_t)layer << 8) | (uint64_t)kind;
}

MS_FN uint64_t ms_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

MS_FN uint64_t ms_key(uint64_t seed, uint64_t tensor_id) {
  return ms_mix64(ms_mix64(seed) ^ tensor_id);
}

MS_FN uint64_t ms_word(uint64_t key, uint64_t counter) {
  return ms_mix64(key + (counter + 1ULL) * MS_GOLDEN_GAMMA);
}

MS_FN int32_t ms_sum16x4(uint64_t w) {
  return (int32_t)(w & 0xFFFFu) + (int32_t)((w >> 16) & 0xFFFFu) +
         (int32_t)((w >> 32) & 0xFFFFu) + (int32_t)(w >> 48);
}

/* Approximately standard-normal value for element i; exact in fp32. */
MS_FN float ms_z(uint64_t key, uint64_t i) {
  int32_t s = ms_sum16x4(ms_word(key, 3 * i)) + ms_sum16x4(ms_word(key, 3 * i + 1)) +
              ms_sum16x4(ms_word(key, 3 * i + 2));
  return (float)(s - MS_IRWIN_HALL_CENTRE) * (1.0f / 65536.0f);
}

MS_FN uint32_t ms_f32_bits(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  return v.u;
}

/* fp32 -> bf16 bit pattern, round to nearest even; NaN maps to a quiet NaN. */
MS_FN uint16_t ms_bf16_rne(float f) {
  uint32_t u = ms_f32_bits(f);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0) return 0x7FC0u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

MS_FN float ms_mul_rn(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fmul_rn(a, b);
#else
  return a * b; /* host objects are built with -ffp-contract=off */
#endif
}

MS_FN float ms_add_rn(float a, float b) {
#if defined(__CUDA_ARCH__)
  return __fadd_rn(a, b);
#else
  return a + b;
#endif
}

/* One generated element: bf16(mean + sigma * z). */
MS_FN uint16_t ms_value_bf16(uint64_t key, uint64_t i, float sigma, float mean) {
  return ms_bf16_rne(ms_add_rn(mean, ms_mul_rn(sigma, ms_z(key, i))));
}

/*
 * FP8 E4M3 inputs (the low-precision expert weights). A code is the E4M3 value
 * (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448) nearest
 * to the fp32 value v (ties to even), after v is clamped to [-448, 448]:
 *   code(i) = e4m3(z(key, i) * (448 / 6))  -- the Irwin-Hall z in [-6, 6] spans the
 *                                             whole finite range
 * and every 128 x 128 block b of a matrix has a power-of-two scale 2^(s0 + d(b)),
 * d(b) = word(key_s, b) mod 3 - 1 (so neighbouring blocks differ). Only input
 * generation lives here: decoding a code and applying its scale is the layer's
 * arithmetic, done separately by the oracle and by the GPU kernel.
 */
MS_FN uint8_t ms_e4m3_rne(float v) {
  uint32_t u = ms_f32_bits(v);
  const uint32_t sign = (u >> 24) & 0x80u;
  float a = v < 0.0f ? -v : v;
  if (!(a < 448.0f)) return (uint8_t)(sign | 0x7Eu); /* clamp (and any NaN) to the largest finite */
  /* quantum of a's binade (normal for a >= 2^-6, else the subnormal spacing 2^-9) */
  uint32_t ab = ms_f32_bits(a);
  int e = (int)((ab >> 23) & 0xFFu) - 127;
  if (e < -6) e = -6;
  /* a / 2^(e-3), rounded to the nearest integer, ties to even: exact fp32 scaling */
  union { uint32_t u; float f; } sc;
  sc.u = (uint32_t)(127 - (e - 3)) << 23;
  const float t = ms_mul_rn(a, sc.f);            /* in [0, 16) */
  uint32_t q = (uint32_t)t;                       /* floor */
  const float frac = t - (float)q;                /* exact */
  if (frac > 0.5f || (frac == 0.5f && (q & 1u))) ++q;
  /* value = q * 2^(e-3); q in [0, 16] (16: carried into the next binade) */
  if (q == 0u) return (uint8_t)sign;
  if (e == -6 && q < 8u) return (uint8_t)(sign | q); /* subnormal: exponent field 0 */
  if (q == 16u) {
    q = 8u;
    ++e;
  }
  return (uint8_t)(sign | ((uint32_t)(e + 7) << 3) | (q - 8u));
}

/* One generated FP8 code (74.66666412353515625 is the fp32 value nearest 448 / 6). */
MS_FN uint8_t ms_code_e4m3(uint64_t key, uint64_t i) {
  return ms_e4m3_rne(ms_mul_rn(ms_z(key, i), 74.66666412353515625f));
}

/* Scale exponent of block b: s0 - 1, s0 or s0 + 1. */
MS_FN int ms_block_exp(uint64_t key, uint64_t b, int s0) {
  return s0 + (int)(ms_word(key, b) % 3ULL) - 1;
}

/*
 * Coverage codes (a test input that gives every E4M3 value full weight). In block b of
 * an expert matrix stack [E][rows][cols] (b counted expert-major, then 128-row block,
 * then 128-column block) every code has the exponent field f(b) = (b + phase) mod 16;
 * sign and 3 mantissa bits are drawn per element (the NaN codes 0x7F / 0xFF become
 * 0x7E / 0xFE). Block b's scale exponent is t + 7 - max(f(b), 1), so every block's
 * weights lie in [2^(t-3), 2^(t+1)) whatever its binade, subnormal blocks included.
 */
MS_FN uint32_t ms_cover_field(uint64_t b, uint32_t phase) { return (uint32_t)((b + phase) % 16u); }

MS_FN uint8_t ms_code_e4m3_cover(uint64_t key, uint64_t i, uint64_t rows, uint64_t cols, uint32_t phase) {
  const uint64_t per = rows * cols, e = i / per, r = (i % per) / cols, c = i % cols;
  const uint64_t b = (e * (rows / 128u) + r / 128u) * (cols / 128u) + c / 128u;
  const uint32_t f = ms_cover_field(b, phase);
  const uint64_t w = ms_word(key, i);
  uint32_t m = (uint32_t)(w & 7u);
  if (f == 15u && m == 7u) m = 6u;
  return (uint8_t)((((uint32_t)(w >> 3) & 1u) << 7) | (f << 3) | m);
}

MS_FN int ms_block_exp_cover(uint64_t b, uint32_t phase, int t) {
  const int f = (int)ms_cover_field(b, phase);
  return t + 7 - (f > 1 ? f : 1);
}

#endif /* MOE_SYNTH_H */
