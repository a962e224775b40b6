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
  MS_KIND_ROW_BASE = 12
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

#endif /* MOE_SYNTH_H */
