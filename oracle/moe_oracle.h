/*
 * moe_oracle.h - fp64 CPU oracle of one MoE decode-layer step.
 * TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline timing).
 * All bf16 tensors are passed as raw bit patterns (uint16_t), row-major.
 */
#ifndef MOE_ORACLE_H
#define MOE_ORACLE_H

#include <stdint.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)
#define ORACLE_EMISSING (-2)    /* a selected expert's weights were not supplied */
#define ORACLE_ENONFINITE (-3)  /* a non-finite router logit */

typedef struct {
  int H, E, k, I, Is;
  double eps;
} oracle_dims;

typedef struct {
  const uint16_t* gamma;          /* [H] */
  const uint16_t* w_router;       /* [E][H] */
  const float* router_bias;       /* [E] or NULL */
  const uint16_t* const* w_gate;  /* E pointers, each [I][H] (NULL: not supplied) */
  const uint16_t* const* w_up;    /* E pointers, each [I][H] */
  const uint16_t* const* w_down;  /* E pointers, each [H][I] */
  const uint16_t* ws_gate;        /* [Is][H] */
  const uint16_t* ws_up;          /* [Is][H] */
  const uint16_t* ws_down;        /* [H][Is] */
} oracle_weights;

/* Planted mistakes (test of the pins only; 0 = the oracle itself). They exist only
 * in the separate build compiled with -DORACLE_MUTANTS (libmoe_oracle_mutants.so),
 * which alone exports oracle_set_mutant. */
#define ORACLE_MUT_NONE 0
#define ORACLE_MUT_NO_N_ROUND 1      /* n not rounded to bf16 */
#define ORACLE_MUT_NO_H_ROUND 2      /* SwiGLU product not rounded to bf16 */
#define ORACLE_MUT_RESIDUAL_N 3      /* residual adds n instead of x */
#define ORACLE_MUT_TIES_HIGH 4       /* ties go to the higher index */
#define ORACLE_MUT_EQUAL_WEIGHTS 5   /* selected experts weighted 1/k */
#define ORACLE_MUT_NO_SHARED 6       /* shared expert dropped */
#define ORACLE_MUT_SILU_ON_UP 7      /* silu applied to the up projection */
#define ORACLE_MUT_NO_GAMMA 8        /* RMSNorm gain dropped */
#define ORACLE_MUT_DOWN_TRANSPOSED 9 /* down projection read transposed */
#define ORACLE_MUT_NO_BIAS 10        /* router bias dropped */
#define ORACLE_MUT_EPS_OUTSIDE 11    /* eps added outside the square root */
#define ORACLE_MUT_E4M3_BIAS 12      /* E4M3 exponent bias 8 instead of 7 */
#define ORACLE_MUT_BLOCK_TRANSPOSED 13 /* FP8 block scales indexed [col block][row block] */
#define ORACLE_MUT_COUNT 14
void oracle_set_mutant(int m);

double oracle_bf16_to_double(uint16_t b);
double oracle_bf16_round(double v);
uint16_t oracle_double_to_bf16_bits(double v);

void oracle_rmsnorm(int H, double eps, const uint16_t* x, const uint16_t* gamma, double* n_out);
void oracle_router(int H, int E, const double* n, const uint16_t* w_router, const float* bias,
                   double* logits);
int oracle_topk(int E, int k, const double* v, int32_t* idx_out);
void oracle_softmax_selected(int k, const double* logits, const int32_t* idx, double* w_out);
void oracle_swiglu(int H, int F, const double* n, const uint16_t* wg, const uint16_t* wu,
                   const uint16_t* wd, double* out);

/* FP8 E4M3 code -> value (NaN for the NaN codes). */
double oracle_e4m3_to_double(uint8_t code);
/* [rows][cols] E4M3 codes times one scale per 128 x 128 block -> bf16 bits;
 * ORACLE_EINVAL if a product is not a bf16 value or a code is NaN. */
int oracle_dequant_e4m3(int rows, int cols, const uint8_t* codes, const float* scales, uint16_t* out);

/* B rows; outputs: logits [B][E], topk_idx [B][k], topk_w [B][k], y_pre [B][H]
 * (fp64 before the final rounding; may be NULL), y [B][H] bf16 bits (may be NULL). */
int oracle_layer(const oracle_dims* d, const oracle_weights* w, int B, const uint16_t* x,
                 double* logits, int32_t* topk_idx, double* topk_w, double* y_pre, uint16_t* y);

/* The same layer with each row's selection given instead of chosen: sel [B][k]
 * holds k distinct experts per row. The logits are still the row's own, and the
 * weights are the softmax of those logits over the given set (so a given set
 * equal to the top-k reproduces oracle_layer exactly). topk_idx receives a copy
 * of sel. ORACLE_EINVAL for a repeated or out-of-range expert. */
int oracle_layer_selected(const oracle_dims* d, const oracle_weights* w, int B, const uint16_t* x,
                          const int32_t* sel, double* logits, int32_t* topk_idx, double* topk_w,
                          double* y_pre, uint16_t* y);

/* The part of the layer's output (fp64, before the final rounding) that the experts
 * e0 <= e < e1 contribute: y_part [B][H] = sum over each row's top-k choices j with
 * e0 <= S_j < e1 of w_j E_{S_j}(n), plus x + s when with_rs -- the split of the layer
 * over GPUs that each own a range of the experts (page post.smzdm.com/p/a6zppe4g,
 * section "改了什么：每层 23 个 kernel 砍到 13 个", item "把通信缝进计算"). Only the
 * experts in the range need weights. sel: NULL (each row's own top-k) or [B][k] given
 * selections as for oracle_layer_selected. */
int oracle_layer_partial(const oracle_dims* d, const oracle_weights* w, int B, const uint16_t* x,
                         const int32_t* sel, int e0, int e1, int with_rs, double* y_part);

#endif
