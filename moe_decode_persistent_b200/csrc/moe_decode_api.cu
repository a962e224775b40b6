// moe_decode_api.cu - the C ABI (include/moe_decode.h): handle creation, TMA
// descriptors, workspace, per-layer cooperative launches, status.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "kernel_params.h"
#include "moe_decode.h"

namespace moe {
size_t smem_bytes();
int threads_per_cta();
const void* kernel_fn();
const void* kernel_fn_trace();
size_t tc_smem_bytes();
int tc_threads_per_cta();
const void* tc_kernel_fn();
const void* tc_kernel_fn_trace();
const void* tc_fp8_kernel_fn();
const void* tc_ep_kernel_fn();
const void* tc_ep_kernel_fn_trace();
int launch_partial_to_bf16(const float* in, uint16_t* out, long long n, int sms, cudaStream_t stream);
const void* tc_fp8_kernel_fn_trace();
const void* fused_kernel_fn();
const void* fused_kernel_fn_trace();
}  // namespace moe

using moe::Params;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct moe_decode_handle {
  moe_decode_config cfg;
  int device;
  int num_sms;
  moe_decode_layer_weights* layers;
  moe_decode_layer_weights_fp8* layers_fp8;  // FP8 handles: the layers as given (else nullptr)
  CUtensorMap* d_tmaps;  // [n_layers][TM_COUNT]
  // workspace
  void* ws;              // one allocation, carved below
  uint16_t* n;
  float* logits;
  uint16_t* hs;
  uint16_t* he;
  float* partial;
  float* rpart;
  float* spart;
  float* epart;
  float* dpart;
  uint64_t* tk_pub;
  uint32_t* row_tix;
  unsigned row_tix_count;
  uint32_t* ctr;         // [n_layers][CTR_COUNT] (a fused launch uses one block per layer)
  uint32_t* tickets;
  uint32_t* pair_done;   // [n_layers][kMaxSlots]
  uint32_t* rows_done;   // [n_layers][max_batch]: output tile pairs combined per row (fused launch)
  int* status;
  uint16_t* layer_io;    // [n_layers - 1][max_batch][H] intermediate outputs
  uint16_t* x_stage;     // [max_batch][H] host-step staging
  uint16_t* y_stage;
  unsigned max_units, max_tiles;
  int ep_e0, ep_e1;  // the experts this handle's steps cover (0, E unless created for a range);
                     // its expert arrays hold experts ep_e0 .. ep_e1 - 1
  int tc_capable;    // every dimension a multiple of 128: the tensor-core kernel can run
  int tc_min_batch;  // batches of at least this many rows take the tensor-core path
  unsigned flags;
  unsigned long long wait_ns;
  unsigned long long* trace;  // nullable [n_layers][num_sms][kTraceSlots]
};

static int cuda_fail(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

static bool tile_dim_ok(int v) { return v >= 32 && v % 32 == 0 && (v % 256 == 0 || v <= 256); }

// Default batch threshold of the tensor-core path: every batch size. On the measured
// 7168-wide layers the tensor-core kernel was faster at batch 1 as well (179 vs
// 211 us per step): it takes the weight tiles straight from shared memory into the
// MMA, where the CUDA-core kernel spends issue slots on unpacking and FMAs.
static const int kDefaultTcMinBatch = 1;

static int encode_box(EncodeTiledFn enc, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swz) {
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return MOE_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// CUDA-core path boxes: 32 rows x min(cols, 256) columns, no swizzle.
static int encode_2d(EncodeTiledFn enc, CUtensorMap* map, const void* base, uint64_t rows,
                     uint64_t cols) {
  const uint32_t box_cols = cols < (uint64_t)moe::kBoxColsMax ? (uint32_t)cols : (uint32_t)moe::kBoxColsMax;
  return encode_box(enc, map, base, rows, cols, box_cols, (uint32_t)moe::kBoxRows, CU_TENSOR_MAP_SWIZZLE_NONE);
}

// FP8 expert codes: boxes of 128 rows x 64 one-byte codes, no swizzle (the routing warps
// read them and write the swizzled bf16 operand).
// E4M3 codes [rows][cols], box 128 columns (one K block) x 128 rows, 128-byte swizzled:
// 16-byte chunk c of box row r lands at chunk c ^ (r mod 8) of the row, so the
// converters, one row per lane, read distinct banks.
static int encode_fp8(EncodeTiledFn enc, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return MOE_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {(cuuint32_t)(2 * moe::kTcAtomK), (cuuint32_t)moe::kTcRows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Activation rows [rows][cols] (bf16) as a 3-D view {64 columns, rows, cols / 64 atoms} with
// box {64, 16, 2}: the 16 rows of two consecutive K atoms in one copy, laid out as two
// 16-row, 128-byte-swizzled boxes one after the other.
static int encode_act_pair(EncodeTiledFn enc, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return MOE_ERR_INVALID_ARG;
  cuuint64_t dims[3] = {(cuuint64_t)moe::kTcAtomK, rows, cols / moe::kTcAtomK};
  cuuint64_t strides[2] = {cols * 2, (cuuint64_t)moe::kTcAtomK * 2};
  cuuint32_t box[3] = {(cuuint32_t)moe::kTcAtomK, (cuuint32_t)moe::kTcActRows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Every FP8 block scale must be a power of two in [2^-117, 2^7] (either sign): the
// kernel turns a code into the bf16 value(code) x 2^-120 (exact; a bf16 subnormal for
// the E4M3 subnormals) and multiplies by scale x 2^120 (a bf16 normal for these scales),
// so the product is the weight value(code) x scale exactly and never a subnormal.
static bool fp8_scale_ok(float s) {
  uint32_t b;
  memcpy(&b, &s, 4);
  const int ex = (int)((b >> 23) & 0xFFu) - 127;
  return (b & 0x7FFFFFu) == 0u && ex >= -117 && ex <= 7 && ((b >> 23) & 0xFFu) != 0u;
}

static int check_fp8_scales(const moe_decode_layer_weights_fp8* f, int L, int E, int I, int H) {
  const size_t n = (size_t)E * (I / moe::kTcRows) * (H / moe::kTcRows);
  float* buf = (float*)malloc(n * sizeof(float));
  if (!buf) return MOE_ERR_NO_MEMORY;
  int rc = MOE_OK;
  for (int l = 0; l < L && rc == MOE_OK; ++l) {
    const float* arr[3] = {f[l].w_gate_scale, f[l].w_up_scale, f[l].w_down_scale};
    for (int a = 0; a < 3 && rc == MOE_OK; ++a) {
      if (cudaMemcpy(buf, arr[a], n * sizeof(float), cudaMemcpyDeviceToHost) != cudaSuccess) {
        rc = MOE_ERR_CUDA;
        break;
      }
      for (size_t i = 0; i < n; ++i)
        if (!fp8_scale_ok(buf[i])) {
          rc = MOE_ERR_INVALID_ARG;
          break;
        }
    }
  }
  free(buf);
  return rc;
}

// Tensor-core path boxes: 64 columns (one 128-byte swizzle atom) x `box_rows` rows.
static int encode_tc(EncodeTiledFn enc, CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                     uint32_t box_rows) {
  return encode_box(enc, map, base, rows, cols, (uint32_t)moe::kTcAtomK, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

static bool tc_shape_ok(const moe_decode_config& c) {
  const int R = moe::kTcRows;
  return c.hidden % R == 0 && c.inter % R == 0 && c.shared_inter % R == 0 && c.n_experts % R == 0 &&
         c.max_batch <= moe::kTcMaxN;
}

extern "C" {

const char* moe_decode_strerror(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_ARCH: return "device is not an sm_100 (B200) GPU";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported layer shape";
    case MOE_ERR_COOPERATIVE: return "cooperative persistent launch not possible on this device";
    case MOE_ERR_CUDA: return "CUDA call failed";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_NONFINITE: return "non-finite router logit";
    case MOE_ERR_NO_MEMORY: return "workspace allocation failed";
    case MOE_ERR_BOUNDS: return "schedule-derived index out of bounds (bounds-checked build)";
    default: return "unknown error";
  }
}

// Both create entry points: layers (bf16 experts), or fp8 (FP8 experts; layers then
// holds the same layers with the expert pointers set to the codes, for the checks).
// e0, e1: the experts the handle covers and its expert arrays hold (0, E: all).
static int create_impl(const moe_decode_config* cfg, const moe_decode_layer_weights* layers,
                       const moe_decode_layer_weights_fp8* fp8, int device, moe_decode_handle** out,
                       int e0 = 0, int e1 = -1) {
  if (!cfg || !layers || !out) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  const moe_decode_config c = *cfg;
  if (e1 < 0) e1 = c.n_experts;
  if (e0 < 0 || e0 >= e1 || e1 > c.n_experts) return MOE_ERR_INVALID_ARG;
  if (c.n_layers < 1 || c.n_layers > 8 || c.max_batch < 1 || c.max_batch > 64 || c.top_k_max < 1 ||
      c.top_k_max > 32 || c.top_k_max > c.n_experts || !(c.eps >= 0.0f))
    return MOE_ERR_INVALID_ARG;
  if (c.max_batch * c.top_k_max > moe::kMaxSlots) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!tile_dim_ok(c.hidden) || c.hidden > 16384 || !tile_dim_ok(c.inter) || !tile_dim_ok(c.shared_inter) ||
      c.n_experts < 32 || c.n_experts % 32 != 0 || c.n_experts > moe::kMaxE)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  for (int l = 0; l < c.n_layers; ++l) {
    const moe_decode_layer_weights& w = layers[l];
    if (!w.gamma || !w.w_router || !w.w_gate || !w.w_up || !w.w_down || !w.ws_gate || !w.ws_up ||
        !w.ws_down)
      return MOE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(w.gamma) & 15u) || (reinterpret_cast<uintptr_t>(w.router_bias) & 3u))
      return MOE_ERR_INVALID_ARG;
  }

  cudaError_t e = cudaSetDevice(device);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  int major = 0, minor = 0, coop = 0, sms = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device);
  cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, device);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device);
  if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED_ARCH;
  if (!coop) return MOE_ERR_COOPERATIVE;

  const size_t smem = moe::smem_bytes();
  e = cudaFuncSetAttribute(moe::kernel_fn(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(moe::kernel_fn_trace(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return MOE_ERR_COOPERATIVE;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, moe::kernel_fn(), moe::threads_per_cta(),
                                                    smem);
  if (e != cudaSuccess || per_sm < 1) return MOE_ERR_COOPERATIVE;
  // the tensor-core kernel: only for shapes whose every dimension is a multiple of 128,
  // and only if it can be made co-resident; otherwise every step takes the CUDA-core kernel
  int tc_ok = tc_shape_ok(c) ? 1 : 0;
  if (fp8 && !tc_ok) return MOE_ERR_UNSUPPORTED_SHAPE;  // FP8 experts: tensor-core path only
  if (fp8) {
    const int rc = check_fp8_scales(fp8, c.n_layers, c.n_experts, c.inter, c.hidden);
    if (rc != MOE_OK) return rc;
  }
  if (tc_ok) {
    const size_t tsm = moe::tc_smem_bytes();
    e = cudaFuncSetAttribute(moe::tc_kernel_fn(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::tc_kernel_fn_trace(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::tc_ep_kernel_fn(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::tc_ep_kernel_fn_trace(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::tc_fp8_kernel_fn(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::tc_fp8_kernel_fn_trace(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::fused_kernel_fn(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(moe::fused_kernel_fn_trace(), cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tsm);
    int tc_per_sm = 0;
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&tc_per_sm, moe::tc_kernel_fn(), moe::tc_threads_per_cta(),
                                                        tsm);
    if (e != cudaSuccess || tc_per_sm < 1) {
      (void)cudaGetLastError();  // clear the runtime's last-error state left by the failed query
      tc_ok = 0;
    }
  }

  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  e = cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return MOE_ERR_CUDA;
  EncodeTiledFn enc = reinterpret_cast<EncodeTiledFn>(fn);

  moe_decode_handle* h = (moe_decode_handle*)calloc(1, sizeof(moe_decode_handle));
  if (!h) return MOE_ERR_NO_MEMORY;
  h->cfg = c;
  h->device = device;
  h->num_sms = sms;
  h->wait_ns = 2000ull * 1000000ull;
  h->tc_capable = tc_ok;
  h->ep_e0 = e0;
  h->ep_e1 = e1;
  h->tc_min_batch = kDefaultTcMinBatch;
  h->layers = (moe_decode_layer_weights*)malloc(sizeof(moe_decode_layer_weights) * c.n_layers);
  memcpy(h->layers, layers, sizeof(moe_decode_layer_weights) * c.n_layers);
  if (fp8) {
    h->layers_fp8 = (moe_decode_layer_weights_fp8*)malloc(sizeof(moe_decode_layer_weights_fp8) * c.n_layers);
    memcpy(h->layers_fp8, fp8, sizeof(moe_decode_layer_weights_fp8) * c.n_layers);
  }

  const int H = c.hidden, E = c.n_experts, I = c.inter, Is = c.shared_inter, L = c.n_layers;
  const int Ew = e1 - e0;  // experts held by the expert arrays
  // host tensor maps
  CUtensorMap* maps = (CUtensorMap*)aligned_alloc(64, sizeof(CUtensorMap) * moe::TM_COUNT * L);
  if (!maps) {
    free(h->layers);
    free(h->layers_fp8);
    free(h);
    return MOE_ERR_NO_MEMORY;
  }
  memset(maps, 0, sizeof(CUtensorMap) * moe::TM_COUNT * L);
  int rc = MOE_OK;
  for (int l = 0; l < L && rc == MOE_OK; ++l) {
    const moe_decode_layer_weights& w = layers[l];
    CUtensorMap* m = maps + l * moe::TM_COUNT;
    rc |= encode_2d(enc, &m[moe::TM_WR], w.w_router, (uint64_t)E, (uint64_t)H);
    if (!fp8) {  // (an FP8 handle never takes the CUDA-core path)
      rc |= encode_2d(enc, &m[moe::TM_WG], w.w_gate, (uint64_t)Ew * I, (uint64_t)H);
      rc |= encode_2d(enc, &m[moe::TM_WU], w.w_up, (uint64_t)Ew * I, (uint64_t)H);
      rc |= encode_2d(enc, &m[moe::TM_WD], w.w_down, (uint64_t)Ew * H, (uint64_t)I);
    }
    rc |= encode_2d(enc, &m[moe::TM_WSG], w.ws_gate, (uint64_t)Is, (uint64_t)H);
    rc |= encode_2d(enc, &m[moe::TM_WSU], w.ws_up, (uint64_t)Is, (uint64_t)H);
    rc |= encode_2d(enc, &m[moe::TM_WSD], w.ws_down, (uint64_t)H, (uint64_t)Is);
    if (tc_ok) {
      const uint32_t R = (uint32_t)moe::kTcRows;
      rc |= encode_tc(enc, &m[moe::TM_T_WR], w.w_router, (uint64_t)E, (uint64_t)H, R);
      if (fp8) {
        rc |= encode_fp8(enc, &m[moe::TM_Q_WG], fp8[l].w_gate, (uint64_t)Ew * I, (uint64_t)H);
        rc |= encode_fp8(enc, &m[moe::TM_Q_WU], fp8[l].w_up, (uint64_t)Ew * I, (uint64_t)H);
        rc |= encode_fp8(enc, &m[moe::TM_Q_WD], fp8[l].w_down, (uint64_t)Ew * H, (uint64_t)I);
      } else {
        rc |= encode_tc(enc, &m[moe::TM_T_WG], w.w_gate, (uint64_t)Ew * I, (uint64_t)H, R);
        rc |= encode_tc(enc, &m[moe::TM_T_WU], w.w_up, (uint64_t)Ew * I, (uint64_t)H, R);
        rc |= encode_tc(enc, &m[moe::TM_T_WD], w.w_down, (uint64_t)Ew * H, (uint64_t)I, R);
      }
      rc |= encode_tc(enc, &m[moe::TM_T_WSG], w.ws_gate, (uint64_t)Is, (uint64_t)H, R);
      rc |= encode_tc(enc, &m[moe::TM_T_WSU], w.ws_up, (uint64_t)Is, (uint64_t)H, R);
      rc |= encode_tc(enc, &m[moe::TM_T_WSD], w.ws_down, (uint64_t)H, (uint64_t)Is, R);
    }
  }
  if (rc != MOE_OK) {
    free(maps);
    free(h->layers);
    free(h->layers_fp8);
    free(h);
    return rc < 0 ? MOE_ERR_INVALID_ARG : rc;
  }

  // workspace bounds (see the unit enumeration in the kernel)
  const int maxB = c.max_batch, maxSlots = c.max_batch * c.top_k_max;
  const int GB = (maxB + moe::kActGroup - 1) / moe::kActGroup;
  const int boxH = H < moe::kBoxColsMax ? H : moe::kBoxColsMax;
  const int nkbH = H / boxH;
  const int KS = nkbH < 4 ? nkbH : 4;
  const int RT = E / 32, ST = Is / 32, IT = I / 32, DT = H / 32;
  const int maxP = maxSlots;
  h->max_units = (unsigned)(GB * RT * KS + GB * ST * KS + maxP * IT * KS +
                            DT * (GB + (maxP + moe::kDownPairsPerSplit - 1) / moe::kDownPairsPerSplit));
  h->max_tiles = (unsigned)(GB * (RT + ST) + maxP * IT + DT);
  // tensor-core path: tile pairs of the router and of the down projection, one pair per
  // unique expert, K splits chosen per batch (tc_router_splits) and fixed otherwise
  const int nkH = H / moe::kTcAtomK;
  size_t rpart_floats = 0, spart_floats = 0, epart_floats = 0, dpart_floats = 0, row_tix_n = 0;
  const int tcS = moe::tc_clamp_splits(moe::kTcSharedSplits, nkH);
  const int tcE = moe::tc_clamp_splits(moe::kTcExpertSplits, nkH);
  if (tc_ok) {
    const int RT2 = (E + 2 * moe::kTcRows - 1) / (2 * moe::kTcRows), DT2 = (H + 2 * moe::kTcRows - 1) / (2 * moe::kTcRows);
    const int TST = Is / moe::kTcRows, TIT = I / moe::kTcRows;
    const int tcP = maxSlots < E ? maxSlots : E;
    int maxRS = 1;
    for (int bb = 1; bb <= maxB; ++bb) {
      const int rs = moe::tc_router_splits(bb, nkH);
      if ((size_t)rs * bb > rpart_floats) rpart_floats = (size_t)rs * bb;
      if (rs > maxRS) maxRS = rs;
    }
    rpart_floats *= (size_t)E;
    spart_floats = (size_t)tcS * maxB * 2 * Is;
    epart_floats = (size_t)tcE * maxSlots * 2 * I;
    dpart_floats = (size_t)(maxSlots + maxB) * H;
    row_tix_n = (size_t)DT2 * maxB;
    const unsigned tu = (unsigned)(RT2 * maxRS + TST * tcS + tcP * TIT * tcE + DT2 * (1 + tcP));
    const unsigned tt = (unsigned)(RT2 + TST + tcP * TIT + DT2);
    if (tu > h->max_units) h->max_units = tu;
    if (tt > h->max_tiles) h->max_tiles = tt;
  }
  const int actRows = (maxB + moe::kTcActRows - 1) / moe::kTcActRows * moe::kTcActRows;

  size_t off = 0;
  auto carve = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  const size_t o_n = carve((size_t)actRows * H * 2);
  const size_t o_logits = carve((size_t)maxB * E * 4);
  const size_t o_hs = carve((size_t)actRows * Is * 2);
  const size_t o_he = carve((size_t)moe::kMaxSlots * I * 2);
  const size_t o_part = carve((size_t)h->max_units * moe::kPartialFloats * 4);
  const size_t o_rpart = carve(rpart_floats * 4);
  const size_t o_spart = carve(spart_floats * 4);
  const size_t o_epart = carve(epart_floats * 4);
  const size_t o_dpart = carve(dpart_floats * 4);
  const size_t o_tkp = carve((size_t)maxSlots * 16);
  const size_t o_rtix = carve(row_tix_n * 4 + 4);
  const size_t o_ctr = carve((size_t)L * moe::CTR_COUNT * 4);
  const size_t o_tix = carve((size_t)h->max_tiles * 4);
  const size_t o_pd = carve((size_t)L * moe::kMaxSlots * 4);
  const size_t o_rows = carve((size_t)L * maxB * 4);
  const size_t o_status = carve(16);
  const size_t o_io = carve((size_t)(L > 1 ? L - 1 : 1) * maxB * H * 2);
  const size_t o_xs = carve((size_t)maxB * H * 2);
  const size_t o_ys = carve((size_t)maxB * H * 2);
  const size_t o_maps = carve(sizeof(CUtensorMap) * moe::TM_COUNT * L);
  e = cudaMalloc(&h->ws, off);
  if (e != cudaSuccess) {
    free(maps);
    free(h->layers);
    free(h->layers_fp8);
    free(h);
    return MOE_ERR_NO_MEMORY;
  }
  uint8_t* b = (uint8_t*)h->ws;
  h->n = (uint16_t*)(b + o_n);
  h->logits = (float*)(b + o_logits);
  h->hs = (uint16_t*)(b + o_hs);
  h->he = (uint16_t*)(b + o_he);
  h->partial = (float*)(b + o_part);
  h->rpart = (float*)(b + o_rpart);
  h->spart = (float*)(b + o_spart);
  h->epart = (float*)(b + o_epart);
  h->dpart = (float*)(b + o_dpart);
  h->tk_pub = (uint64_t*)(b + o_tkp);
  h->row_tix = (uint32_t*)(b + o_rtix);
  h->row_tix_count = (unsigned)row_tix_n;
  h->ctr = (uint32_t*)(b + o_ctr);
  h->tickets = (uint32_t*)(b + o_tix);
  h->pair_done = (uint32_t*)(b + o_pd);
  h->rows_done = (uint32_t*)(b + o_rows);
  h->status = (int*)(b + o_status);
  h->layer_io = (uint16_t*)(b + o_io);
  h->x_stage = (uint16_t*)(b + o_xs);
  h->y_stage = (uint16_t*)(b + o_ys);
  h->d_tmaps = (CUtensorMap*)(b + o_maps);
  if (tc_ok) {
    // activation operands of the tensor-core path (the same buffers in every layer)
    const uint32_t AR = (uint32_t)moe::kTcActRows;
    for (int l = 0; l < L && rc == MOE_OK; ++l) {
      CUtensorMap* m = maps + l * moe::TM_COUNT;
      rc |= encode_tc(enc, &m[moe::TM_T_AN], h->n, (uint64_t)actRows, (uint64_t)H, AR);
      rc |= encode_tc(enc, &m[moe::TM_T_AHS], h->hs, (uint64_t)actRows, (uint64_t)Is, AR);
      rc |= encode_tc(enc, &m[moe::TM_T_AHE], h->he, (uint64_t)moe::kMaxSlots, (uint64_t)I, AR);
      if (fp8) {
        rc |= encode_act_pair(enc, &m[moe::TM_Q_AN], h->n, (uint64_t)actRows, (uint64_t)H);
        rc |= encode_act_pair(enc, &m[moe::TM_Q_AHE], h->he, (uint64_t)moe::kMaxSlots, (uint64_t)I);
      }
    }
    if (rc != MOE_OK) {
      cudaFree(h->ws);
      free(maps);
      free(h->layers);
      free(h->layers_fp8);
    free(h->layers_fp8);
      free(h);
      return MOE_ERR_CUDA;
    }
  }
  // counters, tickets, flags and status start at zero; activations zeroed for hygiene
  e = cudaMemset(h->ws, 0, off);
  if (e == cudaSuccess)
    e = cudaMemcpy(h->d_tmaps, maps, sizeof(CUtensorMap) * moe::TM_COUNT * L, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  free(maps);
  if (e != cudaSuccess) {
    cudaFree(h->ws);
    free(h->layers);
    free(h->layers_fp8);
    free(h);
    return MOE_ERR_CUDA;
  }
  *out = h;
  return MOE_OK;
}

int moe_decode_create(const moe_decode_config* cfg, const moe_decode_layer_weights* layers, int device,
                      moe_decode_handle** out) {
  return create_impl(cfg, layers, nullptr, device, out);
}

int moe_decode_create_ep(const moe_decode_config* cfg, const moe_decode_layer_weights* layers, int device,
                         int expert_begin, int expert_end, moe_decode_handle** out) {
  if (!cfg || !out || cfg->n_layers != 1) return MOE_ERR_INVALID_ARG;
  if (expert_begin < 0 || expert_begin >= expert_end || expert_end > cfg->n_experts) return MOE_ERR_INVALID_ARG;
  const moe_decode_config c = *cfg;
  if (c.hidden % moe::kTcRows || c.inter % moe::kTcRows || c.shared_inter % moe::kTcRows ||
      c.n_experts % moe::kTcRows || c.max_batch > moe::kTcMaxN)
    return MOE_ERR_UNSUPPORTED_SHAPE;  // the tensor-core kernel only
  const int rc = create_impl(cfg, layers, nullptr, device, out, expert_begin, expert_end);
  if (rc != MOE_OK) return rc;
  if (!(*out)->tc_capable) {
    moe_decode_destroy(*out);
    *out = nullptr;
    return MOE_ERR_UNSUPPORTED_SHAPE;
  }
  (*out)->tc_min_batch = 1;
  return MOE_OK;
}

int moe_decode_create_fp8(const moe_decode_config* cfg, const moe_decode_layer_weights_fp8* layers, int device,
                          moe_decode_handle** out) {
  if (!cfg || !layers || !out || cfg->n_layers < 1 || cfg->n_layers > 8) return MOE_ERR_INVALID_ARG;
  moe_decode_layer_weights w[8];
  for (int l = 0; l < cfg->n_layers; ++l) {
    const moe_decode_layer_weights_fp8& f = layers[l];
    if (!f.w_gate_scale || !f.w_up_scale || !f.w_down_scale ||
        ((reinterpret_cast<uintptr_t>(f.w_gate_scale) | reinterpret_cast<uintptr_t>(f.w_up_scale) |
          reinterpret_cast<uintptr_t>(f.w_down_scale)) & 3u))
      return MOE_ERR_INVALID_ARG;
    w[l] = moe_decode_layer_weights{f.gamma, f.w_router, f.router_bias, f.w_gate, f.w_up, f.w_down,
                                    f.ws_gate, f.ws_up, f.ws_down};
  }
  return create_impl(cfg, w, layers, device, out);
}

static bool use_tc(const moe_decode_handle* h, int batch) {
  if (h->layers_fp8) return true;  // FP8 experts: the tensor-core kernel only
  if (h->ep_e0 != 0 || h->ep_e1 != h->cfg.n_experts) return true;  // an expert range: tensor cores only
  return h->tc_capable && h->tc_min_batch > 0 && batch >= h->tc_min_batch;
}

// A tensor-core step of several layers runs them all in one launch (the fused kernel);
// otherwise one launch per layer.
static bool fused_step(const moe_decode_handle* h, int batch) {
  // (an FP8 layer's routing warps convert its expert tiles after the routing, so they
  // cannot route the next layer meanwhile: FP8 stacks run one launch per layer)
  return use_tc(h, batch) && h->cfg.n_layers > 1 && !h->layers_fp8;
}

// y_part (nullable): the fp32 partial output of a one-layer step over the handle's
// experts (with x + s only when add_rs); y_out is then unused.
static int launch_layers(moe_decode_handle* h, const void* x_in, void* y_out, int batch, int top_k,
                         cudaStream_t stream, const moe_decode_debug* dbg, float* y_part = nullptr,
                         int add_rs = 1) {
  const moe_decode_config& c = h->cfg;
  const int L = c.n_layers;
  const bool tc = use_tc(h, batch);
  const bool fused = fused_step(h, batch);
  const int nkH = c.hidden / moe::kTcAtomK;
  moe::FusedParams f;
  memset(&f, 0, sizeof f);
  f.L = L;
  for (int l = 0; l < L; ++l) {
    Params& p = f.layer[l];
    p.H = c.hidden;
    p.E = c.n_experts;
    p.I = c.inter;
    p.Is = c.shared_inter;
    p.B = batch;
    p.k = top_k;
    p.eps = c.eps;
    p.x = l == 0 ? (const uint16_t*)x_in : h->layer_io + (size_t)(l - 1) * c.max_batch * c.hidden;
    p.y = l == L - 1 ? (uint16_t*)y_out : h->layer_io + (size_t)l * c.max_batch * c.hidden;
    p.ep_e0 = h->ep_e0;
    p.ep_e1 = h->ep_e1;
    p.ep_wbase = h->ep_e0;
    p.ep_rs = add_rs;
    p.y_part = y_part;
    const moe_decode_layer_weights& w = h->layers[l];
    p.tmaps = h->d_tmaps + l * moe::TM_COUNT;
    p.gamma = (const uint16_t*)w.gamma;
    p.bias = w.router_bias;
    if (h->layers_fp8) {
      p.fp8 = 1;
      p.sc_gate = h->layers_fp8[l].w_gate_scale;
      p.sc_up = h->layers_fp8[l].w_up_scale;
      p.sc_down = h->layers_fp8[l].w_down_scale;
    }
    p.n = h->n;
    p.logits = h->logits;
    p.hs = h->hs;
    p.he = h->he;
    p.partial = h->partial;
    p.tc = tc ? 1 : 0;
    if (tc) {
      p.RS = moe::tc_router_splits(batch, nkH);
      p.SS = moe::tc_shared_splits(batch, nkH);
      p.rpart = h->rpart;
      p.spart = h->spart;
      p.epart = h->epart;
      p.dpart = h->dpart;
      p.tk_pub = h->tk_pub;
      p.row_tix = h->row_tix;
      p.row_tix_count = h->row_tix_count;
    }
    // one layer per launch: every launch uses the first counter block; a fused launch
    // gives each layer its own block, completion flags and row counts
    p.ctr = h->ctr + (fused ? (size_t)l * moe::CTR_COUNT : 0);
    p.gctr = h->ctr;
    p.layer = fused ? l : 0;
    p.tickets = h->tickets;
    p.pair_done = h->pair_done + (fused ? (size_t)l * moe::kMaxSlots : 0);
    if (fused) {
      p.rows_in = l > 0 ? h->rows_done + (size_t)(l - 1) * c.max_batch : nullptr;
      p.rows_out = l + 1 < L ? h->rows_done + (size_t)l * c.max_batch : nullptr;
    }
    p.status = h->status;
    p.max_units = h->max_units;
    p.max_tiles = h->max_tiles;
    p.cap_slots = (unsigned)(c.max_batch * c.top_k_max);
    p.cap_dpart_rows = (unsigned)(c.max_batch * c.top_k_max + c.max_batch);
    if (dbg) {
      p.dbg_logits = dbg[l].logits;
      p.dbg_idx = dbg[l].topk_idx;
      p.dbg_w = dbg[l].topk_w;
      p.dbg_nuniq = dbg[l].n_unique;
    }
    p.flags = h->flags;
    p.wait_ns = h->wait_ns;
    p.trace = h->trace ? h->trace + (size_t)l * h->num_sms * moe::kTraceSlots : nullptr;
    if (fused) continue;
    void* args[] = {&p};
    const bool ep = y_part != nullptr || h->ep_e0 != 0 || h->ep_e1 != c.n_experts;
    const void* fn = !tc             ? (h->trace ? moe::kernel_fn_trace() : moe::kernel_fn())
                     : h->layers_fp8 ? (h->trace ? moe::tc_fp8_kernel_fn_trace() : moe::tc_fp8_kernel_fn())
                     : ep            ? (h->trace ? moe::tc_ep_kernel_fn_trace() : moe::tc_ep_kernel_fn())
                                     : (h->trace ? moe::tc_kernel_fn_trace() : moe::tc_kernel_fn());
    const int threads = tc ? moe::tc_threads_per_cta() : moe::threads_per_cta();
    const size_t smem = tc ? moe::tc_smem_bytes() : moe::smem_bytes();
    cudaError_t e = cudaLaunchCooperativeKernel(fn, dim3(h->num_sms), dim3(threads), args, smem, stream);
    if (e == cudaErrorCooperativeLaunchTooLarge) return MOE_ERR_COOPERATIVE;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (fused) {
    void* args[] = {&f};
    const void* fn = h->trace ? moe::fused_kernel_fn_trace() : moe::fused_kernel_fn();
    cudaError_t e = cudaLaunchCooperativeKernel(fn, dim3(h->num_sms), dim3(moe::tc_threads_per_cta()), args,
                                                moe::tc_smem_bytes(), stream);
    if (e == cudaErrorCooperativeLaunchTooLarge) return MOE_ERR_COOPERATIVE;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

static int check_step_args(moe_decode_handle* h, const void* x, void* y, int batch, int top_k) {
  if (!h || !x || !y || x == y) return MOE_ERR_INVALID_ARG;
  if (batch < 1 || batch > h->cfg.max_batch || top_k < 1 || top_k > h->cfg.top_k_max ||
      top_k > h->cfg.n_experts)
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

int moe_decode_step(moe_decode_handle* h, const void* x_in, void* y_out, int batch, int top_k,
                    void* stream, const moe_decode_debug* dbg) {
  int rc = check_step_args(h, x_in, y_out, batch, top_k);
  if (rc != MOE_OK) return rc;
  if ((reinterpret_cast<uintptr_t>(x_in) & 15u) || (reinterpret_cast<uintptr_t>(y_out) & 15u))
    return MOE_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return MOE_ERR_CUDA;
  return launch_layers(h, x_in, y_out, batch, top_k, (cudaStream_t)stream, dbg);
}

int moe_decode_step_partial(moe_decode_handle* h, const void* x_in, float* y_partial, int batch, int top_k,
                            int add_residual_shared, void* stream, const moe_decode_debug* dbg) {
  int rc = check_step_args(h, x_in, y_partial, batch, top_k);
  if (rc != MOE_OK) return rc;
  // one bf16 layer on the tensor-core kernel (FP8 handles have no partial step)
  if (h->cfg.n_layers != 1 || !h->tc_capable || h->layers_fp8) return MOE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x_in) & 15u) || (reinterpret_cast<uintptr_t>(y_partial) & 15u))
    return MOE_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return MOE_ERR_CUDA;
  return launch_layers(h, x_in, nullptr, batch, top_k, (cudaStream_t)stream, dbg, y_partial,
                       add_residual_shared ? 1 : 0);
}

int moe_decode_partial_to_bf16(const float* y_partial, void* y_out, long long n, int device, void* stream) {
  if (!y_partial || !y_out || n < 0) return MOE_ERR_INVALID_ARG;
  if (n == 0) return MOE_OK;
  if (cudaSetDevice(device) != cudaSuccess) return MOE_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, device) != cudaSuccess) return MOE_ERR_CUDA;
  return moe::launch_partial_to_bf16(y_partial, (uint16_t*)y_out, n, sms, (cudaStream_t)stream) == 0 ? MOE_OK
                                                                                                    : MOE_ERR_CUDA;
}

int moe_decode_step_host(moe_decode_handle* h, const void* x_host, void* y_host, int batch,
                         int top_k, void* stream, const moe_decode_debug* dbg) {
  int rc = check_step_args(h, x_host, y_host, batch, top_k);
  if (rc != MOE_OK) return rc;
  if (cudaSetDevice(h->device) != cudaSuccess) return MOE_ERR_CUDA;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t bytes = (size_t)batch * h->cfg.hidden * 2;
  if (cudaMemcpyAsync(h->x_stage, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  rc = launch_layers(h, h->x_stage, h->y_stage, batch, top_k, s, dbg);
  if (rc != MOE_OK) return rc;
  return cuda_fail(cudaMemcpyAsync(y_host, h->y_stage, bytes, cudaMemcpyDeviceToHost, s));
}

int moe_decode_get_status(moe_decode_handle* h, int* device_status) {
  if (!h || !device_status) return MOE_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return MOE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, h->status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (v != 0 && cudaMemset(h->status, 0, sizeof v) != cudaSuccess) return MOE_ERR_CUDA;
  *device_status = v;
  return MOE_OK;
}

int moe_decode_launches_per_step(const moe_decode_handle* h) {
  if (!h) return MOE_ERR_INVALID_ARG;
  return fused_step(h, h->cfg.max_batch) ? 1 : h->cfg.n_layers;
}

int moe_decode_set_debug(moe_decode_handle* h, unsigned flags, unsigned wait_ms) {
  if (!h || wait_ms == 0) return MOE_ERR_INVALID_ARG;
  h->flags = flags;
  h->wait_ns = (unsigned long long)wait_ms * 1000000ull;
  return MOE_OK;
}

int moe_decode_set_tc_min_batch(moe_decode_handle* h, int min_batch) {
  if (!h || min_batch < 0) return MOE_ERR_INVALID_ARG;
  h->tc_min_batch = min_batch;
  return MOE_OK;
}

int moe_decode_step_path(const moe_decode_handle* h, int batch) {
  if (!h || batch < 1 || batch > h->cfg.max_batch) return MOE_ERR_INVALID_ARG;
  return use_tc(h, batch) ? MOE_PATH_TENSOR_CORE : MOE_PATH_CUDA_CORE;
}

int moe_decode_trace_slots(const moe_decode_handle* h) {
  return h ? h->num_sms * (int)moe::kTraceSlots : MOE_ERR_INVALID_ARG;
}

int moe_decode_set_trace(moe_decode_handle* h, void* trace) {
  if (!h) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(trace) & 7u) return MOE_ERR_INVALID_ARG;
  h->trace = static_cast<unsigned long long*>(trace);
  return MOE_OK;
}

void moe_decode_destroy(moe_decode_handle* h) {
  if (!h) return;
  cudaSetDevice(h->device);
  cudaFree(h->ws);
  free(h->layers);
  free(h->layers_fp8);
  free(h);
}

}  // extern "C"
