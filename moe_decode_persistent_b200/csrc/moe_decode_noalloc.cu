// moe_decode_noalloc.cu - the decode step for callers that cannot allocate device
// memory (see moe_decode_step_noalloc in include/moe_decode.h).
//
// Some callers cannot call cudaMalloc at all: allocator hooks, plugins hosted by a
// framework that owns all device memory, or processes whose memory budget is fixed
// before they start. For them the step's scratch (normalised rows, logits, SwiGLU
// outputs, split-K partials, counters and the TMA descriptors) lives in one
// file-scope device array sized for the limits below. Every GPU that loads this
// library holds the array until the process exits.
//
// The descriptors are built on the host at every call and reach the array through
// the parameters of a small kernel (na_store_maps), which copy them by value at
// launch: no host buffer is read after the call returns.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "kernel_params.h"
#include "moe_decode.h"

namespace moe {
size_t smem_bytes();
int threads_per_cta();
const void* kernel_fn();
}  // namespace moe

namespace {

// Limits of the no-allocation step.
constexpr int kNaMaxBatch = 4;
constexpr int kNaMaxTopK = 16;
constexpr int kNaMaxHidden = 7168;
constexpr int kNaMaxExperts = 1024;
constexpr int kNaMaxInter = 1024;
constexpr int kNaMaxSharedInter = 2048;
constexpr int kNaMaxLayers = 2;

constexpr size_t na_align(size_t v) { return (v + 255) / 256 * 256; }

// Worst-case work units and tiles at the limits (the kernel's unit enumeration:
// router / shared gate-up / expert gate-up with up to 4 K splits, down tiles with
// one shared split per row group and one split per two (expert, row group) pairs).
constexpr int kNaSlots = kNaMaxBatch * kNaMaxTopK;
constexpr int kNaGroups = (kNaMaxBatch + moe::kActGroup - 1) / moe::kActGroup;
constexpr int kNaRT = kNaMaxExperts / 32, kNaST = kNaMaxSharedInter / 32;
constexpr int kNaIT = kNaMaxInter / 32, kNaDT = kNaMaxHidden / 32;
constexpr unsigned kNaUnits = kNaGroups * kNaRT * 4 + kNaGroups * kNaST * 4 + kNaSlots * kNaIT * 4 +
                              kNaDT * (kNaGroups + (kNaSlots + moe::kDownPairsPerSplit - 1) /
                                                       moe::kDownPairsPerSplit);
constexpr unsigned kNaTiles = kNaGroups * (kNaRT + kNaST) + kNaSlots * kNaIT + kNaDT;

// Scratch layout (byte offsets, 256-byte aligned regions).
constexpr size_t kOffN = 0;
constexpr size_t kOffLogits = kOffN + na_align((size_t)kNaMaxBatch * kNaMaxHidden * 2);
constexpr size_t kOffHs = kOffLogits + na_align((size_t)kNaMaxBatch * kNaMaxExperts * 4);
constexpr size_t kOffHe = kOffHs + na_align((size_t)kNaMaxBatch * kNaMaxSharedInter * 2);
constexpr size_t kOffPartial = kOffHe + na_align((size_t)kNaSlots * kNaMaxInter * 2);
constexpr size_t kOffIo = kOffPartial + na_align((size_t)kNaUnits * moe::kPartialFloats * 4);
constexpr size_t kOffMaps = kOffIo + na_align((size_t)(kNaMaxLayers - 1) * kNaMaxBatch * kNaMaxHidden * 2);
// the regions below must be zero when a step starts; each call clears them
constexpr size_t kOffZero = kOffMaps + na_align(sizeof(CUtensorMap) * (moe::TM_WSD + 1) * kNaMaxLayers);
constexpr size_t kOffCtr = kOffZero;
constexpr size_t kOffTickets = kOffCtr + na_align(moe::CTR_COUNT * 4);
constexpr size_t kOffPairDone = kOffTickets + na_align((size_t)kNaTiles * 4);
constexpr size_t kScratchBytes = kOffPairDone + na_align((size_t)moe::kMaxSlots * 4);
constexpr size_t kZeroBytes = kScratchBytes - kOffZero;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

// The CUDA-core kernel's descriptors of up to kNaMaxLayers layers, by value.
constexpr int kNaMapsPerLayer = moe::TM_WSD + 1;
struct NaMaps {
  CUtensorMap m[kNaMapsPerLayer * kNaMaxLayers];
};
static_assert(sizeof(NaMaps) + 64 <= 4096, "descriptors fit the kernel parameter space");

// Copies the descriptors of n maps from the kernel parameters into dst (global).
__global__ void na_store_maps(const __grid_constant__ NaMaps src, int n, CUtensorMap* dst) {
  const int words = n * (int)(sizeof(CUtensorMap) / 16);
  const uint4* s4 = reinterpret_cast<const uint4*>(&src.m[0]);
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (int i = threadIdx.x; i < words; i += blockDim.x) d4[i] = s4[i];
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceState {
  bool ready;
  unsigned char* scratch;  // device address of g_noalloc_scratch on this device
  int num_sms;
};

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
DeviceState g_state[kMaxDevices];
EncodeTiledFn g_encode = nullptr;

bool na_dim_ok(int v, int max) { return v >= 32 && v <= max && v % 32 == 0 && (v % 256 == 0 || v <= 256); }

// Once per device, with that device current: the array's device address, the
// kernel's shared-memory attribute and the tensor-map encoder.
int na_setup(int dev, DeviceState** out) {
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  DeviceState& st = g_state[dev];
  if (!st.ready) {
    int major = 0, minor = 0, coop = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (major != 10 || minor != 0) return MOE_ERR_UNSUPPORTED_ARCH;
    if (!coop) return MOE_ERR_COOPERATIVE;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    if (cudaFuncSetAttribute(moe::kernel_fn(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)moe::smem_bytes()) != cudaSuccess)
      return MOE_ERR_COOPERATIVE;
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return MOE_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    st.scratch = static_cast<unsigned char*>(p);
    st.num_sms = sms;
    st.ready = true;
  }
  *out = &st;
  return MOE_OK;
}

int na_encode(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols) {
  if (!base || (reinterpret_cast<uintptr_t>(base) & 15u) != 0) return MOE_ERR_INVALID_ARG;
  const uint32_t box_cols = cols < (uint64_t)moe::kBoxColsMax ? (uint32_t)cols : (uint32_t)moe::kBoxColsMax;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, (cuuint32_t)moe::kBoxRows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_INVALID_ARG;
}

}  // namespace

extern "C" int moe_decode_step_noalloc(const moe_decode_config* cfg, const moe_decode_layer_weights* layers,
                                       const void* x_in, void* y_out, int batch, int top_k, void* stream,
                                       int* device_status) {
  if (!cfg || !layers || !x_in || !y_out || x_in == y_out || !device_status) return MOE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(device_status) & 3u) return MOE_ERR_INVALID_ARG;
  const moe_decode_config c = *cfg;
  if (c.n_layers < 1 || batch < 1 || top_k < 1 || top_k > c.n_experts || !(c.eps >= 0.0f))
    return MOE_ERR_INVALID_ARG;
  if (c.n_layers > kNaMaxLayers || batch > kNaMaxBatch || top_k > kNaMaxTopK ||
      !na_dim_ok(c.hidden, kNaMaxHidden) || !na_dim_ok(c.inter, kNaMaxInter) ||
      !na_dim_ok(c.shared_inter, kNaMaxSharedInter) || c.n_experts < 32 || c.n_experts % 32 != 0 ||
      c.n_experts > kNaMaxExperts)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((reinterpret_cast<uintptr_t>(x_in) & 15u) || (reinterpret_cast<uintptr_t>(y_out) & 15u))
    return MOE_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  DeviceState* st = nullptr;
  int rc = na_setup(dev, &st);
  if (rc != MOE_OK) return rc;

  const int H = c.hidden, E = c.n_experts, I = c.inter, Is = c.shared_inter, L = c.n_layers;
  NaMaps maps;
  memset(&maps, 0, sizeof maps);
  for (int l = 0; l < L; ++l) {
    const moe_decode_layer_weights& w = layers[l];
    if (!w.gamma || (reinterpret_cast<uintptr_t>(w.gamma) & 15u) || (reinterpret_cast<uintptr_t>(w.router_bias) & 3u))
      return MOE_ERR_INVALID_ARG;
    CUtensorMap* m = maps.m + l * kNaMapsPerLayer;
    if (na_encode(&m[moe::TM_WR], w.w_router, (uint64_t)E, (uint64_t)H) != MOE_OK ||
        na_encode(&m[moe::TM_WG], w.w_gate, (uint64_t)E * I, (uint64_t)H) != MOE_OK ||
        na_encode(&m[moe::TM_WU], w.w_up, (uint64_t)E * I, (uint64_t)H) != MOE_OK ||
        na_encode(&m[moe::TM_WD], w.w_down, (uint64_t)E * H, (uint64_t)I) != MOE_OK ||
        na_encode(&m[moe::TM_WSG], w.ws_gate, (uint64_t)Is, (uint64_t)H) != MOE_OK ||
        na_encode(&m[moe::TM_WSU], w.ws_up, (uint64_t)Is, (uint64_t)H) != MOE_OK ||
        na_encode(&m[moe::TM_WSD], w.ws_down, (uint64_t)H, (uint64_t)Is) != MOE_OK)
      return MOE_ERR_INVALID_ARG;
  }
  cudaStream_t s = (cudaStream_t)stream;
  unsigned char* base = st->scratch;
  // the descriptors travel in na_store_maps' parameters (by value, at launch); the
  // counters and tickets start at zero
  CUtensorMap* d_maps_w = reinterpret_cast<CUtensorMap*>(base + kOffMaps);
  na_store_maps<<<1, 128, 0, s>>>(maps, kNaMapsPerLayer * L, d_maps_w);
  if (cudaGetLastError() != cudaSuccess || cudaMemsetAsync(base + kOffZero, 0, kZeroBytes, s) != cudaSuccess)
    return MOE_ERR_CUDA;

  const CUtensorMap* d_maps = reinterpret_cast<const CUtensorMap*>(base + kOffMaps);
  for (int l = 0; l < L; ++l) {
    moe::Params p;
    memset(&p, 0, sizeof p);
    p.H = H;
    p.E = E;
    p.I = I;
    p.Is = Is;
    p.B = batch;
    p.k = top_k;
    p.eps = c.eps;
    uint16_t* io = reinterpret_cast<uint16_t*>(base + kOffIo);
    p.x = l == 0 ? (const uint16_t*)x_in : io;
    p.y = l == L - 1 ? (uint16_t*)y_out : io;
    p.ep_e0 = 0;  // every expert, whole-layer output
    p.ep_e1 = E;
    p.ep_rs = 1;
    const moe_decode_layer_weights& w = layers[l];
    p.tmaps = d_maps + l * kNaMapsPerLayer;
    p.gamma = (const uint16_t*)w.gamma;
    p.bias = w.router_bias;
    p.n = reinterpret_cast<uint16_t*>(base + kOffN);
    p.logits = reinterpret_cast<float*>(base + kOffLogits);
    p.hs = reinterpret_cast<uint16_t*>(base + kOffHs);
    p.he = reinterpret_cast<uint16_t*>(base + kOffHe);
    p.partial = reinterpret_cast<float*>(base + kOffPartial);
    p.ctr = reinterpret_cast<uint32_t*>(base + kOffCtr);
    p.gctr = p.ctr;  // one layer per launch: the launch-wide counters share the layer's block
    p.tickets = reinterpret_cast<uint32_t*>(base + kOffTickets);
    p.pair_done = reinterpret_cast<uint32_t*>(base + kOffPairDone);
    p.status = device_status;
    p.max_units = kNaUnits;
    p.max_tiles = kNaTiles;
    p.cap_slots = (unsigned)kNaSlots;
    p.cap_dpart_rows = (unsigned)(kNaSlots + kNaMaxBatch);
    p.wait_ns = 2000ull * 1000000ull;
    void* args[] = {&p};
    const cudaError_t e = cudaLaunchCooperativeKernel(moe::kernel_fn(), dim3(st->num_sms),
                                                      dim3(moe::threads_per_cta()), args, moe::smem_bytes(), s);
    if (e == cudaErrorCooperativeLaunchTooLarge) return MOE_ERR_COOPERATIVE;
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
