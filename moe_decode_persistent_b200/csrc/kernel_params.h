// kernel_params.h - parameters shared by the host API and the persistent kernel.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace moe {

// Tensor-map slots of one layer (all 2-D, bf16, row-major [rows][K]).
enum TensorMapSlot {
  TM_WR = 0,   // W_router  [E][H]
  TM_WG = 1,   // W_gate    [E*I][H]
  TM_WU = 2,   // W_up      [E*I][H]
  TM_WD = 3,   // W_down    [E*H][I]
  TM_WSG = 4,  // Ws_gate   [Is][H]
  TM_WSU = 5,  // Ws_up     [Is][H]
  TM_WSD = 6,  // Ws_down   [H][Is]
  TM_COUNT = 7
};

// Global counters of one step (reset by the last CTA of every launch).
enum Counter {
  CTR_QUEUE = 0,   // next unit of work
  CTR_EXIT = 1,    // CTAs finished
  CTR_NREADY = 2,  // normalised rows published
  CTR_ROUTER = 3,  // router tiles finished (logits published)
  CTR_HS = 4,      // shared gate/up tiles finished
  CTR_ABORT = 5,   // non-zero once any CTA gave up a wait
  CTR_COUNT = 8
};

// Work-unit limits that size the workspace.
constexpr int kBoxRows = 32;           // weight rows per TMA box (one output tile)
constexpr int kBoxColsMax = 256;       // K elements per TMA box
constexpr int kActGroup = 4;           // token rows per activation group (CUDA-core pass)
constexpr int kDownPairsPerSplit = 2;  // (expert, row-group) pairs per down split
constexpr int kPartialFloats = 2 * kBoxRows * kActGroup;  // floats per unit partial
constexpr int kMaxE = 1024;
constexpr int kMaxSlots = 1024;        // batch * top_k

struct Params {
  // shapes of this step
  int H, E, I, Is, B, k;
  float eps;
  // activations
  const uint16_t* x;  // bf16 [B][H]
  uint16_t* y;        // bf16 [B][H]
  // this layer's parameters
  const CUtensorMap* tmaps;  // TM_COUNT maps in global memory
  const uint16_t* gamma;     // bf16 [H]
  const float* bias;         // fp32 [E] or nullptr
  // next layer's router/shared weights (L2 prefetch), nullptr when last layer
  const void* pf_ptr[4];
  unsigned long long pf_bytes[4];
  // workspace
  uint16_t* n;           // bf16 [maxB][H]
  float* logits;         // fp32 [maxB][E]
  uint16_t* hs;          // bf16 [maxB][Is]
  uint16_t* he;          // bf16 [maxSlots][I]
  float* partial;        // fp32 [max_units][kPartialFloats]
  uint32_t* ctr;         // [CTR_COUNT]
  uint32_t* tickets;     // [max_tiles]
  uint32_t* pair_done;   // [kMaxSlots]
  int* status;           // device status word
  unsigned max_units, max_tiles;
  // debug outputs (nullable)
  float* dbg_logits;
  int* dbg_idx;
  float* dbg_w;
  int* dbg_nuniq;
  unsigned flags;        // bit 0: jitter, bit 1: withhold the n-ready signal
  unsigned long long wait_ns;
};

constexpr unsigned kFlagJitter = 1u;
constexpr unsigned kFlagWithholdNReady = 2u;

}  // namespace moe
