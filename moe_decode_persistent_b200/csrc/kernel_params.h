// kernel_params.h - parameters shared by the host API and the persistent kernel.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace moe {

// Tensor-map slots of one layer (all 2-D, bf16, row-major [rows][K]).
// Slots 0-6: CUDA-core path, boxes of 32 rows x up to 256 K columns, no swizzle.
// Slots 7-16: tensor-core path, 128-byte swizzled boxes of 64 K columns (the
// K-major operand layout tcgen05.mma reads): weights 128 rows, activations 16 rows.
enum TensorMapSlot {
  TM_WR = 0,   // W_router  [E][H]
  TM_WG = 1,   // W_gate    [E*I][H]
  TM_WU = 2,   // W_up      [E*I][H]
  TM_WD = 3,   // W_down    [E*H][I]
  TM_WSG = 4,  // Ws_gate   [Is][H]
  TM_WSU = 5,  // Ws_up     [Is][H]
  TM_WSD = 6,  // Ws_down   [H][Is]
  TM_T_WR = 7,
  TM_T_WG = 8,
  TM_T_WU = 9,
  TM_T_WD = 10,
  TM_T_WSG = 11,
  TM_T_WSU = 12,
  TM_T_WSD = 13,
  TM_T_AN = 14,   // normalised rows n  [max_batch][H]
  TM_T_AHS = 15,  // shared SwiGLU rows [max_batch][Is]
  TM_T_AHE = 16,  // expert SwiGLU rows [slots][I]
  // FP8 expert weights (E4M3 codes, one byte each): boxes of 128 rows x 128 codes (one
  // K block), 128-byte swizzled
  TM_Q_WG = 17,   // W_gate codes [E*I][H]
  TM_Q_WU = 18,   // W_up codes   [E*I][H]
  TM_Q_WD = 19,   // W_down codes [E*H][I]
  // FP8 layers: the activations of two K atoms in one box {64 columns, 16 rows, 2 atoms}
  // (3-D view: column within the atom, row, atom), 128-byte swizzled
  TM_Q_AN = 20,   // normalised rows n  [max_batch][H]
  TM_Q_AHE = 21,  // expert SwiGLU rows [slots][I]
  TM_COUNT = 22
};

// Counters of one layer step (reset by the last CTA of every launch, except the epoch).
// A launch that runs several layers has one block per layer (Params::ctr) and keeps
// CTR_EXIT, CTR_ABORT and CTR_EPOCH in the first layer's block (Params::gctr).
enum Counter {
  CTR_QUEUE = 0,   // next unit of work
  CTR_EXIT = 1,    // CTAs finished (launch-wide)
  CTR_NREADY = 2,  // normalised rows published
  CTR_ROUTER = 3,  // router tiles finished (logits published)
  CTR_HS = 4,      // shared gate/up tiles finished
  CTR_ABORT = 5,   // non-zero once any CTA gave up a wait (launch-wide)
  CTR_TOPK = 6,    // tensor-core path: rows whose top-k choices are published
  CTR_EPOCH = 7,   // launches completed on this workspace (never reset): tags the choices
  CTR_COUNT = 8
};

// Layers one launch can run back to back (the tensor-core path's fused stack).
constexpr int kMaxFusedLayers = 8;

// Work-unit limits that size the workspace.
constexpr int kBoxRows = 32;           // weight rows per TMA box (one output tile)
constexpr int kBoxColsMax = 256;       // K elements per TMA box
constexpr int kActGroup = 4;           // token rows per activation group (CUDA-core pass)
constexpr int kDownPairsPerSplit = 2;  // (expert, row-group) pairs per down split
constexpr int kPartialFloats = 2 * kBoxRows * kActGroup;  // floats per unit partial
constexpr int kMaxE = 1024;
constexpr int kMaxSlots = 1024;        // batch * top_k
constexpr int kMaxTopK = 32;

// Tensor-core path geometry.
constexpr int kTcRows = 128;      // M of one tcgen05 tile (weight rows)
constexpr int kTcAtomK = 64;      // K elements of one 128-byte swizzle atom
constexpr int kTcActRows = 16;    // activation rows per TMA box (MMA N granule)
constexpr int kTcMaxN = 64;       // token columns of one tile (max batch)
constexpr int kTcSharedSplits = 4;
constexpr int kTcExpertSplits = 4;

constexpr int kTcRouterSplits = 28;

// K splits of a router tile pair on the tensor-core path: short units (4 K atoms of
// the 7168-wide layer), so the router finishes soon after the normalised rows exist;
// each token row's owner CTA sums its row's partials.
__host__ __device__ inline int tc_router_splits(int B, int nk_atoms) {
  (void)B;
  return kTcRouterSplits < nk_atoms ? kTcRouterSplits : nk_atoms;
}
__host__ __device__ inline int tc_clamp_splits(int s, int nk_atoms) { return s < nk_atoms ? s : nk_atoms; }

// K splits of the shared expert's gate/up tiles on the tensor-core path: short units
// while the batch is small; whole-K units (no fix-up over batch x splits partial sums)
// once the batch is large.
__host__ __device__ inline int tc_shared_splits(int B, int nk_atoms) {
  return tc_clamp_splits(B <= 16 ? kTcSharedSplits : 1, nk_atoms);
}

// K splits of an expert's gate/up tiles on the tensor-core path, by the number of
// token rows that chose the expert: a hot expert streams as whole-K units (no fix-up
// of its many rows), a cold one in short units that spread over the SMs.
__host__ __device__ inline int tc_expert_splits(int rows, int nk_atoms) {
  const int s = rows >= 16 ? 1 : rows >= 4 ? 2 : kTcExpertSplits;
  return s < nk_atoms ? s : nk_atoms;
}

struct Params {
  // shapes of this step
  int H, E, I, Is, B, k;
  float eps;
  int tc;          // 1: tensor-core path (tcgen05 tiles), 0: CUDA-core path
  int RS, SS;      // tensor-core path: K splits of router / shared gate-up units (experts: by row count)
  // activations
  const uint16_t* x;  // bf16 [B][H]
  uint16_t* y;        // bf16 [B][H]
  // expert parallelism (tensor-core path): the step schedules only the selected experts e
  // with ep_e0 <= e < ep_e1, whose weights sit at index e - ep_wbase of the expert arrays;
  // with y_part set, row b's output is the fp32 partial sum_{local j} w_j E_j(n_b), plus
  // x_b + s_b when ep_rs, written to y_part instead of y. A whole-layer step: 0, E, 0,
  // nullptr, 1.
  int ep_e0, ep_e1, ep_wbase, ep_rs;
  float* y_part;      // fp32 [B][H] or nullptr
  // this layer's parameters
  const CUtensorMap* tmaps;  // TM_COUNT maps in global memory
  const uint16_t* gamma;     // bf16 [H]
  const float* bias;         // fp32 [E] or nullptr
  int fp8;                   // 1: expert weights are E4M3 codes (TM_Q_*) with block scales below
  const float* sc_gate;      // fp32 [E][I/128][H/128]: 2^s of each 128 x 128 block
  const float* sc_up;        // fp32 [E][I/128][H/128]
  const float* sc_down;      // fp32 [E][H/128][I/128]
  // workspace
  uint16_t* n;           // bf16 [maxB][H]
  float* logits;         // fp32 [maxB][E]
  uint16_t* hs;          // bf16 [maxB][Is]
  uint16_t* he;          // bf16 [maxSlots][I]
  float* partial;        // fp32 [max_units][kPartialFloats] (CUDA-core path)
  // tensor-core path split-K partial sums (fp32)
  float* rpart;          // [RS][B][E]
  float* spart;          // [SS][B][Is/128][256]
  float* epart;          // [ES][B*k][I/128][256]
  float* dpart;          // [B*k + B][H]: down outputs of expert slot rows, then shared rows
  uint64_t* tk_pub;      // [B][k][2] published top-k choices of each row: the words
                         // (tag << 32 | expert) and (tag << 32 | softmax weight bits)
  uint32_t* row_tix;     // [H/256 tile pairs][max_batch]: down contributions arrived per row
  unsigned row_tix_count;
  uint32_t* ctr;         // [CTR_COUNT] this layer's counters
  uint32_t* gctr;        // the launch's counter block (CTR_EXIT, CTR_ABORT, CTR_EPOCH); == ctr
                         // when the launch runs one layer
  int layer;             // index of this layer within its launch (tags its published choices)
  const uint32_t* rows_in;  // fused stack, layer >= 1: per token row, the previous layer's tile
                            // pairs of output combined (the row is input once all H/256 are)
  uint32_t* rows_out;       // fused stack, all layers but the last: this layer's per-row count
  uint32_t* tickets;     // [max_tiles]
  uint32_t* pair_done;   // [kMaxSlots]
  int* status;           // device status word
  unsigned max_units, max_tiles;
  unsigned cap_slots;       // max_batch x top_k_max: slot rows the workspace holds per split
  unsigned cap_dpart_rows;  // rows of dpart (slot rows + max_batch)
  // debug outputs (nullable)
  float* dbg_logits;
  int* dbg_idx;
  float* dbg_w;
  int* dbg_nuniq;
  unsigned flags;        // bit 0: jitter, bit 1: withhold the n-ready signal
  unsigned long long wait_ns;
  unsigned long long* trace;  // nullable: [gridDim.x][kTraceSlots] timeline (see TraceSlot)
};

// Parameters of a launch that runs L layers back to back (tensor-core path).
struct FusedParams {
  Params layer[kMaxFusedLayers];
  int L;
};

// Per-CTA timeline of one launch (global-timer ns stamps; *_CYC slots are clock64 sums).
enum TraceSlot {
  TR_START = 0,         // kernel start
  TR_NREADY = 1,        // producer acquired the normalised rows
  TR_SCHED = 2,         // producer saw the routing schedule
  TR_FIRST_EXPERT = 3,  // producer issued its first expert gate/up stage
  TR_FIRST_DOWN = 4,    // producer issued its first down stage
  TR_PROD_END = 5,      // producer issued its last stage
  TR_MAC_END = 6,       // MAC warps consumed the last stage
  TR_EPI_END = 7,       // epilogue warp finished its last unit
  TR_EXIT = 8,          // CTA done
  TR_PROD_WAIT_SLOT_CYC = 9,   // producer cycles waiting for a free ring slot
  TR_PROD_WAIT_DEP_CYC = 10,   // producer cycles waiting for activations to be published
  TR_PROD_GRAB_CYC = 11,       // producer cycles waiting for the queue's next unit
  TR_MAC_WAIT_FULL_CYC = 12,   // MAC warp 0 cycles waiting for a stage
  TR_MAC_WAIT_RB_CYC = 13,     // MAC warp 0 cycles waiting for a free result buffer
  TR_EPI_BUSY_CYC = 14,        // epilogue warp cycles inside unit epilogues
  TR_UNITS = 15,               // units this CTA processed
  TR_MAC_COMPUTE_CYC = 16,     // MAC warp 0 cycles in the stage arithmetic
  TR_MAC_STAGES = 17,          // stages MAC warp 0 consumed
  TR_PROD_ISSUE_CYC = 18,      // producer cycles issuing stages (waits excluded)
  TR_PROD_STAGES = 19,         // stages the producer issued
  TR_MAC_SCHED_CYC = 20,       // MAC warp 0 cycles building the schedule
  TR_MAC_REDUCE_CYC = 21,      // MAC warp 0 cycles in reductions and result hand-off
  TR_MAC_LOOP_CYC = 22,        // MAC warp 0 cycles in the stage loop in total
  TR_PROD_SETUP_CYC = 23,      // producer cycles decoding units and building segment contexts
  TR_PROD_SCHED_CYC = 24,      // producer cycles waiting for the routing schedule
  TR_PROD_LOOP_CYC = 25,       // producer cycles in its unit loop in total
  TR_ROUTER_SEEN = 26,         // MAC warps observed all router tiles finished (stamp)
  TR_SCHED_BUILT = 27,         // MAC warps finished the schedule (stamp)
  TR_TOPK_DONE = 28,           // schedule: this CTA's top-k rows done (stamp)
  TR_TOPK_SYNCED = 29,         // schedule: all MAC warps past the top-k (stamp)
  TR_UNIQUE_DONE = 30,         // schedule: unique-expert list and pairs done (stamp)
  TR_N_PUBLISHED = 31,         // a normalised row published by this CTA (stamp)
  TR_TOPK_LOADED = 32,         // schedule: first top-k row's logits loaded (stamp)
  TR_TOPK_SELECTED = 33,       // schedule: first top-k row's selection rounds done (stamp)
  TR_TOPK_CHOSEN = 34,         // tensor-core path: owned row's top-k chosen (stamp)
  TR_TOPK_CYC = 35,            // tensor-core path: cycles of the owned row's top-k selection
  TR_SCHED_PLACED = 36,        // tensor-core path: unique experts placed (stamp)
  TR_SCHED_SORTED = 37,        // tensor-core path: pairs sorted and counted (stamp, warp 0)
  TR_START_CLK = 38,           // clock64 at kernel start (on the tensor-core path the routing
                               // stamps, slots 26-30, 32-34 and 36-37, are clock64 values)
  TR_ROLES = 40,               // warp roles start, after the set-up rendezvous (stamp)
  TR_FIRST_TMA = 41,           // producer issued its first weight tile (stamp)
  TR_NORM_SUMMED = 42,         // RMSNorm: first row's x and gamma loaded and squares summed (stamp)
  TR_NORM_REDUCED = 43,        // RMSNorm: the row's sum of squares known to every routing warp (stamp)
  TR_NORM_STORED = 44,         // RMSNorm: the row's n stored and fenced (stamp)
  TR_CONV_WAIT_CYC = 45,       // FP8 converter warp 0 cycles waiting for stages
  TR_CONV_WORK_CYC = 46,       // FP8 converter warp 0 cycles converting
  TR_MMA_WAIT_CONV_CYC = 47,   // MMA warp cycles waiting for converted FP8 stages
  kTraceSlots = 48
};

constexpr unsigned kFlagJitter = 1u;
constexpr unsigned kFlagWithholdNReady = 2u;
// Bounds-checked build only: after the schedule is built, row 0's first choice points at
// the first slot row past the schedule (inside the workspace, so an unchecked read
// stays in bounds); the combine's check must report MOE_ERR_BOUNDS.
constexpr unsigned kFlagBadSlot = 4u;

}  // namespace moe
