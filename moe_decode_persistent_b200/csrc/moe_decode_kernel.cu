// moe_decode_kernel.cu - the persistent sm_100a kernels of one MoE decode-layer step.
//
// One launch per layer, one CTA per SM (cooperative launch, all CTAs
// co-resident). The pages this follows replace a chain of per-layer kernels by
// one persistent kernel that keeps the GPU streaming (page "Kimi K3推理吞吐提升
// 1.68倍", section "为什么解码阶段适合Megakernel"; page post.smzdm.com/p/a6zppe4g,
// section "改了什么：每层 23 个 kernel 砍到 13 个": 23 -> 13 kernels per layer).
//
// Instances of moe_decode_layer_kernel<trace, tc, fp8, ep> implement the step; the host
// picks one per step (the batch-shape switch; fp8 for a handle with FP8 experts; ep for
// a handle over a range of the experts, whose step yields its fp32 part of the output):
//
// Tensor-core kernel (tc = true, 14 warps)
//   warp 0      producer: takes units of work from a global queue and streams, per
//               64-column K atom, up to two 128-row weight tiles and the activation
//               operand (all 128-byte swizzled TMA boxes) into a shared-memory ring.
//   warps 1-8   routing: RMSNorm of the CTA's rows; for the row the CTA owns, the sum
//               of the router's K-split partials, the top-k and the softmax, published;
//               then the schedule every CTA builds from the published choices.
//   warp 9      MMA issuer: owns 512 tensor-memory columns; one lane issues
//               tcgen05.mma (M = 128 weight rows, N = the token rows, K = 16, bf16,
//               fp32 accumulate) per stage and commits the slot back to the producer.
//   warps 10-13 epilogue: read the accumulators (tcgen05.ld, one warp per lane
//               quadrant) and finish the unit: split-K partials and fix-ups, SwiGLU,
//               down partials and the per-row combine with the residual.
//   FP8 experts (fp8 = true): the producer streams the expert tiles as E4M3 codes and
//               their block scales; once the schedule is built the routing warps turn
//               each stage into bf16 weights in tensor memory, which the MMA reads as
//               its A operand (the bf16 instance has none of this code).
//
// CUDA-core kernel (tc = false, 10 warps)
//   warp 0      producer: 32-row weight boxes and the activation rows (1-D bulk copies).
//   warps 1-8   MAC warps: fp32-FMA GEMV over each stage (each warp 4 weight rows of a
//               box, each lane 8 K columns), warp-shuffle reductions; RMSNorm and the
//               routing schedule (every CTA computes every row's top-k).
//   warp 9      epilogue: split-K partials, tickets, fixed-order fix-ups, outputs.
//
// Units of work (queue order): router, shared gate/up (and, on the tensor-core path,
// the shared expert's down tiles) -- all streamed while the routing resolves (page
// post.smzdm.com/p/a6zppe4g, same section: the shared expert moved beside the router
// computation) -- then expert gate/up and down units over the unique selected experts
// only (each selected expert's weights stream once however many rows chose it). A
// stack of layers runs in one launch on the tensor-core path: CTAs that run out of one
// layer's work arm the next layer's first weight tiles while the layer drains. (The
// same section's L2 prefetch of the next layer's weights was measured here and did not
// pay: it is not done.)
//
// Memory ordering: data produced inside the kernel (normalised rows, logits, h,
// partials, published choices) is read only after an acquire on the counter that
// publishes it, and never through the non-coherent path -- except a one-row step's
// top-k choices, which are polled directly: each is an 8-byte word that carries the
// launch's tag beside its value, valid once the tag matches; only static weights are
// loaded ahead of a wait (the pages' review finding: page "vLLM 合併 Kimi K3 專用解碼…",
// section "AI 寫的 GPU 核心 vLLM 怎麼驗證正確"). Every wait, between CTAs and between
// warps of a CTA, is bounded; when one runs out the kernel records MOE_ERR_TIMEOUT, all
// CTAs unwind, drain their bulk copies and MMAs, and exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "kernel_params.h"
#include "moe_decode.h"
#include "ptx.cuh"

namespace moe {

constexpr int kMacWarps = 8;
constexpr int kMacThreads = 32 * kMacWarps;
constexpr int kThreads = 32 * (kMacWarps + 2);
constexpr int kRowsPerWarp = kBoxRows / kMacWarps;                // 4
constexpr int kBoxBytesMax = kBoxRows * kBoxColsMax * 2;          // 16 KB
constexpr int kActSegBytes = kActGroup * kBoxColsMax * 2;         // 2 KB: one K box of <= 4 rows
constexpr int kSlotBytes = 2 * kBoxBytesMax + 2 * kActSegBytes;   // 36 KB
constexpr int kStages = 5;
constexpr int kKSplits = 4;
constexpr int kRB = 4;  // MAC -> epilogue result buffers
constexpr int kCcRingBytes = kStages * kSlotBytes;

// Tensor-core path: warp 0 producer, warps 1-8 RMSNorm + routing schedule, warp 9
// MMA issuer (owns tensor memory), warps 10-13 tensor-memory epilogue (one warp per
// 32-lane quadrant: warp w reads lanes 32 (w % 4) .. 32 (w % 4) + 31).
constexpr int kTcMmaWarp = kMacWarps + 1;
constexpr int kTcEpiWarp0 = kMacWarps + 2;
constexpr int kTcEpiWarps = 4;
constexpr int kTcThreads = 32 * (kTcEpiWarp0 + kTcEpiWarps);       // 448
constexpr int kTcTileBytes = kTcRows * kTcAtomK * 2;               // 16 KB: 128 rows x 64 K
constexpr int kTcActBytes = kTcMaxN * kTcAtomK * 2;                // 8 KB: <= 64 rows x 64 K
constexpr int kTcSlotBytes = 2 * kTcTileBytes + kTcActBytes;       // 40 KB: a slot for 64 token columns
constexpr int kTcRingBytes = 180 * 1024;
// The slot holds the two weight tiles and N x 128 bytes of activations (N = the step's
// token columns, rounded up to 16): the ring fits 5 stages up to 32 columns, 4 above.
// A fifth stage speeds streaming but, before the routing schedule exists, its deeper HBM
// queue delays the routing's own loads: a step of at most 4 rows keeps at most 4 stages
// in flight until the schedule is built (Producer::wait_slot_pre; measured: batch 1
// 156.0 -> 154.9 us, batch 4 451.5 -> 442.4 us against 4 stages throughout).
constexpr int kTcStagesMax = 5;
__host__ __device__ constexpr int tc_slot_bytes(int na) { return 2 * kTcTileBytes + ((na * kTcAtomK * 2 + 1023) / 1024) * 1024; }
// A layer with FP8 experts: an FP8 stage holds one 128-column K block, so its slot takes
// the activations of two K atoms (the second at +na x 128 bytes).
__host__ __device__ constexpr int tc_slot_bytes_fp8(int na) { return 2 * kTcTileBytes + 2 * na * kTcAtomK * 2; }
__host__ __device__ constexpr int tc_stages_in(int ring_bytes, int slot_bytes, int batch) {
  return ring_bytes / slot_bytes < kTcStagesMax ? ring_bytes / slot_bytes : kTcStagesMax;
}
__host__ __device__ constexpr int tc_stages_of(int slot_bytes, int batch) {
  return tc_stages_in(kTcRingBytes, slot_bytes, batch);
}
__host__ __device__ constexpr int tc_stages(int na, int batch) { return tc_stages_of(tc_slot_bytes(na), batch); }
static_assert(tc_stages(16, 1) == 5 && tc_stages(16, 8) == 5 && tc_stages(32, 32) == 5 && tc_stages(64, 64) == 4,
              "ring depths");
constexpr int kTcAccBufs = 4;       // accumulator buffers in tensor memory
constexpr int kTcAccCols = 128;     // columns per buffer: tile 0 at +0, tile 1 at +64
constexpr int kTmemCols = kTcAccBufs * kTcAccCols;  // 512 (a power of two >= 32)
// A layer with FP8 experts keeps 2 accumulator buffers and uses the rest of tensor memory
// as stages of the MMA's A operand: the converted bf16 weight tiles of an FP8 stage (128
// K columns, 128 TMEM columns; tile j at +64 j; row m in lane m, K elements 2c and 2c + 1
// in column c). With at most 32 token columns an accumulator buffer needs only 64 columns
// (tile 1 at +32): 2 x 64 + 3 A stages; with more, 2 x 128 + 2 A stages.
constexpr int kFp8AccBufs = 2;
constexpr int kFp8AStagesMax = 3;
constexpr int kFp8AStageCols = 2 * kTcAtomK;
__host__ __device__ constexpr int fp8_acc_cols(int na) { return na <= 32 ? kTcAccCols / 2 : kTcAccCols; }
__host__ __device__ constexpr int fp8_astages(int na) { return na <= 32 ? 3 : 2; }
static_assert(kFp8AccBufs * kTcAccCols / 2 + 3 * kFp8AStageCols <= kTmemCols &&
                  kFp8AccBufs * kTcAccCols + 2 * kFp8AStageCols <= kTmemCols,
              "FP8 tensor-memory plans");
// The activations of each A stage (two K atoms of na rows, as they lay in the slot) sit in
// front of an FP8 layer's ring, so a slot is free once its codes are converted.
__host__ __device__ constexpr int fp8_act_stage_bytes(int na) { return 2 * na * kTcAtomK * 2; }
__host__ __device__ constexpr int fp8_actbuf_bytes(int na) { return fp8_astages(na) * fp8_act_stage_bytes(na); }

static_assert(kTcSlotBytes % 1024 == 0 && kTcTileBytes % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(kCcRingBytes % 1024 == 0 && kTcRingBytes % 1024 == 0, "ring keeps the state block aligned");

enum UnitType { UT_ROUTER = 0, UT_SHARED = 1, UT_EXPERT = 2, UT_DOWN_SHARED = 3, UT_DOWN_EXPERT = 4 };
// HK_SWITCH (FP8 layers): the CTA's FP8 stages begin; the MMA warp takes them from the
// tensor-memory A stages from now on, and the ring slots are released by the converters.
enum HeaderKind { HK_STAGE = 0, HK_SCHED = 1, HK_END = 2, HK_SWITCH = 3 };

// Written by the producer for every ring slot; everything a MAC warp needs for the
// stage, so the MAC warps never decode units.
struct StageHeader {
  int kind;  // HK_*
  int unit;
  int info;  // bits 0-1 boxes, 2 K-pair, 3-5 activation rows, 6 segment end, 7 unit end,
             // 8 pair index in the unit, 9 first stage of the unit, 16-31 box columns
  int wrow;  // down-expert stages: first slot row of the pair (routing weights); else -1
};

constexpr int kInfoKpair = 1 << 2, kInfoSegEnd = 1 << 6, kInfoUnitEnd = 1 << 7, kInfoFirst = 1 << 9;
// Tensor-core stages: bits 0-1 weight tiles, 2-4 activation boxes of 16 rows (N / 16),
// 5 first stage of the unit (overwrite the accumulator), 6 last stage of the unit.
constexpr int kTcInfoFirst = 1 << 5, kTcInfoLast = 1 << 6;
// Tensor-core stage whose weight tiles arrive as E4M3 codes: one 128-column K block (two
// K atoms) per stage, 16 KB per tile at the start of the slot (tile 1 at +16 KB; 128
// bytes a row, 128-byte swizzled), converted by the routing warps into an A stage in
// tensor memory, which the MMA reads instead of shared memory. The activations of the
// two atoms follow at +32 KB and +32 KB + NA x 128. The codes are counted on
// Smem::wfull of the slot (the activations stay on full). The converters load the
// tiles' block scales themselves: the header's wrow holds tile 0's scale index (gate or
// down array; tile 1 of a gate/up stage: the same index of the up array, of a down
// stage: I / 128 further), and info bit 8 marks a down stage.
constexpr int kTcInfoFp8 = 1 << 7, kTcInfoFp8Down = 1 << 8;
constexpr int kFp8TileBytes = kTcRows * 2 * kTcAtomK;  // 16 KB: 128 rows x 128 codes
constexpr int kCq = 8;                            // entries of the converter queue

// Layout constants of one step (identical in every CTA).
// On the tensor-core path RT and DT count tile pairs (256 rows), ST and IT 128-row
// tiles, and the nkb* fields 64-column K atoms.
struct Shape {
  int B, k, GB;
  int boxH, boxI, boxIs, nkbH, nkbI, nkbIs;
  int RT, ST, IT, DT;
  int RS, SS, ES;
  int NR, NS;
  int spp;  // stages per (expert, row group) pair of a down unit
  int NA;   // tensor-core path: token columns of n- and hs-based tiles (B rounded up to 16)
  int nst, slot_bytes;  // ring stages and slot size
  int kblk;             // 1: FP8 experts (expert gate/up K splits at 128-column K blocks)
  int acc_cols, nas;    // FP8: TMEM columns per accumulator buffer; tensor-memory A stages
  int pre;  // units queued before the routing schedule (no unit before it needs the schedule)
  int router_target, hs_target, pair_target;  // tiles that publish logits / h_s / one pair's h
};

// Routing schedule (identical in every CTA once built).
struct Sched {
  int U, P, S;
  int NE, ND, total, down_splits;
  int16_t slot_expert[kMaxE];     // expert id of unique slot i, ascending
  int16_t slot_cnt[kMaxE];        // rows that chose it
  int16_t slot_base[kMaxE + 1];   // first slot row of unique slot i
  int16_t pair_slot[kMaxSlots];   // unique slot of (expert, row group) pair p
  uint8_t pair_group[kMaxSlots];  // row group of pair p
  uint8_t row_of[kMaxSlots];      // token row of slot row r
  float w_of[kMaxSlots];          // routing weight of slot row r
  int16_t slot_of[kMaxSlots];     // slot row of (token b, choice j) at b * k + j
  // tensor-core path: pairs are the unique experts, hottest first (stable)
  int16_t eslot[kMaxE];           // unique slot of expert e (valid for selected experts)
  int pair_ubase[kMaxSlots + 1];  // first expert gate/up unit of pair p (prefix over pairs)
  uint8_t pair_es[kMaxSlots];     // K splits of pair p's gate/up tiles
};

// Per-CTA state. The stage ring (kCcRingBytes or kTcRingBytes) sits in front of it in
// dynamic shared memory, 1024-byte aligned.
constexpr int kMaxRingStages = kStages > kTcStagesMax ? kStages : kTcStagesMax;
struct Smem {
  uint64_t full[kMaxRingStages];
  uint64_t empty[kMaxRingStages];
  uint64_t sched_bar;       // schedule built (MAC warps -> producer)
  uint64_t mac_bar;         // MAC-warp rendezvous (bounded)
  uint64_t rb_full[kRB];    // MAC warps -> epilogue warp
  uint64_t rb_empty[kRB];   // epilogue warp -> MAC warps
  uint64_t acc_full[kTcAccBufs];   // tensor-core path: MMA warp -> epilogue warps
  uint64_t acc_empty[kTcAccBufs];  // epilogue warps -> MMA warp
  uint64_t mma_bar;                // MMA warp: its last MMAs completed (drain)
  uint64_t epi_bar;                // rendezvous of the tensor-core epilogue warps (bounded)
  uint64_t conv_bar[kTcStagesMax]; // FP8 stage of the slot converted (routing warps -> MMA warp)
  uint64_t cq_full[kCq];           // converter queue: FP8 stages issued (producer -> routing warps)
  uint64_t cq_empty[kCq];
  uint64_t wfull[kTcStagesMax];    // FP8 stage: codes and scales of the slot landed
  uint64_t cdone[kTcStagesMax];    // FP8 stage: the converters are done with the slot (codes, activations)
  int16_t cq_slot[kCq];            // ring slot of the queued stage (-1: no more stages)
  uint8_t cq_par[kCq];             // the slot's wfull parity for that stage
  uint8_t cq_fpar[kCq];            // the slot's full parity (its activations) for that stage
  StageHeader ahdr[kFp8AStagesMax];  // FP8: the header of the stage in each tensor-memory A stage
  StageHeader hdr[kMaxRingStages];
  int rb_unit[kRB];         // unit id of the buffer, or -1 (stop)
  int acc_unit[kTcAccBufs]; // unit id of the accumulator buffer, or -1 (stop)
  uint32_t tmem_base;
  int epi_last;             // tensor-core epilogue: this unit's split completed its tile
  int ncomb;                // tensor-core epilogue: rows whose down combine falls to this unit
  int16_t comb_rows[kTcMaxN];
  int cnt_base[kTcMaxN + 2];  // tensor-core schedule: pairs per row count, then their bases
  uint64_t topk_cand[64];     // tensor-core routing: top-k candidates of the owned row
  int bcast;
  int bcast2;
  int nuniq;
  int16_t chunk_cnt[kMaxE / 32];
  float red_ss[kMacWarps];
  unsigned known_done[kMaxSlots / 32];  // producer: pairs known complete
  Shape sh;
  Sched sc;
  alignas(16) float rb[kRB][2][kBoxRows][kActGroup];   // read as float4 by the epilogue warp
  alignas(16) float fin[2][kBoxRows][kActGroup];       // written as float4
  union alignas(16) {
    struct {
      int topk_idx[kMaxSlots];
      float topk_w[kMaxSlots];
      unsigned long long mask[kMaxE];
    } t;                               // schedule construction
    float yacc[kBoxRows][65];          // down-tile fix-up (epilogue warp)
    uint64_t keys[kMaxE];              // tensor-core path: the owned row's packed top-k keys
  } u;
};

static_assert(kCcRingBytes + sizeof(Smem) + 1024 <= 227 * 1024, "shared memory budget of one CTA");
// The CUDA-core path's result-buffer barriers (rb_full) serve a tensor-core launch with
// FP8 experts as its A-stage barriers: the MMAs that read a tensor-memory A stage
// completed (the two paths never run in one launch).
static_assert(kFp8AStagesMax <= kRB, "A-stage barriers");
__device__ __forceinline__ uint64_t* astage_empty(Smem& sm) { return sm.rb_full; }
static_assert(kTcRingBytes + sizeof(Smem) + 1024 <= 227 * 1024, "shared memory budget of one CTA");
static_assert(offsetof(Smem, rb) % 16 == 0 && offsetof(Smem, fin) % 16 == 0, "float4 views of rb / fin");
static_assert(offsetof(Smem, full) % 8 == 0 && offsetof(Smem, rb_full) % 8 == 0 &&
              offsetof(Smem, acc_full) % 8 == 0, "mbarrier alignment");
static_assert(kSlotBytes % 1024 == 0 && kBoxBytesMax % 128 == 0 && kActSegBytes % 16 == 0,
              "TMA / bulk-copy destinations");
static_assert(kRowsPerWarp == 4 && kActGroup == 4, "MAC lane mapping assumes 4 rows x 4 row slots");

struct UnitDesc {
  int type;
  int tile;      // tile within its type
  int ticket;    // global tile id
  int split, nsplit;
  int g;         // row group (router / shared / down-shared)
  int pair;      // expert: the pair; down-expert: first pair
  int npair;     // down-expert
  int kb0, nkb;  // K boxes of this unit (router / gate-up split)
  int nstages;
};

// ---- small helpers -------------------------------------------------------------------

__device__ __forceinline__ float bf2f(uint32_t b16) { return __uint_as_float(b16 << 16); }

__device__ __forceinline__ uint16_t f2bf(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xFFFF0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xFFFF0000u);
  f[4] = __uint_as_float(v.z << 16);
  f[5] = __uint_as_float(v.z & 0xFFFF0000u);
  f[6] = __uint_as_float(v.w << 16);
  f[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

__device__ __forceinline__ float silu(float v) { return v / (1.0f + __expf(-v)); }

__device__ __forceinline__ float ld_cg_f32(const float* p) { return __ldcg(p); }

__device__ __forceinline__ void record_error(const Params& p, int code) {
  atomicCAS(p.status, 0, code);
}

__device__ __forceinline__ void record_abort(const Params& p, int code) {
  record_error(p, code);
  atomicExch(&p.gctr[CTR_ABORT], 1u);
}

__device__ __forceinline__ bool abort_seen(const Params& p) {
  return ld_relaxed_gpu(&p.gctr[CTR_ABORT]) != 0u;
}

// Bounds-checked build (compiled with -DMOE_BOUNDS_CHECK into libmoe_decode_checked.so):
// every global or shared-memory index that the routing schedule produces is checked
// before its access; a failed check records MOE_ERR_BOUNDS, raises the abort flag (every
// CTA unwinds) and the access is skipped. In the product build IDX_OK is `true` and the
// condition is not evaluated.
#ifdef MOE_BOUNDS_CHECK
__device__ __noinline__ bool bounds_fail(const Params& p) {
  record_abort(p, MOE_ERR_BOUNDS);
  return false;
}
#define IDX_OK(p, cond) ((cond) || ::moe::bounds_fail(p))
#else
#define IDX_OK(p, cond) true
#endif


// Bounded wait on an mbarrier phase by one thread (suspended while waiting). Between
// polls the thread sleeps, doubling up to max_sleep_ns, so a waiting warp takes no
// issue slots from the warps that work.
__device__ bool wait_mbar(uint64_t* bar, uint32_t parity, const Params& p, uint32_t max_sleep_ns = 128) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  uint32_t ns = 16;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    __nanosleep(ns);
    ns = ns * 2 < max_sleep_ns ? ns * 2 : max_sleep_ns;
    // the abort flag is a global load (about a microsecond under load): not every poll
    if ((it & 31u) == 31u) {
      if (abort_seen(p)) return false;
      if (globaltimer_ns() - t0 > p.wait_ns) {
        record_abort(p, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait on an mbarrier phase by a whole warp: every lane observes the
// completion itself, lane 0 alone decides to give up, and the result is uniform.
// max_sleep_ns > 0: sleep between polls (doubling up to it); 0: poll without sleeping.
__device__ bool warp_wait(uint64_t* bar, uint32_t parity, const Params& p, int lane, uint32_t max_sleep_ns = 256) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  uint64_t t0 = 0;
  if (lane == 0) t0 = globaltimer_ns();
  uint32_t ns = 16;
  for (uint32_t it = 0;; ++it) {
    const bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    if (max_sleep_ns) {
      __nanosleep(ns);
      ns = ns * 2 < max_sleep_ns ? ns * 2 : max_sleep_ns;
    }
    if ((it & 31u) == 31u) {  // the abort flag is a global load: not every poll
      int stop = 0;
      if (lane == 0) {
        if (abort_seen(p)) {
          stop = 1;
        } else if (globaltimer_ns() - t0 > p.wait_ns) {
          record_abort(p, MOE_ERR_TIMEOUT);
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
}

// Bounded wait until *c >= target (acquire). Single thread.
__device__ bool wait_counter(const uint32_t* c, uint32_t target, const Params& p) {
  if (ld_acquire_gpu(c) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    __nanosleep(64);
    if (ld_acquire_gpu(c) >= target) return true;
    if ((it & 7u) == 7u && abort_seen(p)) return false;
    if (globaltimer_ns() - t0 > p.wait_ns) {
      record_abort(p, MOE_ERR_TIMEOUT);
      return false;
    }
  }
}

// Tag of this layer's published top-k choices: odd, so a zeroed word never carries it,
// and different in consecutive launches (the epoch counts completed launches) and for
// each layer of one launch.
__device__ __forceinline__ uint32_t choice_tag(const Params& p) {
  return ((ld_relaxed_gpu(&p.gctr[CTR_EPOCH]) * (uint32_t)kMaxFusedLayers + (uint32_t)p.layer) << 1) | 1u;
}

// Bounded wait of one warp for the k choices of row 0 (lane j < k polls choice j's two
// tagged words) and their values: a choice is valid once both of its words carry this
// launch's tag, so the load that observes the publication also brings the data (no flag
// followed by a second round trip for what it guards). The result is warp-uniform.
__device__ bool warp_poll_choices(const Params& p, uint32_t tag, int k, int lane, int& e, float& w) {
  const uint64_t* pub = p.tk_pub + 2 * lane;
  uint64_t a = 0ull, c = 0ull;
  bool have = lane >= k;
  uint64_t t0 = 0;
  if (lane == 0) t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    if (!have) {
      ld_relaxed_gpu_v2(pub, a, c);
      have = (uint32_t)(a >> 32) == tag && (uint32_t)(c >> 32) == tag;
    }
    if (__all_sync(0xffffffffu, have)) break;
    __nanosleep(32);
    if ((it & 15u) == 15u) {  // the abort flag is a global load: not every poll
      int stop = 0;
      if (lane == 0) {
        if (abort_seen(p)) {
          stop = 1;
        } else if (globaltimer_ns() - t0 > p.wait_ns) {
          record_abort(p, MOE_ERR_TIMEOUT);
          stop = 1;
        }
      }
      if (__shfl_sync(0xffffffffu, stop, 0)) return false;
    }
  }
  if (lane < k) {
    e = (int)(uint32_t)a;
    w = __uint_as_float((uint32_t)c);
  }
  return true;
}

// Rendezvous of the 8 MAC warps (an mbarrier with bounded waits, polled without sleeping).
__device__ __forceinline__ bool mac_sync(Smem& sm, uint32_t& phase, const Params& p, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(&sm.mac_bar);
  const bool ok = warp_wait(&sm.mac_bar, phase, p, lane, 64);
  phase ^= 1u;
  return ok;
}

__device__ __forceinline__ uint32_t hash32(uint32_t a) {
  a ^= a >> 16;
  a *= 0x7feb352dU;
  a ^= a >> 15;
  a *= 0x846ca68bU;
  a ^= a >> 16;
  return a;
}

// Timeline instrumentation: compiled into the tracing instance of the kernel only.
template <bool kTrace>
__device__ __forceinline__ void trace_stamp(const Params& p, int slot) {
  if (kTrace) p.trace[(size_t)blockIdx.x * kTraceSlots + slot] = globaltimer_ns();
}

template <bool kTrace>
__device__ __forceinline__ void trace_put(const Params& p, int slot, unsigned long long v) {
  if (kTrace) p.trace[(size_t)blockIdx.x * kTraceSlots + slot] = v;
}

template <bool kTrace>
__device__ __forceinline__ long long tclock() {
  return kTrace ? clock64() : 0;
}

// SM-clock stamp (clock64 of this CTA's SM; compare only with TR_START_CLK of the same CTA).
template <bool kTrace>
__device__ __forceinline__ void trace_clk(const Params& p, int slot) {
  if (kTrace) p.trace[(size_t)blockIdx.x * kTraceSlots + slot] = (unsigned long long)clock64();
}

// ---- shape and unit decoding ---------------------------------------------------------------

__device__ void make_shape(const Params& p, Shape& s) {
  s.B = p.B;
  s.k = p.k;
  s.GB = (p.B + kActGroup - 1) / kActGroup;
  s.boxH = p.H < kBoxColsMax ? p.H : kBoxColsMax;
  s.boxI = p.I < kBoxColsMax ? p.I : kBoxColsMax;
  s.boxIs = p.Is < kBoxColsMax ? p.Is : kBoxColsMax;
  s.nkbH = p.H / s.boxH;
  s.nkbI = p.I / s.boxI;
  s.nkbIs = p.Is / s.boxIs;
  s.RT = p.E / kBoxRows;
  s.ST = p.Is / kBoxRows;
  s.IT = p.I / kBoxRows;
  s.DT = p.H / kBoxRows;
  s.RS = s.nkbH < kKSplits ? s.nkbH : kKSplits;
  s.SS = s.RS;
  s.ES = s.RS;
  s.NR = s.GB * s.RT * s.RS;
  s.NS = s.GB * s.ST * s.SS;
  s.spp = (s.nkbI + 1) / 2;
  s.NA = 0;
  s.nst = kStages;
  s.slot_bytes = kSlotBytes;
  s.pre = s.NR + s.NS;
  s.router_target = s.GB * s.RT;
  s.hs_target = s.GB * s.ST;
  s.pair_target = s.IT;
}

// Tensor-core path: router and down units cover a pair of 128-row tiles (the second
// absent when the rows end half-way), shared and expert gate/up units a 128-row tile
// of the gate matrix with the same rows of the up matrix. Every token row of the batch
// is one MMA column (N = B rounded up to 16) except on down-expert units, whose
// columns are the expert's own slot rows.
__device__ void make_shape_tc(const Params& p, Shape& s) {
  s.B = p.B;
  s.k = p.k;
  s.GB = 1;
  s.NA = (p.B + kTcActRows - 1) / kTcActRows * kTcActRows;
  s.kblk = p.fp8 ? 1 : 0;
  s.acc_cols = p.fp8 ? fp8_acc_cols(s.NA) : kTcAccCols;
  s.nas = fp8_astages(s.NA);
  s.slot_bytes = p.fp8 ? tc_slot_bytes_fp8(s.NA) : tc_slot_bytes(s.NA);
  s.nst = p.fp8 ? tc_stages_in(kTcRingBytes - fp8_actbuf_bytes(s.NA), s.slot_bytes, p.B)
                : tc_stages_of(s.slot_bytes, p.B);
  s.boxH = s.boxI = s.boxIs = kTcAtomK;
  s.nkbH = p.H / kTcAtomK;
  s.nkbI = p.I / kTcAtomK;
  s.nkbIs = p.Is / kTcAtomK;
  s.RT = (p.E + 2 * kTcRows - 1) / (2 * kTcRows);
  s.ST = p.Is / kTcRows;
  s.IT = p.I / kTcRows;
  s.DT = (p.H + 2 * kTcRows - 1) / (2 * kTcRows);
  s.RS = p.RS;
  s.SS = p.SS;
  s.ES = 0;  // per expert: sc.pair_es
  s.NR = s.RT * s.RS;
  s.NS = s.ST * s.SS;
  s.spp = 0;
  s.pre = s.NR + s.NS + s.DT;  // the shared expert's down tiles need only h_s
  s.router_target = s.NR;  // every router unit publishes its own partial sums
  s.hs_target = s.ST;
  s.pair_target = s.IT;
}

__device__ __forceinline__ void split_range(int nkb, int nsplit, int s, int& kb0, int& nkb_s) {
  kb0 = (nkb * s) / nsplit;
  nkb_s = (nkb * (s + 1)) / nsplit - kb0;
}

__device__ UnitDesc decode_unit(const Shape& sh, const Sched& sc, int u) {
  UnitDesc d;
  d.npair = 0;
  d.pair = 0;
  d.g = 0;
  d.kb0 = 0;
  d.nkb = 0;
  if (u < sh.NR) {
    d.type = UT_ROUTER;
    d.split = u % sh.RS;
    d.tile = (u / sh.RS) % sh.RT;
    d.g = u / (sh.RS * sh.RT);
    d.nsplit = sh.RS;
    d.ticket = d.g * sh.RT + d.tile;
    split_range(sh.nkbH, sh.RS, d.split, d.kb0, d.nkb);
    d.nstages = (d.nkb + 1) / 2;  // two K boxes per stage
  } else if (u < sh.NR + sh.NS) {
    const int v = u - sh.NR;
    d.type = UT_SHARED;
    d.split = v % sh.SS;
    d.tile = (v / sh.SS) % sh.ST;
    d.g = v / (sh.SS * sh.ST);
    d.nsplit = sh.SS;
    d.ticket = sh.GB * sh.RT + d.g * sh.ST + d.tile;
    split_range(sh.nkbH, sh.SS, d.split, d.kb0, d.nkb);
    d.nstages = d.nkb;  // gate box + up box per stage
  } else if (u < sh.NR + sh.NS + sc.NE) {
    const int v = u - sh.NR - sh.NS;
    d.type = UT_EXPERT;
    d.split = v % sh.ES;
    d.tile = (v / sh.ES) % sh.IT;
    d.pair = v / (sh.ES * sh.IT);
    d.nsplit = sh.ES;
    d.ticket = sh.GB * (sh.RT + sh.ST) + d.pair * sh.IT + d.tile;
    split_range(sh.nkbH, sh.ES, d.split, d.kb0, d.nkb);
    d.nstages = d.nkb;
  } else {
    const int v = u - sh.NR - sh.NS - sc.NE;
    d.tile = v % sh.DT;
    d.split = v / sh.DT;
    d.nsplit = sc.down_splits;
    d.ticket = sh.GB * (sh.RT + sh.ST) + sc.P * sh.IT + d.tile;
    if (d.split < sh.GB) {
      d.type = UT_DOWN_SHARED;
      d.g = d.split;
      d.nkb = sh.nkbIs;
      d.nstages = (sh.nkbIs + 1) / 2;
    } else {
      d.type = UT_DOWN_EXPERT;
      d.pair = (d.split - sh.GB) * kDownPairsPerSplit;
      d.npair = sc.P - d.pair < kDownPairsPerSplit ? sc.P - d.pair : kDownPairsPerSplit;
      d.nstages = d.npair * sh.spp;
    }
  }
  return d;
}

// Tensor-core path unit enumeration (queue order): router (tile pair, K split),
// shared gate/up (tile, K split), shared down (tile pair) -- all before the routing
// schedule -- then expert gate/up ((pair, tile), K split) and expert down (pair, tile
// pair). Down units carry no K split; each row of a down tile pair is combined by the
// unit that brings its last contribution.
__device__ UnitDesc decode_unit_tc(const Shape& sh, const Sched& sc, int u) {
  UnitDesc d;
  d.npair = 0;
  d.pair = 0;
  d.g = 0;
  if (u < sh.NR) {
    d.type = UT_ROUTER;
    d.tile = u / sh.RS;
    d.split = u % sh.RS;
    d.nsplit = sh.RS;
    d.ticket = d.tile;
    split_range(sh.nkbH, sh.RS, d.split, d.kb0, d.nkb);
  } else if (u < sh.NR + sh.NS) {
    const int v = u - sh.NR;
    d.type = UT_SHARED;
    d.tile = v / sh.SS;
    d.split = v % sh.SS;
    d.nsplit = sh.SS;
    d.ticket = sh.RT + d.tile;
    split_range(sh.nkbH, sh.SS, d.split, d.kb0, d.nkb);
  } else if (u < sh.pre) {
    d.type = UT_DOWN_SHARED;
    d.tile = u - sh.NR - sh.NS;
    d.split = 0;
    d.nsplit = 1;
    d.ticket = 0;
    d.kb0 = 0;
    d.nkb = sh.nkbIs;
  } else if (u < sh.pre + sc.NE) {
    // pair p owns units [pair_ubase[p], pair_ubase[p + 1]): its IT tiles x pair_es[p] splits
    const int v = u - sh.pre;
    int lo = 0, hi = sc.P - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sc.pair_ubase[mid] <= v) lo = mid;
      else hi = mid - 1;
    }
    const int es = sc.pair_es[lo];
    const int w = v - sc.pair_ubase[lo];
    d.type = UT_EXPERT;
    d.pair = lo;
    d.split = w % es;
    d.tile = w / es;
    d.nsplit = es;
    d.ticket = sh.RT + sh.ST + lo * sh.IT + d.tile;
    if (sh.kblk) {  // FP8: whole 128-column K blocks
      split_range(sh.nkbH / 2, es, d.split, d.kb0, d.nkb);
      d.kb0 *= 2;
      d.nkb *= 2;
    } else {
      split_range(sh.nkbH, es, d.split, d.kb0, d.nkb);
    }
  } else {
    const int v = u - sh.pre - sc.NE;
    d.type = UT_DOWN_EXPERT;
    d.pair = v / sh.DT;
    d.tile = v % sh.DT;
    d.npair = 1;
    d.split = 0;
    d.nsplit = 1;
    d.ticket = 0;
    d.kb0 = 0;
    d.nkb = sh.nkbI;
  }
  d.nstages = d.nkb;
  return d;
}

// Unit id of split s of the tile that unit d belongs to.
__device__ __forceinline__ int unit_of_split(const Shape& sh, const Sched& sc, const UnitDesc& d,
                                             int s) {
  switch (d.type) {
    case UT_ROUTER: return (d.g * sh.RT + d.tile) * sh.RS + s;
    case UT_SHARED: return sh.NR + (d.g * sh.ST + d.tile) * sh.SS + s;
    case UT_EXPERT: return sh.NR + sh.NS + (d.pair * sh.IT + d.tile) * sh.ES + s;
    default: return sh.NR + sh.NS + sc.NE + s * sh.DT + d.tile;
  }
}

// Token rows of activation group g of the batch, and of pair p.
__device__ __forceinline__ int group_rows(int B, int g) {
  const int c = B - g * kActGroup;
  return c < kActGroup ? c : kActGroup;
}

__device__ __forceinline__ int pair_rows(const Sched& sc, int pr) {
  const int i = sc.pair_slot[pr];
  const int c = sc.slot_cnt[i] - sc.pair_group[pr] * kActGroup;
  return c < kActGroup ? c : kActGroup;
}

__device__ __forceinline__ int pair_first_slot_row(const Sched& sc, int pr) {
  return sc.slot_base[sc.pair_slot[pr]] + sc.pair_group[pr] * kActGroup;
}

// Per-stage geometry shared by producer and MAC warps. A stage holds one or two
// weight boxes: gate and up rows of the same K box (`kpair` 0), or two
// consecutive K boxes of the same rows (`kpair` 1, one activation segment each).
struct StageDesc {
  int nbox;
  int kpair;
  int box_cols;
  int c;     // activation rows
  int pair;  // down-expert: the pair of this stage
  int q;     // down-expert: index of the pair within the unit
  int kb;    // first K box
  int last_of_pair;
};

__device__ __forceinline__ StageDesc stage_desc(const Shape& sh, const Sched& sc, const UnitDesc& d,
                                                int st) {
  StageDesc s;
  s.pair = d.pair;
  s.q = 0;
  s.last_of_pair = 0;
  switch (d.type) {
    case UT_ROUTER:
      s.kpair = 1;
      s.box_cols = sh.boxH;
      s.c = group_rows(sh.B, d.g);
      s.kb = d.kb0 + 2 * st;
      s.nbox = d.kb0 + d.nkb - s.kb < 2 ? 1 : 2;
      break;
    case UT_SHARED:
      s.kpair = 0;
      s.box_cols = sh.boxH;
      s.c = group_rows(sh.B, d.g);
      s.kb = d.kb0 + st;
      s.nbox = 2;
      break;
    case UT_EXPERT:
      s.kpair = 0;
      s.box_cols = sh.boxH;
      s.c = pair_rows(sc, d.pair);
      s.kb = d.kb0 + st;
      s.nbox = 2;
      break;
    case UT_DOWN_SHARED:
      s.kpair = 1;
      s.box_cols = sh.boxIs;
      s.c = group_rows(sh.B, d.g);
      s.kb = 2 * st;
      s.nbox = sh.nkbIs - s.kb < 2 ? 1 : 2;
      break;
    default: {
      s.kpair = 1;
      s.q = st / sh.spp;
      const int local = st % sh.spp;
      s.pair = d.pair + s.q;
      s.box_cols = sh.boxI;
      s.c = pair_rows(sc, s.pair);
      s.kb = 2 * local;
      s.nbox = sh.nkbI - s.kb < 2 ? 1 : 2;
      s.last_of_pair = local == sh.spp - 1;
      break;
    }
  }
  return s;
}

// Producer-side context of one unit (or, for a down-expert unit, of one of its pairs):
// tensor maps, box row, K-box range and the activation rows, computed once.
struct SegCtx {
  const CUtensorMap* tm0;
  const CUtensorMap* tm1;
  int y0;
  int box_cols;
  int kpair;
  int kb0, kb_end;
  int c;
  int wrow;
  int dep;  // 0: normalised rows, 1: shared h, 2: the pair's h
  int pair;
  const uint16_t* abase;     // activation matrix
  uint32_t aoff[kActGroup];  // element offsets of the activation rows
};

__device__ __forceinline__ void make_seg(const Params& p, const Shape& sh, const Sched& sc, const UnitDesc& d,
                                         int q, SegCtx& x) {
  x.wrow = -1;
  x.pair = d.pair;
  switch (d.type) {
    case UT_ROUTER:
    case UT_SHARED: {
      const bool r = d.type == UT_ROUTER;
      x.tm0 = &p.tmaps[r ? TM_WR : TM_WSG];
      x.tm1 = &p.tmaps[r ? TM_WR : TM_WSU];
      x.y0 = d.tile * kBoxRows;
      x.box_cols = sh.boxH;
      x.kpair = r ? 1 : 0;
      x.kb0 = d.kb0;
      x.kb_end = d.kb0 + d.nkb;
      x.c = group_rows(sh.B, d.g);
      x.dep = 0;
      x.abase = p.n;
#pragma unroll
      for (int j = 0; j < kActGroup; ++j) x.aoff[j] = (uint32_t)((d.g * kActGroup + (j < x.c ? j : 0)) * p.H);
      break;
    }
    case UT_EXPERT: {
      int e = sc.slot_expert[sc.pair_slot[d.pair]];
      int r0 = pair_first_slot_row(sc, d.pair);
      if (!IDX_OK(p, (unsigned)e < (unsigned)p.E && (unsigned)(r0 + kActGroup) <= (unsigned)kMaxSlots))
        e = r0 = 0;  // reported; the step is abandoned, the copies stay in bounds
      x.tm0 = &p.tmaps[TM_WG];
      x.tm1 = &p.tmaps[TM_WU];
      x.y0 = e * p.I + d.tile * kBoxRows;
      x.box_cols = sh.boxH;
      x.kpair = 0;
      x.kb0 = d.kb0;
      x.kb_end = d.kb0 + d.nkb;
      x.c = pair_rows(sc, d.pair);
      x.dep = 0;
      x.abase = p.n;
#pragma unroll
      for (int j = 0; j < kActGroup; ++j) {
        int b = sc.row_of[r0 + (j < x.c ? j : 0)];
        if (!IDX_OK(p, b < p.B)) b = 0;
        x.aoff[j] = (uint32_t)(b * p.H);
      }
      break;
    }
    case UT_DOWN_SHARED:
      x.tm0 = x.tm1 = &p.tmaps[TM_WSD];
      x.y0 = d.tile * kBoxRows;
      x.box_cols = sh.boxIs;
      x.kpair = 1;
      x.kb0 = 0;
      x.kb_end = sh.nkbIs;
      x.c = group_rows(sh.B, d.g);
      x.dep = 1;
      x.abase = p.hs;
#pragma unroll
      for (int j = 0; j < kActGroup; ++j) x.aoff[j] = (uint32_t)((d.g * kActGroup + (j < x.c ? j : 0)) * p.Is);
      break;
    default: {
      const int pr = d.pair + q;
      int e = sc.slot_expert[sc.pair_slot[pr]];
      int r0 = pair_first_slot_row(sc, pr);
      if (!IDX_OK(p, (unsigned)e < (unsigned)p.E && (unsigned)(r0 + kActGroup) <= (unsigned)kMaxSlots))
        e = r0 = 0;  // reported; the step is abandoned, the copies stay in bounds
      x.pair = pr;
      x.tm0 = x.tm1 = &p.tmaps[TM_WD];
      x.y0 = e * p.H + d.tile * kBoxRows;
      x.box_cols = sh.boxI;
      x.kpair = 1;
      x.kb0 = 0;
      x.kb_end = sh.nkbI;
      x.c = pair_rows(sc, pr);
      x.wrow = r0;
      x.dep = 2;
      x.abase = p.he;
#pragma unroll
      for (int j = 0; j < kActGroup; ++j) x.aoff[j] = (uint32_t)((r0 + (j < x.c ? j : 0)) * p.I);
      break;
    }
  }
}

// ---- MAC warps: math ---------------------------------------------------------------------------

// One stage: box m's rows (warp + 8 r) times the activation rows of its segment.
// KPAIR 0: box 0 -> acc[0] (gate), box 1 -> acc[1] (up), one activation segment.
// KPAIR 1: both boxes -> acc[0], box m uses activation segment m.
template <int KPAIR, int NBOX, int CP>
__device__ __forceinline__ void mac_stage(const uint8_t* slot, int box_cols, int c,
                                          float (&acc)[2][kRowsPerWarp][kActGroup], int warp,
                                          int lane) {
  const int row_bytes = box_cols * 2;
  const int colb = lane * 16;
  if (colb >= row_bytes) return;
  const uint8_t* act = slot + 2 * kBoxBytesMax;
  float a[CP][8];
#pragma unroll
  for (int m = 0; m < NBOX; ++m) {
    if (m == 0 || KPAIR) {
      const uint8_t* seg = act + (KPAIR ? m : 0) * kActSegBytes;
#pragma unroll
      for (int j = 0; j < CP; ++j) {
        if (j < c) {
          const uint4 v = *reinterpret_cast<const uint4*>(seg + j * row_bytes + colb);
          unpack8(v, a[j]);
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) a[j][t] = 0.0f;
        }
      }
    }
    const int am = KPAIR ? 0 : m;
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const uint4 wv = *reinterpret_cast<const uint4*>(slot + m * kBoxBytesMax +
                                                       (warp + kMacWarps * r) * row_bytes + colb);
      float w[8];
      unpack8(wv, w);
#pragma unroll
      for (int j = 0; j < CP; ++j) {
#pragma unroll
        for (int t = 0; t < 8; ++t) acc[am][r][j] = fmaf(w[t], a[j][t], acc[am][r][j]);
      }
    }
  }
}

template <int KPAIR, int NBOX>
__device__ __forceinline__ void mac_cp(const uint8_t* slot, int box_cols, int c,
                                       float (&acc)[2][kRowsPerWarp][kActGroup], int warp, int lane) {
  if (c <= 1) mac_stage<KPAIR, NBOX, 1>(slot, box_cols, c, acc, warp, lane);
  else if (c <= 2) mac_stage<KPAIR, NBOX, 2>(slot, box_cols, c, acc, warp, lane);
  else mac_stage<KPAIR, NBOX, kActGroup>(slot, box_cols, c, acc, warp, lane);
}

__device__ __forceinline__ void mac_dispatch(const uint8_t* slot, int kpair, int nbox, int box_cols, int c,
                                             float (&acc)[2][kRowsPerWarp][kActGroup], int warp,
                                             int lane) {
  if (kpair) {
    if (nbox == 2) mac_cp<1, 2>(slot, box_cols, c, acc, warp, lane);
    else mac_cp<1, 1>(slot, box_cols, c, acc, warp, lane);
  } else {
    mac_cp<0, 2>(slot, box_cols, c, acc, warp, lane);
  }
}

__device__ __forceinline__ void zero_acc(float (&acc)[2][kRowsPerWarp][kActGroup]) {
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
      for (int j = 0; j < kActGroup; ++j) acc[m][r][j] = 0.0f;
}

// Warp-reduce the 32 accumulators acc[m][r][j] (value v = m*16 + r*4 + j) with a
// butterfly reduce-scatter: 31 shuffles in 5 dependent steps, after which lane L
// holds the full sum of value L. Lanes holding values of boxes [0, nacc) store
// (m, row = warp + 8 r, j) into dst[m0 + m][row][j]; `wscale` (nullable) scales j.
__device__ __forceinline__ void reduce_to(float (&acc)[2][kRowsPerWarp][kActGroup], int nacc,
                                          float (*dst)[kBoxRows][kActGroup], int m0,
                                          const float* wscale, int c, int warp, int lane) {
  float v[32];
#pragma unroll
  for (int m = 0; m < 2; ++m)
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
      for (int j = 0; j < kActGroup; ++j) v[m * 16 + r * 4 + j] = acc[m][r][j];
#pragma unroll
  for (int half = 16; half >= 1; half >>= 1) {
    const bool upper = (lane & half) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float keep = upper ? v[half + i] : v[i];
      const float send = upper ? v[i] : v[half + i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, half);
    }
  }
  const int m = lane >> 4, r = (lane >> 2) & 3, j = lane & 3;
  if (m < nacc) {
    float out = v[0];
    if (wscale) out = j < c ? out * wscale[j] : 0.0f;
    dst[m0 + m][warp + kMacWarps * r][j] = out;
  }
}

// ---- routing schedule (MAC warps, every CTA) ---------------------------------------------

// Order-preserving 32-bit key of a finite float (larger float -> larger key; -0 and +0
// map to the same key, so they tie like equal floats).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f == 0.0f ? 0.0f : f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-k of one row by one warp: the k largest logits, ties to the lower expert index,
// then softmax over the selected logits. Each round takes the warp-wide maximum key
// (redux.sync) and, among lanes holding it, the lowest expert index (redux.sync).
template <bool kTrace>
__device__ void warp_topk_row(const Params& p, Smem& sm, int b, int lane) {
  const int E = p.E, k = p.k;
  const int nq = E / 32;
  uint32_t key[kMaxE / 32];
  bool bad = false;
#pragma unroll
  for (int q = 0; q < kMaxE / 32; ++q) {
    key[q] = 0u;  // below every finite key: never selected while a real value remains
    if (q < nq) {
      const float t = ld_cg_f32(&p.logits[(size_t)b * E + lane + 32 * q]);
      if (!isfinite(t)) bad = true;
      else key[q] = float_key(t);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(p, MOE_ERR_NONFINITE);
  if (b == 0 && lane == 0) trace_stamp<kTrace>(p, TR_TOPK_LOADED);
  uint32_t taken = 0;
  int my_idx = 0;
  for (int j = 0; j < k; ++j) {
    // lane-local best: largest key, lowest q (= lowest expert index) among equals
    uint32_t bk = 0u;
    int bq = -1;
#pragma unroll
    for (int q = 0; q < kMaxE / 32; ++q) {
      if (q < nq && !((taken >> q) & 1u) && (bq < 0 || key[q] > bk)) {
        bk = key[q];
        bq = q;
      }
    }
    const uint32_t kmax = __reduce_max_sync(0xffffffffu, bq >= 0 ? bk : 0u);
    const uint32_t cand = (bq >= 0 && bk == kmax) ? (uint32_t)(lane + 32 * bq) : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, cand);
    if ((int)(win & 31u) == lane) taken |= 1u << (win >> 5);
    if (lane == j) my_idx = (int)win;
  }
  if (b == 0 && lane == 0) trace_stamp<kTrace>(p, TR_TOPK_SELECTED);
  const float my_val = lane < k ? ld_cg_f32(&p.logits[(size_t)b * E + my_idx]) : 0.0f;
  const float mx = __shfl_sync(0xffffffffu, my_val, 0);
  const float ex = lane < k ? expf(my_val - mx) : 0.0f;
  float z = ex;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  if (lane < k) {
    sm.u.t.topk_idx[b * k + lane] = my_idx;
    sm.u.t.topk_w[b * k + lane] = ex / z;
    atomicOr(&sm.u.t.mask[my_idx], 1ull << b);
  }
}

// Builds sm.sc from the final logits (CUDA-core path). Called by all MAC warps; false
// on abort. An expert's rows form (expert, row group) pairs of up to kActGroup rows.
template <bool kTrace>
__device__ bool build_schedule(const Params& p, Smem& sm, int mw, int lane, uint32_t& mphase) {
  constexpr int kGroup = kActGroup;
  const Shape& sh = sm.sh;
  Sched& sc = sm.sc;
  const int mtid = mw * 32 + lane;
  if (mw == 0) {
    int ok = 1;
    if (lane == 0) ok = wait_counter(&p.ctr[CTR_ROUTER], (uint32_t)sh.router_target, p) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (lane == 0) sm.bcast = ok;
  }
  for (int e = mtid; e < p.E; e += kMacThreads) sm.u.t.mask[e] = 0ull;
  if (!mac_sync(sm, mphase, p, lane)) return false;
  if (!sm.bcast) return false;
  if (mtid == 0) trace_stamp<kTrace>(p, TR_ROUTER_SEEN);
  for (int b = mw; b < p.B; b += kMacWarps) warp_topk_row<kTrace>(p, sm, b, lane);
  if (mtid == 0) trace_stamp<kTrace>(p, TR_TOPK_DONE);
  if (!mac_sync(sm, mphase, p, lane)) return false;
  if (mtid == 0) trace_stamp<kTrace>(p, TR_TOPK_SYNCED);
  // unique experts in ascending id: per-chunk counts by all MAC warps, then placement
  const int nchunk = p.E / 32;
  for (int ch = mw; ch < nchunk; ch += kMacWarps) {
    const uint32_t bal = __ballot_sync(0xffffffffu, sm.u.t.mask[ch * 32 + lane] != 0ull);
    if (lane == 0) sm.chunk_cnt[ch] = (int16_t)__popc(bal);
  }
  if (!mac_sync(sm, mphase, p, lane)) return false;
  {
    // exclusive prefix of the chunk counts (each warp computes it; kMaxE / 32 <= 32 chunks)
    const int cnt = lane < nchunk ? sm.chunk_cnt[lane] : 0;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    for (int ch = mw; ch < nchunk; ch += kMacWarps) {
      const int chbase = __shfl_sync(0xffffffffu, incl - cnt, ch);
      const unsigned long long m = sm.u.t.mask[ch * 32 + lane];
      const uint32_t bal = __ballot_sync(0xffffffffu, m != 0ull);
      if (m != 0ull) {
        const int pos = chbase + __popc(bal & ((1u << lane) - 1u));
        sc.slot_expert[pos] = (int16_t)(ch * 32 + lane);
        sc.slot_cnt[pos] = (int16_t)__popcll(m);
      }
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (mw == 0 && lane == 0) sm.nuniq = total;
  }
  if (!mac_sync(sm, mphase, p, lane)) return false;
  if (mw == 0) {
    const int U = sm.nuniq;
    __syncwarp();
    // slot bases and (expert, row group) pairs
    int rbase = 0, pbase = 0;
    for (int i0 = 0; i0 < U; i0 += 32) {
      const int i = i0 + lane;
      const int c = i < U ? sc.slot_cnt[i] : 0;
      const int gcount = (c + kGroup - 1) / kGroup;
      int cs = c, gs = gcount;  // inclusive scans
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int tc = __shfl_up_sync(0xffffffffu, cs, off);
        const int tg = __shfl_up_sync(0xffffffffu, gs, off);
        if (lane >= off) {
          cs += tc;
          gs += tg;
        }
      }
      if (i < U) {
        sc.slot_base[i] = (int16_t)(rbase + cs - c);
        const int pb = pbase + gs - gcount;
        for (int g = 0; g < gcount; ++g) {
          sc.pair_slot[pb + g] = (int16_t)i;
          sc.pair_group[pb + g] = (uint8_t)g;
        }
      }
      rbase += __shfl_sync(0xffffffffu, cs, 31);
      pbase += __shfl_sync(0xffffffffu, gs, 31);
    }
    if (lane == 0) {
      sc.U = U;
      sc.S = rbase;
      sc.slot_base[U] = (int16_t)rbase;
      sc.P = pbase;
      sc.NE = pbase * sh.IT * sh.ES;
      sc.down_splits = sh.GB + (pbase + kDownPairsPerSplit - 1) / kDownPairsPerSplit;
      sc.ND = sh.DT * sc.down_splits;
      sc.total = sh.NR + sh.NS + sc.NE + sc.ND;
      const unsigned tiles = (unsigned)(sh.GB * (sh.RT + sh.ST) + pbase * sh.IT + sh.DT);
      sm.bcast2 = ((unsigned)sc.total <= p.max_units && tiles <= p.max_tiles && pbase <= kMaxSlots) ? 1 : 0;
      if (!sm.bcast2) record_abort(p, MOE_ERR_UNSUPPORTED_SHAPE);
    }
  }
  if (mtid == 0) trace_stamp<kTrace>(p, TR_UNIQUE_DONE);
  if (!mac_sync(sm, mphase, p, lane)) return false;
  if (!sm.bcast2) return false;
  // token rows and routing weights of every slot row (rows ascending within an expert)
  for (int i = mtid; i < sc.U; i += kMacThreads) {
    const int e = sc.slot_expert[i];
    if (!IDX_OK(p, (unsigned)e < (unsigned)p.E)) continue;
    unsigned long long m = sm.u.t.mask[e];
    int r = sc.slot_base[i];
    while (m) {
      const int b = __ffsll((long long)m) - 1;
      m &= m - 1ull;
      if (!IDX_OK(p, (unsigned)r < (unsigned)kMaxSlots)) break;
      float w = 0.0f;
      for (int j = 0; j < p.k; ++j)
        if (sm.u.t.topk_idx[b * p.k + j] == e) {
          w = sm.u.t.topk_w[b * p.k + j];
          sc.slot_of[b * p.k + j] = (int16_t)r;
        }
      sc.row_of[r] = (uint8_t)b;
      sc.w_of[r] = w;
      ++r;
    }
  }
  if (blockIdx.x == 0) {
    for (int t = mtid; t < p.B * p.k; t += kMacThreads) {
      if (p.dbg_idx) p.dbg_idx[t] = sm.u.t.topk_idx[t];
      if (p.dbg_w) p.dbg_w[t] = sm.u.t.topk_w[t];
    }
    if (mtid == 0 && p.dbg_nuniq) *p.dbg_nuniq = sc.U;
  }
  const bool ok = mac_sync(sm, mphase, p, lane);
  if (mtid == 0) trace_stamp<kTrace>(p, TR_SCHED_BUILT);
  return ok;
}

// ---- tensor-core path: routing (MAC warps, i.e. warps 1-8) -------------------------------------

__device__ __forceinline__ uint64_t umax64(uint64_t a, uint64_t b) { return a > b ? a : b; }

__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
  const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
  const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
  return ((uint64_t)hi << 32) | lo;
}

// Inverse of float_key.
__device__ __forceinline__ float key_float(uint32_t key) {
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Packed top-k key of logit t of expert e: (order key << 32) | ~e. The largest packed
// key is the largest logit with the lowest index among equals; all packed keys
// differ; 0 (a non-finite logit) is below every finite key.
__device__ __forceinline__ uint64_t topk_key(float t, int e) {
  return isfinite(t) ? (((uint64_t)float_key(t) << 32) | (uint64_t)(~(uint32_t)e)) : 0ull;
}

// Top-k of one row by one warp from its packed keys in shared memory (keys[0..E),
// E a multiple of 32, k <= 32): the k largest, ties to the lower expert index. The
// k-th largest of the 32 lane maxima, L, bounds the k-th largest key from below (k
// lanes hold a key >= L), so the top k are among the keys >= L. Those candidates
// (usually a few dozen) are gathered, and each one's position in the descending order
// is its rank, the number of candidates above it. With more than 64 candidates the
// exact fallback takes k rounds of warp-wide maxima, dropping each winner from keys.
// This code runs once per launch, usually with its instructions evicted from L2 by
// the weight stream, so it is kept compact (loops, not unrolled register arrays).
// Lane j < k returns the j-th choice's packed key. cand: 64 entries.
__device__ uint64_t warp_topk_keys(uint64_t* keys, int E, int k, int lane, uint64_t* cand) {
  const int nq = E / 32;
  uint64_t m = 0ull;
#pragma unroll 4
  for (int q = 0; q < nq; ++q) m = umax64(m, keys[q * 32 + lane]);
  int lrank = 0;
#pragma unroll 4
  for (int sl = 0; sl < 32; ++sl) lrank += shfl_u64(m, sl) > m ? 1 : 0;
  const uint32_t lb = __ballot_sync(0xffffffffu, lrank == k - 1 && m != 0ull);
  const uint64_t L = lb ? shfl_u64(m, __ffs(lb) - 1) : 1ull;
  int c = 0;
#pragma unroll 4
  for (int q = 0; q < nq; ++q) c += keys[q * 32 + lane] >= L ? 1 : 0;
  int incl = c;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  uint64_t mine = 0ull;
  if (total <= 64) {
    int o = incl - c;
#pragma unroll 4
    for (int q = 0; q < nq; ++q) {
      const uint64_t x = keys[q * 32 + lane];
      if (x >= L) cand[o++] = x;
    }
    __syncwarp();
    const uint64_t x0 = lane < total ? cand[lane] : 0ull;
    const uint64_t x1 = lane + 32 < total ? cand[lane + 32] : 0ull;
    int r0 = 0, r1 = 0;
#pragma unroll 4
    for (int sl = 0; sl < 32; ++sl) {
      const uint64_t o0 = shfl_u64(x0, sl), o1 = shfl_u64(x1, sl);
      r0 += (o0 > x0 ? 1 : 0) + (o1 > x0 ? 1 : 0);
      r1 += (o0 > x1 ? 1 : 0) + (o1 > x1 ? 1 : 0);
    }
    __syncwarp();
    if (lane < total) cand[r0] = x0;
    if (lane + 32 < total) cand[r1] = x1;
    __syncwarp();
    mine = lane < k ? cand[lane] : 0ull;
    __syncwarp();
  } else {
#pragma unroll 4
    for (int j = 0; j < k; ++j) {
      uint64_t best = 0ull;
#pragma unroll 4
      for (int q = 0; q < nq; ++q) best = umax64(best, keys[q * 32 + lane]);
      const uint32_t hi = (uint32_t)(best >> 32);
      const uint32_t kmax = __reduce_max_sync(0xffffffffu, hi);
      const uint32_t wlo = __reduce_max_sync(0xffffffffu, hi == kmax ? (uint32_t)best : 0u);
      const uint64_t win = ((uint64_t)kmax << 32) | wlo;
      if (lane == j) mine = win;
      const int e = (int)(~wlo);
      __syncwarp();
      if (lane == 0 && e >= 0 && e < E) keys[e] = 0ull;
      __syncwarp();
    }
  }
  return mine;
}

// The rows this CTA owns (row b is owned by CTA b): once every router unit has
// published its partial sums, the row's logits are their sum in split order plus the
// bias; one warp takes the top-k and the softmax over it and publishes the choices
// (tagged words, then a release of the row count for readers of many rows).
template <bool kTrace>
__device__ bool route_rows_tc(const Params& p, Smem& sm, int mw, int lane, uint32_t& mphase, uint32_t tag) {
  const Shape& sh = sm.sh;
  const int mtid = mw * 32 + lane;
  const int E = p.E;
  for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
    if (mw == 0) {
      int ok = 1;
      if (lane == 0) ok = wait_counter(&p.ctr[CTR_ROUTER], (uint32_t)sh.router_target, p) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (lane == 0) {
        sm.bcast = ok;
        sm.bcast2 = 0;  // non-finite logit seen
      }
    }
    if (!mac_sync(sm, mphase, p, lane)) return false;
    if (!sm.bcast) return false;
    if (mtid == 0) trace_clk<kTrace>(p, TR_ROUTER_SEEN);
    const size_t stride4 = (size_t)p.B * E / 4;  // float4 stride between splits
    const float4* src = reinterpret_cast<const float4*>(p.rpart + (size_t)b * E);
    bool nonfinite = false;
    for (int e4 = mtid; e4 < E / 4; e4 += kMacThreads) {
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
      for (int s0 = 0; s0 < sh.RS; s0 += 8) {
        float4 t[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          if (s0 + i < sh.RS) t[i] = __ldcg(src + (size_t)(s0 + i) * stride4 + e4);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (s0 + i < sh.RS) {
            acc.x += t[i].x;
            acc.y += t[i].y;
            acc.z += t[i].z;
            acc.w += t[i].w;
          }
        }
      }
      if (p.bias) {  // 4-byte aligned: scalar loads
        acc.x += p.bias[4 * e4];
        acc.y += p.bias[4 * e4 + 1];
        acc.z += p.bias[4 * e4 + 2];
        acc.w += p.bias[4 * e4 + 3];
      }
      reinterpret_cast<float4*>(p.logits + (size_t)b * E)[e4] = acc;
      const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint64_t key = topk_key(a4[i], 4 * e4 + i);
        if (key == 0ull) nonfinite = true;
        sm.u.keys[4 * e4 + i] = key;
        if (p.dbg_logits) p.dbg_logits[(size_t)b * E + 4 * e4 + i] = a4[i];
      }
    }
    if (__any_sync(0xffffffffu, nonfinite) && lane == 0) sm.bcast2 = 1;
    if (!mac_sync(sm, mphase, p, lane)) return false;
    if (mtid == 0) trace_clk<kTrace>(p, TR_TOPK_LOADED);
    if (mw == 0) {
      const long long tk0 = tclock<kTrace>();
      const uint64_t mine = warp_topk_keys(sm.u.keys, E, p.k, lane, sm.topk_cand);
      if (lane == 0 && kTrace) {
        trace_put<kTrace>(p, TR_TOPK_CYC, (unsigned long long)(tclock<kTrace>() - tk0));
        trace_clk<kTrace>(p, TR_TOPK_CHOSEN);
      }
      // a non-finite logit ends the step: with fewer than k finite logits the row's
      // choices would not be k distinct experts, which the schedule's per-row
      // bookkeeping assumes (the abort path resets every ticket for the next step)
      if (sm.bcast2 && lane == 0) record_abort(p, MOE_ERR_NONFINITE);
      int e = (int)(~(uint32_t)mine);
      if (e < 0 || e >= E) e = 0;  // only with a non-finite row (reported)
      const float val = lane < p.k ? key_float((uint32_t)(mine >> 32)) : 0.0f;
      const float mx = __shfl_sync(0xffffffffu, val, 0);
      const float ex = lane < p.k ? expf(val - mx) : 0.0f;
      float z = ex;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
      if (lane < p.k)
        st_relaxed_gpu_v2(p.tk_pub + 2 * (b * p.k + lane), ((uint64_t)tag << 32) | (uint32_t)e,
                          ((uint64_t)tag << 32) | __float_as_uint(ex / z));
      __threadfence();
      __syncwarp();
      if (lane == 0) {
        red_release_add(&p.ctr[CTR_TOPK], 1u);
        trace_clk<kTrace>(p, TR_TOPK_SELECTED);
      }
    }
    if (!mac_sync(sm, mphase, p, lane)) return false;  // sm.u.keys free again
  }
  return true;
}

// Every CTA: the schedule of the tensor-core path from the published choices. Pairs
// are the unique experts ordered by row count, hottest first (stable in expert order),
// so the largest units are queued first and the down units that complete rows last
// are those of experts with few rows. An expert's slot rows keep expert order.
// The schedule of a one-row step: the row's k choices are k distinct experts with one
// row each, so the unique experts are the choices in ascending id (each one's slot is
// its rank among them) and the hottest-first order is that same order. One warp
// builds it (the general builder's result, without its masks, scans and rendezvous).
template <bool kTrace, bool kEp = false>
__device__ bool build_schedule_b1(const Params& p, Smem& sm, int mw, int lane, uint32_t& mphase, uint32_t tag) {
  const Shape& sh = sm.sh;
  Sched& sc = sm.sc;
  const int k = p.k;
  if (mw == 0) {
    int e = 0x7fffffff;
    float w = 0.0f;
    const bool ok = warp_poll_choices(p, tag, k, lane, e, w);
    if (lane == 0) sm.bcast = ok ? 1 : 0;
    if (ok) {
      if (lane == 0) trace_clk<kTrace>(p, TR_TOPK_SYNCED);
      // this step's experts (all, unless the step covers an expert range): rank r among them
      const bool local = lane < k && (!kEp || (e >= p.ep_e0 && e < p.ep_e1));
      const int el = local ? e : 0x7fffffff;
      int r = 0;
#pragma unroll 4
      for (int sl = 0; sl < 32; ++sl) r += __shfl_sync(0xffffffffu, el, sl) < el ? 1 : 0;
      const int kl = __popc(__ballot_sync(0xffffffffu, local));
      const int es = tc_expert_splits(1, sh.kblk ? sh.nkbH / 2 : sh.nkbH);
      if (local && !IDX_OK(p, (unsigned)e < (unsigned)p.E && (unsigned)r < (unsigned)kMaxSlots)) {
        e = 0;  // reported; the step is abandoned
        r = lane;
      }
      if (lane < k) {
        sm.u.t.topk_idx[lane] = e;
        sm.u.t.topk_w[lane] = w;
        if (!local) sc.slot_of[lane] = (int16_t)-1;  // another rank's expert: no slot row here
      }
      if (local) {
        sc.slot_expert[r] = (int16_t)e;
        sc.slot_cnt[r] = 1;
        sc.slot_base[r] = (int16_t)r;
        sc.eslot[e] = (int16_t)r;
        sc.pair_slot[r] = (int16_t)r;
        sc.pair_group[r] = 0;
        sc.pair_es[r] = (uint8_t)es;
        sc.pair_ubase[r] = r * sh.IT * es;
        sc.row_of[r] = 0;
        sc.w_of[r] = w;
        sc.slot_of[lane] = (int16_t)r;
      }
      if (lane == 0) {
        sc.U = kl;
        sc.S = kl;
        sc.P = kl;
        sc.slot_base[kl] = (int16_t)kl;
        sc.pair_ubase[kl] = kl * sh.IT * es;
        sc.NE = kl * sh.IT * es;
        sc.down_splits = 1 + kl;
        sc.ND = sh.DT * kl;
        sc.total = sh.pre + sc.NE + sc.ND;
        const unsigned tiles = (unsigned)(sh.RT + sh.ST + kl * sh.IT + sh.DT);
        sm.bcast2 = ((unsigned)sc.total <= p.max_units && tiles <= p.max_tiles) ? 1 : 0;
        if (!sm.bcast2) record_abort(p, MOE_ERR_UNSUPPORTED_SHAPE);
      }
      __syncwarp();
#ifdef MOE_BOUNDS_CHECK
      if (lane == 0 && (p.flags & kFlagBadSlot)) sc.slot_of[0] = (int16_t)kl;  // the first row past the schedule
      __syncwarp();
#endif
      if (blockIdx.x == 0 && lane < k) {
        if (p.dbg_idx) p.dbg_idx[lane] = e;
        if (p.dbg_w) p.dbg_w[lane] = w;
      }
      if (blockIdx.x == 0 && lane == 0 && p.dbg_nuniq) *p.dbg_nuniq = kl;
    }
  }
  const bool ok = mac_sync(sm, mphase, p, lane) && sm.bcast && sm.bcast2;
  if (mw == 0 && lane == 0) trace_clk<kTrace>(p, TR_SCHED_BUILT);
  return ok;
}

// dry: a pass over synthetic choices of at most 4 rows (row b takes experts
// (13 j + b) mod E, distinct for j < 32 as 13 is odd and E a multiple of 128 below
// 13 * 128) with no global effects, made by CTAs that own no row while they wait for
// the published choices, so that the real pass runs with its instructions cached
// (one out-of-line copy of the code serves both passes).
template <bool kTrace, bool kEp = false>
__device__ __noinline__ bool build_schedule_tc(const Params& p, Smem& sm, int mw, int lane, uint32_t& mphase,
                                               bool dry) {
  const Shape& sh = sm.sh;
  Sched& sc = sm.sc;
  const int mtid = mw * 32 + lane;
  // the dry pass runs the same instructions over at most 4 synthetic rows
  const int B = dry && p.B > 4 ? 4 : p.B, k = p.k;
  for (int e = mtid; e < p.E; e += kMacThreads) sm.u.t.mask[e] = 0ull;
  if (mw == 0) {
    int ok = 1;
    if (lane == 0 && !dry) ok = wait_counter(&p.ctr[CTR_TOPK], (uint32_t)B, p) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (lane == 0) sm.bcast = ok;
  }
  if (!mac_sync(sm, mphase, p, lane)) return false;
  if (!sm.bcast) return false;
  if (mtid == 0 && !dry) trace_clk<kTrace>(p, TR_TOPK_SYNCED);
  for (int t = mtid; t < B * k; t += kMacThreads) {
    ulonglong2 ch = make_ulonglong2(0ull, 0ull);
    if (!dry) ch = __ldcg(reinterpret_cast<const ulonglong2*>(p.tk_pub) + t);
    int e = dry ? (13 * (t % k) + t / k) % p.E : (int)(uint32_t)ch.x;
    if (!IDX_OK(p, (unsigned)e < (unsigned)p.E)) e = 0;  // reported; the step is abandoned
    const float w = dry ? 1.0f : __uint_as_float((uint32_t)ch.y);
    sm.u.t.topk_idx[t] = e;
    sm.u.t.topk_w[t] = w;
    if (!kEp || (e >= p.ep_e0 && e < p.ep_e1)) atomicOr(&sm.u.t.mask[e], 1ull << (t / k));  // this step's experts
  }
  if (!mac_sync(sm, mphase, p, lane)) return false;
  if (mtid == 0 && !dry) trace_clk<kTrace>(p, TR_TOPK_DONE);
  // unique experts in ascending id: per-chunk counts, then placement
  const int nchunk = p.E / 32;
  for (int ch = mw; ch < nchunk; ch += kMacWarps) {
    const uint32_t bal = __ballot_sync(0xffffffffu, sm.u.t.mask[ch * 32 + lane] != 0ull);
    if (lane == 0) sm.chunk_cnt[ch] = (int16_t)__popc(bal);
  }
  if (!mac_sync(sm, mphase, p, lane)) return false;
  {
    const int cnt = lane < nchunk ? sm.chunk_cnt[lane] : 0;
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += t;
    }
    for (int ch = mw; ch < nchunk; ch += kMacWarps) {
      const int chbase = __shfl_sync(0xffffffffu, incl - cnt, ch);
      const unsigned long long m = sm.u.t.mask[ch * 32 + lane];
      const uint32_t bal = __ballot_sync(0xffffffffu, m != 0ull);
      if (m != 0ull) {
        const int pos = chbase + __popc(bal & ((1u << lane) - 1u));
        sc.slot_expert[pos] = (int16_t)(ch * 32 + lane);
        sc.slot_cnt[pos] = (int16_t)__popcll(m);
        sc.eslot[ch * 32 + lane] = (int16_t)pos;
      }
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (mw == 0 && lane == 0) sm.nuniq = total;
  }
  if (mtid <= kTcMaxN + 1 && mtid < kMacThreads) sm.cnt_base[mtid] = 0;
  if (!mac_sync(sm, mphase, p, lane)) return false;
  if (mtid == 0 && !dry) trace_clk<kTrace>(p, TR_SCHED_PLACED);
  if (mw == 0) {
    const int U = sm.nuniq;
    // slot bases (slot order)
    int rbase = 0;
    for (int i0 = 0; i0 < U; i0 += 32) {
      const int i = i0 + lane;
      const int c = i < U ? sc.slot_cnt[i] : 0;
      int cs = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, cs, off);
        if (lane >= off) cs += t;
      }
      if (i < U) sc.slot_base[i] = (int16_t)(rbase + cs - c);
      rbase += __shfl_sync(0xffffffffu, cs, 31);
    }
    // stable counting sort of the slots by row count, descending
    for (int i = lane; i < U; i += 32) atomicAdd(&sm.cnt_base[sc.slot_cnt[i]], 1);
    __syncwarp();
    {
      const int c0 = kTcMaxN - 2 * lane, c1 = c0 - 1;  // lane 0: counts 64, 63; lane 31: 2, 1
      const int h0 = sm.cnt_base[c0], h1 = sm.cnt_base[c1];
      int incl = h0 + h1;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      __syncwarp();
      sm.cnt_base[c0] = incl - h0 - h1;
      sm.cnt_base[c1] = incl - h1;
    }
    __syncwarp();
    for (int i0 = 0; i0 < U; i0 += 32) {
      const int i = i0 + lane;
      const int c = i < U ? sc.slot_cnt[i] : 0;
      const uint32_t m = __match_any_sync(0xffffffffu, c);
      const int rank = __popc(m & ((1u << lane) - 1u));
      if (c > 0 && IDX_OK(p, c <= kTcMaxN && (unsigned)(sm.cnt_base[c] + rank) < (unsigned)kMaxSlots))
        sc.pair_slot[sm.cnt_base[c] + rank] = (int16_t)i;
      __syncwarp();
      if (c > 0 && lane == __ffs(m) - 1) sm.cnt_base[c] += __popc(m);
      __syncwarp();
    }
    if (lane == 0 && !dry) trace_clk<kTrace>(p, TR_SCHED_SORTED);
    // gate/up units per pair and their prefix
    int ubase = 0;
    for (int p0 = 0; p0 < U; p0 += 32) {
      const int pr = p0 + lane;
      int units = 0;
      if (pr < U) {
        const int es = tc_expert_splits(sc.slot_cnt[sc.pair_slot[pr]], sh.kblk ? sh.nkbH / 2 : sh.nkbH);
        sc.pair_es[pr] = (uint8_t)es;
        sc.pair_group[pr] = 0;
        units = sh.IT * es;
      }
      int cs = units;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, cs, off);
        if (lane >= off) cs += t;
      }
      if (pr < U) sc.pair_ubase[pr] = ubase + cs - units;
      ubase += __shfl_sync(0xffffffffu, cs, 31);
    }
    if (lane == 0) {
      sc.U = U;
      sc.S = rbase;
      sc.slot_base[U] = (int16_t)rbase;
      sc.P = U;
      sc.pair_ubase[U] = ubase;
      sc.NE = ubase;
      sc.down_splits = 1 + U;
      sc.ND = sh.DT * U;
      sc.total = sh.pre + sc.NE + sc.ND;
      const unsigned tiles = (unsigned)(sh.RT + sh.ST + U * sh.IT + sh.DT);
      sm.bcast2 = ((unsigned)sc.total <= p.max_units && tiles <= p.max_tiles && U <= kMaxSlots) ? 1 : 0;
      if (!sm.bcast2 && !dry) record_abort(p, MOE_ERR_UNSUPPORTED_SHAPE);
    }
  }
  if (mtid == 0 && !dry) trace_clk<kTrace>(p, TR_UNIQUE_DONE);
  if (!mac_sync(sm, mphase, p, lane)) return false;
  if (!sm.bcast2) return false;
  // slot rows: an expert's rows in token order; rank of row b among them by popcount
  for (int t = mtid; t < B * k; t += kMacThreads) {
    const int b = t / k;
    const int e = sm.u.t.topk_idx[t];
    if (kEp && (e < p.ep_e0 || e >= p.ep_e1)) {  // another rank's expert: no slot row here
      sc.slot_of[t] = (int16_t)-1;
      continue;
    }
    const unsigned long long m = sm.u.t.mask[e];
    const int r = sc.slot_base[sc.eslot[e]] + __popcll(m & ((1ull << b) - 1ull));
    if (!IDX_OK(p, (unsigned)r < (unsigned)kMaxSlots)) continue;
    sc.row_of[r] = (uint8_t)b;
    sc.w_of[r] = sm.u.t.topk_w[t];
    sc.slot_of[t] = (int16_t)r;
  }
#ifdef MOE_BOUNDS_CHECK
  if (!dry && (p.flags & kFlagBadSlot)) {  // row 0's first choice: the first slot row past the schedule
    if (!mac_sync(sm, mphase, p, lane)) return false;
    if (mtid == 0) sc.slot_of[0] = (int16_t)sc.S;
  }
#endif
  if (blockIdx.x == 0 && !dry) {
    for (int t = mtid; t < B * k; t += kMacThreads) {
      if (p.dbg_idx) p.dbg_idx[t] = sm.u.t.topk_idx[t];
      if (p.dbg_w) p.dbg_w[t] = sm.u.t.topk_w[t];
    }
    if (mtid == 0 && p.dbg_nuniq) *p.dbg_nuniq = sc.U;
  }
  const bool ok = mac_sync(sm, mphase, p, lane);
  if (mtid == 0 && !dry) trace_clk<kTrace>(p, TR_SCHED_BUILT);
  return ok;
}

// ---- RMSNorm of the rows this CTA publishes (MAC warps) ---------------------------------------

template <bool kTrace>
__device__ bool normalise_rows(const Params& p, Smem& sm, int mw, int lane, uint32_t& mphase) {
  // This runs once per launch, first thing, with its instructions usually evicted from
  // L2 (each new instruction line then comes from DRAM): the loops are kept short
  // rather than unrolled over register arrays. Pass 1 loads x and gamma (4 vectors in
  // flight per thread) and sums the squares; pass 2 re-reads both from L1.
  const int mtid = mw * 32 + lane;
  const int nv = p.H / 8;
  const uint4* g4 = reinterpret_cast<const uint4*>(p.gamma);
  const bool fresh = p.rows_in != nullptr;  // input rows written during this launch
  for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
    if (fresh) {
      // the previous layer's output row b is input once all of its tile pairs are combined
      if (mw == 0) {
        int ok = 1;
        if (lane == 0) ok = wait_counter(&p.rows_in[b], (uint32_t)((p.H + 2 * kTcRows - 1) / (2 * kTcRows)), p) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (lane == 0) sm.bcast = ok;
      }
      if (!mac_sync(sm, mphase, p, lane)) return false;
      if (!sm.bcast) return false;
    }
    const uint4* x4 = reinterpret_cast<const uint4*>(p.x + (size_t)b * p.H);
    float ss = 0.0f;
#pragma unroll 4
    for (int v = mtid; v < nv; v += kMacThreads) {
      const uint4 xv = fresh ? ld_cg_v4(x4 + v) : ld_nc_v4(x4 + v);
      (void)ld_nc_v4(g4 + v);  // brings gamma into L1 for pass 2 (a volatile load is kept)
      float f[8];
      unpack8(xv, f);
#pragma unroll
      for (int t = 0; t < 8; ++t) ss = fmaf(f[t], f[t], ss);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) sm.red_ss[mw] = ss;
    if (mtid == 0 && b == (int)blockIdx.x) trace_stamp<kTrace>(p, TR_NORM_SUMMED);
    if (!mac_sync(sm, mphase, p, lane)) return false;
    if (mtid == 0 && b == (int)blockIdx.x) trace_stamp<kTrace>(p, TR_NORM_REDUCED);
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < kMacWarps; ++w) tot += sm.red_ss[w];
    const float r = 1.0f / sqrtf(tot / (float)p.H + p.eps);
    uint4* n4 = reinterpret_cast<uint4*>(p.n + (size_t)b * p.H);
#pragma unroll 1
    for (int v = mtid; v < nv; v += kMacThreads) {
      float f[8], g[8];
      unpack8(fresh ? ld_cg_v4(x4 + v) : ld_nc_v4(x4 + v), f);
      unpack8(ld_nc_v4(g4 + v), g);
      uint32_t o[4];
#pragma unroll
      for (int t = 0; t < 4; ++t)
        o[t] = (uint32_t)f2bf(f[2 * t] * r * g[2 * t]) | ((uint32_t)f2bf(f[2 * t + 1] * r * g[2 * t + 1]) << 16);
      n4[v] = make_uint4(o[0], o[1], o[2], o[3]);
    }
    fence_proxy_async_global();
    if (!mac_sync(sm, mphase, p, lane)) return false;
    if (mtid == 0 && b == (int)blockIdx.x) trace_stamp<kTrace>(p, TR_NORM_STORED);
    if (mtid == 0 && !((p.flags & kFlagWithholdNReady) && b == 0)) red_release_add(&p.ctr[CTR_NREADY], 1u);
    if (mtid == 0) trace_stamp<kTrace>(p, TR_N_PUBLISHED);
  }
  return true;
}

// ---- epilogue warp: one finished unit ------------------------------------------------------------

// Completion counter a finished tile of this unit's type releases.
__device__ __forceinline__ uint32_t* done_counter(const Params& p, const UnitDesc& d) {
  switch (d.type) {
    case UT_ROUTER: return &p.ctr[CTR_ROUTER];
    case UT_SHARED: return &p.ctr[CTR_HS];
    case UT_EXPERT: return &p.pair_done[d.pair];
    default: return nullptr;
  }
}

// Lane = tile row everywhere. `res` holds the unit's reduced values [2][32][4].
__device__ void epi_finish(const Params& p, Smem& sm, const UnitDesc& d, int u,
                           float (*res)[kBoxRows][kActGroup], int lane) {
  const Shape& sh = sm.sh;
  const Sched& sc = sm.sc;
  const bool down = d.type == UT_DOWN_SHARED || d.type == UT_DOWN_EXPERT;
  float(*src)[kBoxRows][kActGroup] = res;
  if (d.nsplit > 1) {
    float4* part = reinterpret_cast<float4*>(p.partial + (size_t)u * kPartialFloats);
    const float4* r4 = reinterpret_cast<const float4*>(&res[0][0][0]);
    part[lane] = r4[lane];
    part[32 + lane] = r4[32 + lane];
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      // acq_rel: releases this warp's partial (ordered by the warp barrier above),
      // acquires the other splits' partials when this split is the tile's last
      const uint32_t old = atom_add_acq_rel(&p.tickets[d.ticket], 1u);
      last = old == (uint32_t)(d.nsplit - 1);
      if (last) st_relaxed_gpu(&p.tickets[d.ticket], 0u);
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __syncwarp();
    if (!down) {
      // fixed split order -> deterministic sums
      float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
      for (int sp = 0; sp < d.nsplit; ++sp) {
        const float4* q = reinterpret_cast<const float4*>(
            p.partial + (size_t)unit_of_split(sh, sc, d, sp) * kPartialFloats);
        const float4 a = __ldcg(q + lane), b = __ldcg(q + 32 + lane);
        s0.x += a.x; s0.y += a.y; s0.z += a.z; s0.w += a.w;
        s1.x += b.x; s1.y += b.y; s1.z += b.z; s1.w += b.w;
      }
      reinterpret_cast<float4*>(&sm.fin[0][0][0])[lane] = s0;
      reinterpret_cast<float4*>(&sm.fin[0][0][0])[32 + lane] = s1;
      __syncwarp();
      src = sm.fin;
    }
  }
  const int row = lane;
  if (d.type == UT_ROUTER) {
    const int c = group_rows(sh.B, d.g);
    const int e = d.tile * kBoxRows + row;
    const float bias = p.bias ? p.bias[e] : 0.0f;
    for (int j = 0; j < c; ++j) {
      const int b = d.g * kActGroup + j;
      const float v = src[0][row][j] + bias;
      p.logits[(size_t)b * p.E + e] = v;
      if (p.dbg_logits) p.dbg_logits[(size_t)b * p.E + e] = v;
    }
  } else if (d.type == UT_SHARED) {
    const int c = group_rows(sh.B, d.g);
    for (int j = 0; j < c; ++j) {
      const int b = d.g * kActGroup + j;
      p.hs[(size_t)b * p.Is + d.tile * kBoxRows + row] = f2bf(silu(src[0][row][j]) * src[1][row][j]);
    }
  } else if (d.type == UT_EXPERT) {
    const int c = pair_rows(sc, d.pair);
    const int r0 = pair_first_slot_row(sc, d.pair);
    for (int j = 0; j < c; ++j)
      if (IDX_OK(p, (unsigned)(r0 + j) < (unsigned)kMaxSlots))
        p.he[(size_t)(r0 + j) * p.I + d.tile * kBoxRows + row] = f2bf(silu(src[0][row][j]) * src[1][row][j]);
  } else {
    // down tile fix-up: y = bf16(x + s + sum_e w_e d_e) in fixed split / pair / row order
    float* yacc = sm.u.yacc[row];
    for (int b = 0; b < sh.B; ++b) yacc[b] = 0.0f;
    for (int sp = 0; sp < d.nsplit; ++sp) {
      const float* part =
          p.partial + (size_t)(sh.NR + sh.NS + sc.NE + sp * sh.DT + d.tile) * kPartialFloats;
      if (sp < sh.GB) {
        const float4 v = __ldcg(reinterpret_cast<const float4*>(part) + row);
        const float vv[4] = {v.x, v.y, v.z, v.w};
        const int c = group_rows(sh.B, sp);
        for (int j = 0; j < c; ++j) yacc[sp * kActGroup + j] += vv[j];
      } else {
        const int pr0 = (sp - sh.GB) * kDownPairsPerSplit;
        const int np = sc.P - pr0 < kDownPairsPerSplit ? sc.P - pr0 : kDownPairsPerSplit;
        for (int q = 0; q < np; ++q) {
          const int pr = pr0 + q;
          const float4 v = __ldcg(reinterpret_cast<const float4*>(part + q * kBoxRows * kActGroup) + row);
          const float vv[4] = {v.x, v.y, v.z, v.w};
          const int c = pair_rows(sc, pr);
          const int r0 = pair_first_slot_row(sc, pr);
          for (int j = 0; j < c; ++j)
            if (IDX_OK(p, (unsigned)(r0 + j) < (unsigned)kMaxSlots && sc.row_of[r0 + j] < sh.B))
              yacc[sc.row_of[r0 + j]] += vv[j];
        }
      }
    }
    const int h = d.tile * kBoxRows + row;
    for (int b = 0; b < sh.B; ++b) {
      const float xv = bf2f(p.x[(size_t)b * p.H + h]);
      p.y[(size_t)b * p.H + h] = f2bf(xv + yacc[b]);
    }
  }
  uint32_t* done = done_counter(p, d);
  if (done) {
    fence_proxy_async_global();
    __syncwarp();
    if (lane == 0) red_release_add(done, 1u);
  }
}

// ---- producer warp (both paths) ------------------------------------------------------------------

// Ring position and the producer's waits. A slot's pending record is the phase of its
// last TMA stage that no later use of the slot has shown to be complete.
struct Producer {
  const Params& p;
  Smem& sm;
  int lane;
  int nst;  // ring stages
  int slot;
  uint32_t phase;
  uint32_t pend_mask, pend_parity;

  int cq_pos;        // converter queue: next entry and its phase
  uint32_t cq_phase;
  uint32_t wpar, wpend;  // FP8: per slot the parity of its next wfull phase; slots used
  uint32_t fp8prev, cdpar;  // FP8: slots whose last stage was FP8 (released on cdone); cdone parities
  bool switched;            // FP8: HK_SWITCH issued (the MMA warp reads the A stages)

  __device__ Producer(const Params& p_, Smem& sm_, int lane_, int nst_)
      : p(p_), sm(sm_), lane(lane_), nst(nst_), slot(0), phase(0u), pend_mask(0u), pend_parity(0u), cq_pos(0),
        cq_phase(0u), wpar(0u), wpend(0u), fp8prev(0u), cdpar(0u), switched(false) {}

  // An FP8 stage in the current slot: the parity of the wfull phase its codes complete.
  __device__ uint32_t mark_fp8() {
    const uint32_t par = (wpar >> slot) & 1u;
    wpar ^= 1u << slot;
    wpend |= 1u << slot;
    fp8prev |= 1u << slot;
    return par;
  }
  __device__ uint32_t last_wpar() const { return ((wpar >> slot) & 1u) ^ 1u; }

  // Hands the FP8 stage in ring slot `s` (wfull parity `par`, full parity `fpar`) to the
  // converters; s = -1 tells them that no more stages follow.
  __device__ bool push_conv(int s, uint32_t par, uint32_t fpar = 0u) {
    if (!wait_bar(&sm.cq_empty[cq_pos], cq_phase ^ 1u)) return false;
    if (lane == 0) {
      sm.cq_slot[cq_pos] = (int16_t)s;
      sm.cq_par[cq_pos] = (uint8_t)par;
      sm.cq_fpar[cq_pos] = (uint8_t)fpar;
      mbar_arrive(&sm.cq_full[cq_pos]);
    }
    __syncwarp();
    if (++cq_pos == kCq) {
      cq_pos = 0;
      cq_phase ^= 1u;
    }
    return true;
  }

  __device__ int grab() {
    int v = 0;
    if (lane == 0) v = (int)atom_add_relaxed(&p.ctr[CTR_QUEUE], 1u);
    return __shfl_sync(0xffffffffu, v, 0);
  }
  __device__ void advance() {
    if (++slot == nst) {
      slot = 0;
      phase ^= 1u;
    }
  }
  __device__ void mark_pending() {
    pend_mask |= 1u << slot;
    pend_parity = (pend_parity & ~(1u << slot)) | (phase << slot);
  }
  __device__ bool wait_bar(uint64_t* bar, uint32_t parity) {
    int r = 1;
    if (lane == 0) r = wait_mbar(bar, parity, p) ? 1 : 0;
    r = __shfl_sync(0xffffffffu, r, 0);
    __syncwarp();
    return r != 0;
  }
  // Waits for a free slot; the slot's previous stage has then been consumed (an FP8
  // stage's by the converters, any other by the MMAs).
  // Before the schedule of a step of at most 4 rows, at most nst - 1 stages in flight: the
  // next slot's previous stage must be consumed too.
  __device__ bool wait_slot_pre() {
    if (p.B > 4 || nst < 5) return true;
    const int s1 = slot + 1 == nst ? 0 : slot + 1;
    return wait_bar(&sm.empty[s1], s1 == 0 ? phase : phase ^ 1u);
  }
  __device__ bool wait_slot() {
    if ((fp8prev >> slot) & 1u) {
      const uint32_t par = (cdpar >> slot) & 1u;
      cdpar ^= 1u << slot;
      fp8prev &= ~(1u << slot);
      return wait_bar(&sm.cdone[slot], par);
    }
    return wait_bar(&sm.empty[slot], phase ^ 1u);
  }
  // FP8: the MMA warp is told, through the ring, that the A stages carry the rest.
  __device__ bool emit_switch() {
    if (!wait_slot()) return false;
    // the slot's previous stage has been consumed, so its copies have landed; this use
    // completes a full phase of its own (the drain must not wait for the earlier one)
    pend_mask &= ~(1u << slot);
    if (lane == 0) {
      sm.hdr[slot].kind = HK_SWITCH;
      mbar_arrive(&sm.full[slot]);
    }
    __syncwarp();
    advance();
    switched = true;
    return true;
  }
  __device__ bool wait_dep(const uint32_t* c, uint32_t target) {
    int r = 1;
    if (lane == 0) {
      r = wait_counter(c, target, p) ? 1 : 0;
      fence_proxy_async_global();
    }
    r = __shfl_sync(0xffffffffu, r, 0);
    __syncwarp();
    return r != 0;
  }
  // (expert, row group) pair pr complete? One acquire round trip polls 32 pairs.
  __device__ bool wait_pair(int pr) {
    const Shape& sh = sm.sh;
    if (!IDX_OK(p, (unsigned)pr < (unsigned)kMaxSlots)) return false;
    if ((sm.known_done[pr >> 5] >> (pr & 31)) & 1u) return true;
    const int q = pr + lane;
    const bool done = q < sm.sc.P && ld_acquire_gpu(&p.pair_done[q]) >= (uint32_t)sh.pair_target;
    const uint32_t bal = __ballot_sync(0xffffffffu, done);
    if (lane == 0) {
      for (int i = 0; i < 32; ++i)
        if ((bal >> i) & 1u) sm.known_done[(pr + i) >> 5] |= 1u << ((pr + i) & 31);
    }
    __syncwarp();
    bool r = (bal & 1u) != 0u;
    if (!r) {
      r = wait_dep(&p.pair_done[pr], (uint32_t)sh.pair_target);
      if (r && lane == 0) sm.known_done[pr >> 5] |= 1u << (pr & 31);
      __syncwarp();
    } else if (lane == 0) {
      fence_proxy_async_global();
    }
    return r;
  }

  // After the last stage: the stop header and the drain of every bulk copy still in
  // flight.
  __device__ void finish(bool fp8 = false) {
    // the converters stop (bounded: they also stop on abort); after HK_SWITCH they pass
    // the end on to the MMA warp, otherwise it comes through the ring
    if (fp8) push_conv(-1, 0u);
    if (!switched && wait_slot()) {
      pend_mask &= ~(1u << slot);
      if (lane == 0) {
        sm.hdr[slot].kind = HK_END;
        mbar_arrive(&sm.full[slot]);
      }
    }
    __syncwarp();
    if (lane == 0) {
      // every bulk copy this CTA issued lands before its shared memory is given up;
      // a copy that never lands is reported like every other wait that runs out
      for (int s = 0; s < nst; ++s) {
        if (!((pend_mask >> s) & 1u)) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&sm.full[s], (pend_parity >> s) & 1u)) {
          if (globaltimer_ns() - t0 > 50000000ull) {
            record_abort(p, MOE_ERR_TIMEOUT);
            break;
          }
        }
      }
      for (int s = 0; s < nst; ++s) {  // FP8 codes and scales
        if (!((wpend >> s) & 1u)) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&sm.wfull[s], ((wpar >> s) & 1u) ^ 1u)) {
          if (globaltimer_ns() - t0 > 50000000ull) {
            record_abort(p, MOE_ERR_TIMEOUT);
            break;
          }
        }
      }
    }
    __syncwarp();
  }
};

// Ring position carried by the producer from one layer of a fused launch to the next.
struct RingState {
  int slot;
  uint32_t phase, pend_mask, pend_parity;
};

// CUDA-core path producer: units of 32 weight rows, activation rows by 1-D bulk copies.
template <bool kTrace>
__device__ void producer_cc(Producer& pr, uint8_t* ring) {
  const Params& p = pr.p;
  Smem& sm = pr.sm;
  const Shape& sh = sm.sh;
  const int lane = pr.lane;
  const uint64_t pol = policy_evict_first();
  if (lane == 0)
    for (int t = 0; t < TM_T_WR; ++t) prefetch_tensormap(&p.tmaps[t]);
  bool ok = true, sched_ready = false, n_ok = false, hs_ok = false;
  const int pre = sh.NR + sh.NS;
  int u = pr.grab();
  bool first_expert = true, first_down = true;
  unsigned long long c_slot = 0, c_dep = 0, c_grab = 0, c_issue = 0, c_stages = 0, c_units = 0;
  unsigned long long c_setup = 0, c_schedw = 0;
  const long long tploop0 = tclock<kTrace>();
  while (ok) {
    if (u >= pre && !sched_ready) {
      ok = pr.wait_slot();
      if (!ok) break;
      pr.pend_mask &= ~(1u << pr.slot);
      if (lane == 0) {
        sm.hdr[pr.slot].kind = HK_SCHED;
        mbar_arrive(&sm.full[pr.slot]);
      }
      __syncwarp();
      pr.advance();
      const long long tw0 = tclock<kTrace>();
      ok = pr.wait_bar(&sm.sched_bar, 0u);
      c_schedw += (unsigned long long)(tclock<kTrace>() - tw0);
      if (!ok) break;
      sched_ready = true;
      if (lane == 0) trace_stamp<kTrace>(p, TR_SCHED);
    }
    if (sched_ready && u >= sm.sc.total) break;
    const long long tu0 = tclock<kTrace>();
    const UnitDesc d = decode_unit(sh, sm.sc, u);
    // the next unit's queue ticket is requested now and read after this unit's
    // stages are issued, so the atomic's round trip overlaps the issue loop
    uint32_t next_ticket = 0;
    if (lane == 0) next_ticket = atom_add_relaxed(&p.ctr[CTR_QUEUE], 1u);
    if (lane == 0 && kTrace) {
      if (first_expert && d.type == UT_EXPERT) { trace_stamp<kTrace>(p, TR_FIRST_EXPERT); first_expert = false; }
      if (first_down && (d.type == UT_DOWN_SHARED || d.type == UT_DOWN_EXPERT)) { trace_stamp<kTrace>(p, TR_FIRST_DOWN); first_down = false; }
      ++c_units;
    }
    if ((p.flags & kFlagJitter) && lane == 0) __nanosleep(hash32(blockIdx.x * 7919u + (uint32_t)u) % 3000u);
    const int nseg_units = d.type == UT_DOWN_EXPERT ? d.npair : 1;
    c_setup += (unsigned long long)(tclock<kTrace>() - tu0);
    for (int q = 0; q < nseg_units && ok; ++q) {
      SegCtx x;
      const long long tm0 = tclock<kTrace>();
      make_seg(p, sh, sm.sc, d, q, x);
      c_setup += (unsigned long long)(tclock<kTrace>() - tm0);
      const uint32_t box_bytes = (uint32_t)(x.box_cols * kBoxRows * 2);
      const uint32_t row_bytes = (uint32_t)(x.box_cols * 2);
      const int step = x.kpair ? 2 : 1;
      const int info0 = (x.kpair ? kInfoKpair : 0) | (x.c << 3) | (q << 8) | (x.box_cols << 16);
      for (int kb = x.kb0; kb < x.kb_end && ok; kb += step) {
        {
          const long long t0 = tclock<kTrace>();
          ok = pr.wait_slot();
          c_slot += (unsigned long long)(tclock<kTrace>() - t0);
        }
        if (!ok) break;
        const long long ti0 = tclock<kTrace>();
        const int nbox = x.kpair ? (x.kb_end - kb < 2 ? 1 : 2) : 2;
        const int nseg = x.kpair ? nbox : 1;
        const bool seg_end = kb + step >= x.kb_end;
        uint8_t* dst = ring + pr.slot * kSlotBytes;
        uint64_t* fb = &sm.full[pr.slot];
        pr.mark_pending();
        if (lane == 0) {
          StageHeader h;
          h.kind = HK_STAGE;
          h.unit = u;
          h.info = info0 | nbox | (seg_end ? kInfoSegEnd : 0) | (seg_end && q == nseg_units - 1 ? kInfoUnitEnd : 0) |
                   (kb == x.kb0 && q == 0 ? kInfoFirst : 0);
          h.wrow = x.wrow;
          sm.hdr[pr.slot] = h;
          mbar_arrive_expect_tx(fb, (uint32_t)nbox * box_bytes + (uint32_t)(nseg * x.c) * row_bytes);
          const int col = kb * x.box_cols;
          tma_load_2d(dst, x.tm0, col, x.y0, fb, pol);
          if (nbox == 2) tma_load_2d(dst + kBoxBytesMax, x.tm1, x.kpair ? col + x.box_cols : col, x.y0, fb, pol);
        }
        // activations: only after the acquire that publishes them
        bool dep_ok = true;
        const long long td0 = tclock<kTrace>();
        if (kb == x.kb0) {
          if (x.dep == 0) {
            if (!n_ok) {
              dep_ok = n_ok = pr.wait_dep(&p.ctr[CTR_NREADY], (uint32_t)p.B);
              if (lane == 0) trace_stamp<kTrace>(p, TR_NREADY);
            }
          } else if (x.dep == 1) {
            if (!hs_ok) dep_ok = hs_ok = pr.wait_dep(&p.ctr[CTR_HS], (uint32_t)sh.hs_target);
          } else {
            dep_ok = pr.wait_pair(x.pair);
          }
        }
        const long long td1 = tclock<kTrace>();
        c_dep += (unsigned long long)(td1 - td0);
        if (lane == 0) {
          uint8_t* act = dst + 2 * kBoxBytesMax;
          for (int sg = 0; sg < nseg; ++sg) {
            const int col = (kb + sg) * x.box_cols;
#pragma unroll
            for (int j = 0; j < kActGroup; ++j)
              if (j < x.c) bulk_load(act + sg * kActSegBytes + j * row_bytes, x.abase + x.aoff[j] + col, row_bytes, fb);
          }
        }
        __syncwarp();
        pr.advance();
        c_issue += (unsigned long long)(tclock<kTrace>() - ti0) - (unsigned long long)(td1 - td0);
        ++c_stages;
        if (!dep_ok) ok = false;
      }
    }
    {
      const long long t0 = tclock<kTrace>();
      u = __shfl_sync(0xffffffffu, (int)next_ticket, 0);
      c_grab += (unsigned long long)(tclock<kTrace>() - t0);
    }
  }
  if (lane == 0 && kTrace) {
    trace_stamp<kTrace>(p, TR_PROD_END);
    trace_put<kTrace>(p, TR_PROD_WAIT_SLOT_CYC, c_slot);
    trace_put<kTrace>(p, TR_PROD_WAIT_DEP_CYC, c_dep);
    trace_put<kTrace>(p, TR_PROD_GRAB_CYC, c_grab);
    trace_put<kTrace>(p, TR_PROD_ISSUE_CYC, c_issue);
    trace_put<kTrace>(p, TR_PROD_STAGES, c_stages);
    trace_put<kTrace>(p, TR_UNITS, c_units);
    trace_put<kTrace>(p, TR_PROD_SETUP_CYC, c_setup);
    trace_put<kTrace>(p, TR_PROD_SCHED_CYC, c_schedw);
    trace_put<kTrace>(p, TR_PROD_LOOP_CYC, (unsigned long long)(tclock<kTrace>() - tploop0));
  }
  pr.finish();
}

// Tensor-core path: one unit's tensor maps, rows and activation operand.
struct TcSeg {
  const CUtensorMap* tw0;  // weight tile 0 (accumulator columns +0)
  const CUtensorMap* tw1;  // weight tile 1 (accumulator columns +64)
  const CUtensorMap* ta;   // activation operand
  int y0, y1, nbox;
  int N;     // MMA N: activation rows loaded (multiple of 16)
  int arow;  // first activation row
  int dep;   // 0: normalised rows, 1: shared h, 2: the expert's h
  int pair;
  int fp8;   // 1: the weight tiles are E4M3 codes (expert units of an FP8 layer)
  const CUtensorMap* ta2;  // FP8: the activations of two K atoms in one box (16-row tiles)
  int sc0;    // FP8: index of tile 0's scale at K block 0 (gate or down array)
  int sdown;  // FP8: a down unit
};

template <bool kFp8, bool kEp = false>
__device__ __forceinline__ void make_seg_tc(const Params& p, const Shape& sh, const Sched& sc, const UnitDesc& d,
                                            TcSeg& x) {
  x.pair = d.pair;
  x.arow = 0;
  x.N = sh.NA;
  x.ta = &p.tmaps[TM_T_AN];
  x.dep = 0;
  x.fp8 = 0;
  switch (d.type) {
    case UT_ROUTER:
      x.tw0 = x.tw1 = &p.tmaps[TM_T_WR];
      x.y0 = d.tile * 2 * kTcRows;
      x.y1 = x.y0 + kTcRows;
      x.nbox = x.y1 < p.E ? 2 : 1;
      break;
    case UT_SHARED:
      x.tw0 = &p.tmaps[TM_T_WSG];
      x.tw1 = &p.tmaps[TM_T_WSU];
      x.y0 = x.y1 = d.tile * kTcRows;
      x.nbox = 2;
      break;
    case UT_EXPERT: {
      // every token row is an MMA column; the epilogue keeps the expert's own rows
      // e: the expert's index in this layer's expert arrays (they start at expert ep_wbase)
      int e = sc.slot_expert[sc.pair_slot[d.pair]] - (kEp ? p.ep_wbase : 0);
      if (!IDX_OK(p, (unsigned)d.pair < (unsigned)kMaxSlots && (unsigned)e < (unsigned)(p.ep_e1 - (kEp ? p.ep_wbase : 0)))) e = 0;
      x.tw0 = &p.tmaps[kFp8 ? TM_Q_WG : TM_T_WG];
      x.tw1 = &p.tmaps[kFp8 ? TM_Q_WU : TM_T_WU];
      x.y0 = x.y1 = e * p.I + d.tile * kTcRows;
      x.nbox = 2;
      x.fp8 = kFp8;
      if (kFp8) {  // gate and up blocks [e][tile][K block]
        x.ta2 = &p.tmaps[TM_Q_AN];
        x.sc0 = (e * (p.I / kTcRows) + d.tile) * (p.H / kTcRows);
        x.sdown = 0;
      }
      break;
    }
    case UT_DOWN_SHARED:
      x.tw0 = x.tw1 = &p.tmaps[TM_T_WSD];
      x.y0 = d.tile * 2 * kTcRows;
      x.y1 = x.y0 + kTcRows;
      x.nbox = x.y1 < p.H ? 2 : 1;
      x.ta = &p.tmaps[TM_T_AHS];
      x.dep = 1;
      break;
    default: {
      // the expert's slot rows of h are contiguous: they are the MMA columns
      int i = sc.pair_slot[d.pair];
      if (!IDX_OK(p, (unsigned)i < (unsigned)kMaxE)) i = 0;
      int e = sc.slot_expert[i] - (kEp ? p.ep_wbase : 0);  // index in this layer's expert arrays
      if (!IDX_OK(p, (unsigned)e < (unsigned)(p.ep_e1 - (kEp ? p.ep_wbase : 0)) &&
                         (unsigned)sc.slot_base[i] < (unsigned)kMaxSlots))
        e = 0;
      x.tw0 = x.tw1 = &p.tmaps[kFp8 ? TM_Q_WD : TM_T_WD];
      x.fp8 = kFp8;
      if (kFp8) {  // down blocks [e][row block 2 tile, 2 tile + 1][K block]
        x.ta2 = &p.tmaps[TM_Q_AHE];
        x.sc0 = (e * (p.H / kTcRows) + 2 * d.tile) * (p.I / kTcRows);
        x.sdown = 1;
      }
      x.y0 = e * p.H + d.tile * 2 * kTcRows;
      x.y1 = x.y0 + kTcRows;
      x.nbox = d.tile * 2 * kTcRows + kTcRows < p.H ? 2 : 1;
      x.ta = &p.tmaps[TM_T_AHE];
      x.arow = sc.slot_base[i];
      x.N = (sc.slot_cnt[i] + kTcActRows - 1) / kTcActRows * kTcActRows;
      x.dep = 2;
      break;
    }
  }
}

// Tensor-core path producer: per 64-column K atom one stage of up to two 128-row weight
// tiles and the activation operand (N rows, boxes of 16), all 128-byte swizzled.
// last: the launch's last layer (then the stop header and the drain follow); false is
// returned on abort (after the same stop header and drain).
template <bool kTrace, bool kFp8 = false, bool kEp = false>
__device__ bool producer_tc(Producer& pr, uint8_t* ring, bool last = true) {
  const Params& p = pr.p;
  Smem& sm = pr.sm;
  const Shape& sh = sm.sh;
  const int lane = pr.lane;
  const uint64_t pol = policy_evict_first();
  // the maps are written before the launch (a host copy, or a preceding kernel on the
  // no-allocation path): the launch boundary orders them, no proxy fence is needed
  // (measured: one acquire fence per map cost ~4 us per step)
  if (lane == 0)
    for (int t = TM_T_WR; t < TM_COUNT; ++t) {
      const bool qmap = t >= TM_Q_WG, bf16_expert = t == TM_T_WG || t == TM_T_WU || t == TM_T_WD;  // (Q: FP8)
      if (kFp8 ? !bf16_expert : !qmap) prefetch_tensormap(&p.tmaps[t]);  // the maps this layer has
    }
  if (p.layer > 0) {  // the previous layer's record of completed experts
    for (int w = lane; w < kMaxSlots / 32; w += 32) sm.known_done[w] = 0u;
    __syncwarp();
  }
  bool ok = true, sched_ready = false, n_ok = false, hs_ok = false;
  const int pre = sh.pre;
  int total = 0;  // this layer's units, once its schedule exists (kept: the schedule may be
                  // rebuilt for the next layer while this warp still draws tickets)
  int u = pr.grab();
  bool first_expert = true, first_down = true, first_tma = true;
  unsigned long long c_slot = 0, c_dep = 0, c_grab = 0, c_issue = 0, c_stages = 0, c_units = 0;
  unsigned long long c_setup = 0, c_schedw = 0;
  const long long tploop0 = tclock<kTrace>();
  while (ok) {
    if (u >= pre && !sched_ready) {
      const long long tw0 = tclock<kTrace>();
      ok = pr.wait_bar(&sm.sched_bar, (uint32_t)(p.layer & 1));
      c_schedw += (unsigned long long)(tclock<kTrace>() - tw0);
      if (!ok) break;
      sched_ready = true;
      total = sm.sc.total;
      if (lane == 0) trace_stamp<kTrace>(p, TR_SCHED);
    }
    if (sched_ready && u >= total) break;
    const long long tu0 = tclock<kTrace>();
    const UnitDesc d = decode_unit_tc(sh, sm.sc, u);
    // the next unit's ticket is requested now (its round trip overlaps this unit's
    // issue), except after a router unit: the router units are then spread over the
    // SMs instead of pairs of them landing on the CTAs that start first
    const bool early_grab = d.type != UT_ROUTER;
    uint32_t next_ticket = 0;
    if (lane == 0 && early_grab) next_ticket = atom_add_relaxed(&p.ctr[CTR_QUEUE], 1u);
    const int hunit = (p.layer << 24) | u;  // stage headers name the layer and the unit
    if (lane == 0 && kTrace) {
      if (first_expert && d.type == UT_EXPERT) { trace_stamp<kTrace>(p, TR_FIRST_EXPERT); first_expert = false; }
      if (first_down && (d.type == UT_DOWN_SHARED || d.type == UT_DOWN_EXPERT)) { trace_stamp<kTrace>(p, TR_FIRST_DOWN); first_down = false; }
      ++c_units;
    }
    if ((p.flags & kFlagJitter) && lane == 0) __nanosleep(hash32(blockIdx.x * 7919u + (uint32_t)u) % 3000u);
    TcSeg x;
    make_seg_tc<kFp8, kEp>(p, sh, sm.sc, d, x);
    const bool xf = kFp8 && x.fp8;  // an FP8 stage (compiled out of the bf16 kernel)
    if (xf && !pr.switched && !pr.emit_switch()) {
      ok = false;
      break;
    }
    c_setup += (unsigned long long)(tclock<kTrace>() - tu0);
    // bytes of a stage: on full the activations and (bf16) the weight tiles; on wfull the
    // codes and scales of an FP8 stage
    const int kstep = xf ? 2 : 1;  // K atoms per stage
    const uint32_t tx = (uint32_t)((xf ? 0 : x.nbox * kTcTileBytes) + kstep * x.N * kTcAtomK * 2);
    const uint32_t wtx = (uint32_t)(x.nbox * kFp8TileBytes);
    const int info0 = x.nbox | ((x.N / kTcActRows) << 2) | (xf ? kTcInfoFp8 | (x.sdown ? kTcInfoFp8Down : 0) : 0);
    const int ka_end = d.kb0 + d.nkb;
    // one stage: header, barrier armed for weights + activations, the weight tiles
    auto issue_weights = [&](int ka) {
      uint8_t* dst = ring + pr.slot * sh.slot_bytes;
      uint64_t* fb = &sm.full[pr.slot];
      uint64_t* wb = &sm.wfull[pr.slot];
      pr.mark_pending();
      if (xf) pr.mark_fp8();
      if (lane == 0) {
        StageHeader h;
        h.kind = HK_STAGE;
        h.unit = hunit;
        h.info = info0 | (ka == d.kb0 ? kTcInfoFirst : 0) | (ka + kstep >= ka_end ? kTcInfoLast : 0);
        h.wrow = xf ? x.sc0 + (ka >> 1) : -1;
        sm.hdr[pr.slot] = h;
        if (xf) mbar_arrive_expect_tx(wb, wtx);
        mbar_arrive_expect_tx(fb, tx);
        if (kTrace && first_tma) {
          trace_stamp<kTrace>(p, TR_FIRST_TMA);
          first_tma = false;
        }
        if (xf) {  // codes of K block ka / 2, converted into tensor memory by the routing warps
          tma_load_2d(dst, x.tw0, ka * kTcAtomK, x.y0, wb, pol);
          if (x.nbox == 2) tma_load_2d(dst + kFp8TileBytes, x.tw1, ka * kTcAtomK, x.y1, wb, pol);
        } else {
          tma_load_2d(dst, x.tw0, ka * kTcAtomK, x.y0, fb, pol);
          if (x.nbox == 2) tma_load_2d(dst + kTcTileBytes, x.tw1, ka * kTcAtomK, x.y1, fb, pol);
        }
      }
    };
    // the activation operand of stage ka into ring slot s (only after its publication)
    auto issue_act = [&](int ka, int slot) {
      if (lane == 0) {
        uint8_t* act = ring + slot * sh.slot_bytes + 2 * kTcTileBytes;
        uint64_t* fb = &sm.full[slot];
        if (xf && x.N == kTcActRows && sh.NA == kTcActRows) {
          // an FP8 stage of 16 token rows: both atoms in one copy (the second at +16 x 128 bytes)
          tma_load_3d_plain(act, x.ta2, 0, x.arow, ka, fb);
          return;
        }
        for (int a = 0; a < kstep; ++a)  // an FP8 stage: two atoms, the second at +NA x 128 bytes
          for (int q = 0; q < x.N / kTcActRows; ++q)
            tma_load_2d_plain(act + a * sh.NA * kTcAtomK * 2 + q * kTcActRows * kTcAtomK * 2, x.ta,
                              (ka + a) * kTcAtomK, x.arow + q * kTcActRows, fb);
      }
    };
    bool dep_known = x.dep == 0 ? n_ok
                   : x.dep == 1 ? hs_ok
                                : ((sm.known_done[x.pair >> 5] >> (x.pair & 31)) & 1u) != 0u;
    int ka = d.kb0;
    if (!dep_known) {
      // input not yet published: arm stages with their weight tiles first, so the
      // weights stream while the input is awaited -- a ring's worth for h, one stage
      // for the normalised rows (at the start of the step the HBM queue must stay short
      // for the loads of x that the normalisation waits on)
      // before the schedule of a small step at most nst - 1 stages are in flight, also
      // while arming (arming all nst would wait on the first armed stage, which has no
      // activations yet)
      const int depth = (x.dep == 0 ? 1 : (!sched_ready && p.B <= 4 && pr.nst >= 5 ? pr.nst - 1 : pr.nst)) * kstep;
      const int pre_end = ka_end < d.kb0 + depth ? ka_end : d.kb0 + depth;
      const int slot0 = pr.slot;
      for (; ka < pre_end && ok; ka += kstep) {
        const long long t0 = tclock<kTrace>();
        ok = (sched_ready || pr.wait_slot_pre()) && pr.wait_slot();
        c_slot += (unsigned long long)(tclock<kTrace>() - t0);
        if (!ok) break;
        issue_weights(ka);
        __syncwarp();
        if (xf && !pr.push_conv(pr.slot, pr.last_wpar(), pr.phase)) ok = false;
        pr.advance();
        ++c_stages;
      }
      const int narmed = (ka - d.kb0) / kstep;  // stages
      bool dep_ok = ok;
      const long long td0 = tclock<kTrace>();
      if (ok) {
        if (x.dep == 0) {
          dep_ok = n_ok = pr.wait_dep(&p.ctr[CTR_NREADY], (uint32_t)p.B);
          if (lane == 0) trace_stamp<kTrace>(p, TR_NREADY);
        } else if (x.dep == 1) {
          dep_ok = hs_ok = pr.wait_dep(&p.ctr[CTR_HS], (uint32_t)sh.hs_target);
        } else {
          dep_ok = pr.wait_pair(x.pair);
        }
      }
      c_dep += (unsigned long long)(tclock<kTrace>() - td0);
      // every armed barrier gets its activation bytes, also after a failed wait
      for (int i = 0; i < narmed; ++i) issue_act(d.kb0 + i * kstep, (slot0 + i) % pr.nst);
      __syncwarp();
      if (!dep_ok) ok = false;
    }
    for (; ka < ka_end && ok; ka += kstep) {
      {
        const long long t0 = tclock<kTrace>();
        ok = (sched_ready || pr.wait_slot_pre()) && pr.wait_slot();
        c_slot += (unsigned long long)(tclock<kTrace>() - t0);
      }
      if (!ok) break;
      const long long ti0 = tclock<kTrace>();
      const int slot = pr.slot;
      issue_weights(ka);
      issue_act(ka, slot);
      __syncwarp();
      if (xf && !pr.push_conv(pr.slot, pr.last_wpar(), pr.phase)) ok = false;
      pr.advance();
      c_issue += (unsigned long long)(tclock<kTrace>() - ti0);
      ++c_stages;
    }
    {
      const long long t0 = tclock<kTrace>();
      if (lane == 0 && !early_grab) next_ticket = atom_add_relaxed(&p.ctr[CTR_QUEUE], 1u);
      u = __shfl_sync(0xffffffffu, (int)next_ticket, 0);
      c_grab += (unsigned long long)(tclock<kTrace>() - t0);
    }
  }
  if (lane == 0 && kTrace) {
    trace_stamp<kTrace>(p, TR_PROD_END);
    trace_put<kTrace>(p, TR_PROD_WAIT_SLOT_CYC, c_slot);
    trace_put<kTrace>(p, TR_PROD_WAIT_DEP_CYC, c_dep);
    trace_put<kTrace>(p, TR_PROD_GRAB_CYC, c_grab);
    trace_put<kTrace>(p, TR_PROD_ISSUE_CYC, c_issue);
    trace_put<kTrace>(p, TR_PROD_STAGES, c_stages);
    trace_put<kTrace>(p, TR_UNITS, c_units);
    trace_put<kTrace>(p, TR_PROD_SETUP_CYC, c_setup);
    trace_put<kTrace>(p, TR_PROD_SCHED_CYC, c_schedw);
    trace_put<kTrace>(p, TR_PROD_LOOP_CYC, (unsigned long long)(tclock<kTrace>() - tploop0));
  }
  if (last || !ok) pr.finish(kFp8);
  return ok;
}

// ---- CUDA-core path: MAC warps and the epilogue warp ------------------------------------------

template <bool kTrace>
__device__ void mac_warps_cc(const Params& p, Smem& sm, uint8_t* ring, int mw, int lane) {
  uint32_t mphase = 0;
  bool ok = normalise_rows<kTrace>(p, sm, mw, lane, mphase);
  int slot = 0;
  uint32_t phase = 0;
  int ub = 0;
  uint32_t ubphase = 0;
  bool rb_claimed = false;
  float acc[2][kRowsPerWarp][kActGroup];
  zero_acc(acc);
  const long long tloop0 = tclock<kTrace>();
  unsigned long long c_full = 0, c_rb = 0, c_comp = 0, c_st = 0, c_sched = 0, c_red = 0;
  while (ok) {
    {
      const long long t0 = tclock<kTrace>();
      const bool got = warp_wait(&sm.full[slot], phase, p, lane, 0);
      c_full += (unsigned long long)(tclock<kTrace>() - t0);
      if (!got) break;
    }
    const StageHeader hd = sm.hdr[slot];
    if (hd.kind == HK_END) {
      if (mw == 0 && lane == 0) trace_stamp<kTrace>(p, TR_MAC_END);
      break;
    }
    if (hd.kind == HK_SCHED) {
      const long long ts0 = tclock<kTrace>();
      ok = build_schedule<kTrace>(p, sm, mw, lane, mphase);
      c_sched += (unsigned long long)(tclock<kTrace>() - ts0);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
      if (mw == 0 && lane == 0 && ok) mbar_arrive(&sm.sched_bar);
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1u;
      }
      continue;
    }
    const int info = hd.info;
    const int kpair = (info & kInfoKpair) ? 1 : 0;
    const int nbox = info & 3;
    const int c = (info >> 3) & 7;
    const int box_cols = info >> 16;
    if (info & kInfoFirst) {
      zero_acc(acc);
      rb_claimed = false;
      if ((p.flags & kFlagJitter) && lane == 0) __nanosleep(hash32(hd.unit * 131u + mw * 7u + blockIdx.x) % 1500u);
      __syncwarp();
    }
    const long long tc0 = tclock<kTrace>();
    mac_dispatch(ring + slot * kSlotBytes, kpair, nbox, box_cols, c, acc, mw, lane);
    __syncwarp();
    c_comp += (unsigned long long)(tclock<kTrace>() - tc0);
    ++c_st;
    if (lane == 0) mbar_arrive(&sm.empty[slot]);
    if (++slot == kStages) {
      slot = 0;
      phase ^= 1u;
    }
    const bool unit_end = (info & kInfoUnitEnd) != 0;
    const bool seg_end = (info & kInfoSegEnd) != 0;
    const long long tr0 = tclock<kTrace>();
    if (seg_end) {
      if (!rb_claimed) {
        const long long t0 = tclock<kTrace>();
        const bool got = warp_wait(&sm.rb_empty[ub], ubphase ^ 1u, p, lane, 0);
        c_rb += (unsigned long long)(tclock<kTrace>() - t0);
        if (!got) break;
        rb_claimed = true;
      }
      if (hd.wrow >= 0) {
        reduce_to(acc, 1, sm.rb[ub], (info >> 8) & 1, &sm.sc.w_of[hd.wrow], c, mw, lane);
        zero_acc(acc);
      } else {
        reduce_to(acc, kpair ? 1 : 2, sm.rb[ub], 0, nullptr, c, mw, lane);
      }
    }
    if (unit_end) {
      if (mw == 0 && lane == 0) sm.rb_unit[ub] = hd.unit;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.rb_full[ub]);
      if (++ub == kRB) {
        ub = 0;
        ubphase ^= 1u;
      }
      rb_claimed = false;
    }
    if (seg_end || unit_end) c_red += (unsigned long long)(tclock<kTrace>() - tr0);
  }
  if (mw == 0 && lane == 0 && kTrace) {
    trace_put<kTrace>(p, TR_MAC_LOOP_CYC, (unsigned long long)(tclock<kTrace>() - tloop0));
    trace_put<kTrace>(p, TR_MAC_WAIT_FULL_CYC, c_full);
    trace_put<kTrace>(p, TR_MAC_WAIT_RB_CYC, c_rb);
    trace_put<kTrace>(p, TR_MAC_COMPUTE_CYC, c_comp);
    trace_put<kTrace>(p, TR_MAC_STAGES, c_st);
    trace_put<kTrace>(p, TR_MAC_SCHED_CYC, c_sched);
    trace_put<kTrace>(p, TR_MAC_REDUCE_CYC, c_red);
  }
  // tell the epilogue warp to stop (bounded)
  if (warp_wait(&sm.rb_empty[ub], ubphase ^ 1u, p, lane)) {
    if (mw == 0 && lane == 0) sm.rb_unit[ub] = -1;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.rb_full[ub]);
  }
}

template <bool kTrace>
__device__ void epilogue_cc(const Params& p, Smem& sm, int lane) {
  int ub = 0;
  uint32_t ubphase = 0;
  unsigned long long c_busy = 0;
  for (;;) {
    if (!warp_wait(&sm.rb_full[ub], ubphase, p, lane)) break;
    const int u = sm.rb_unit[ub];
    if (u < 0 || abort_seen(p)) {
      if (lane == 0 && kTrace) {
        trace_stamp<kTrace>(p, TR_EPI_END);
        trace_put<kTrace>(p, TR_EPI_BUSY_CYC, c_busy);
      }
      break;
    }
    const UnitDesc d = decode_unit(sm.sh, sm.sc, u);
    const long long t0 = tclock<kTrace>();
    epi_finish(p, sm, d, u, sm.rb[ub], lane);
    c_busy += (unsigned long long)(tclock<kTrace>() - t0);
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.rb_empty[ub]);
    if (++ub == kRB) {
      ub = 0;
      ubphase ^= 1u;
    }
  }
}

// ---- tensor-core path: FP8 converters (the routing warps, once the schedule exists) --------------

// Four E4M3 codes (byte i of w = code i) to two bf16 pairs (codes 0, 1 and 2, 3), each
// value(code) x 2^-120 exactly, with integer operations only: a code's 7 magnitude bits
// (exponent field e, mantissa m) become the low bits of the bf16's exponent field and the
// top 3 of its mantissa, so the bf16 reads 2^(e-127) (1 + m/8) = value x 2^-120 for e >= 1
// and 2^-126 (m/8) = value x 2^-120 (a bf16 subnormal) for e = 0. With v = [0, c1, 0, c0]
// in 16-bit lanes, adding 15 x (v's sign bits 7 and 23) moves each sign 4 places up
// (bit 7 + 15 x 2^7 = 2^11), and the shift by 4 puts the magnitudes at bits 4-10 of their
// lanes and the signs at bits 15 and 31.
__device__ __forceinline__ void e4m3x4_to_bf16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t v0 = __byte_perm(w, 0u, 0x4140), v1 = __byte_perm(w, 0u, 0x4342);
  lo = (v0 + 15u * (v0 & 0x00800080u)) << 4;
  hi = (v1 + 15u * (v1 & 0x00800080u)) << 4;
}

// bf16 pair (s x 2^120, s x 2^120) of a power-of-two fp32 scale s in [2^-117, 2^7]: times
// a converted code it gives the weight value(code) x s exactly (a bf16 normal, >= 2^-126).
__device__ __forceinline__ uint32_t scale_bf16x2(float s) {
  // exact: a power of two has no mantissa bits; the exponent field grows by 120
  const uint32_t b = (__float_as_uint(s) >> 16) + (120u << 7);
  return (b << 16) | b;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The routing warps turn every FP8 stage (handed over by the producer through the
// converter queue) into the MMA's A operand in tensor memory: warp w (of 8) converts
// tile w / 4 of the stage, lane l the tile row 32 q + l of its lane quadrant q (its 128
// codes, each times the scale of the tile's 128 x 128 block), and stores the row's 128
// bf16 values as 64 columns of its lane. The codes sit 128-byte swizzled (chunk c of row
// r at chunk c ^ (r mod 8)), so the 8 lanes of a shared-memory phase read 8 distinct
// 16-byte chunks while the whole warp reads one logical chunk. A stages rotate in stage
// order; one is rewritten only after the MMAs that read it completed. With its A stage a
// stage's activations (two K atoms) are copied in front of the ring and its header into
// Smem::ahdr, so the slot is released (cdone) once converted, before the MMAs run. The
// warps need nothing from one another: each waits for the stage itself (bounded) and
// signals its part done on the slot's cdone and the A stage's conv_bar; the end of the
// stages reaches the MMA warp the same way (an HK_END header in the next A stage).
template <bool kTrace>
__device__ void convert_fp8_stages(const Params& p, Smem& sm, uint8_t* ring, uint8_t* actring, int mw, int lane,
                                   bool ok) {
  if (!ok) return;
  unsigned long long c_wait = 0, c_work = 0;
  struct Flush {  // the warp's cycle counts into the trace (warp 0) on every way out
    const Params& p;
    int mw, lane;
    unsigned long long &w, &k;
    __device__ ~Flush() {
      if (kTrace && mw == 0 && lane == 0) {
        trace_put<kTrace>(p, TR_CONV_WAIT_CYC, w);
        trace_put<kTrace>(p, TR_CONV_WORK_CYC, k);
      }
    }
  } flush{p, mw, lane, c_wait, c_work};
  const Shape& sh = sm.sh;
  const int quad = (mw + 1) & 3;     // lane quadrant of this warp (warp id mod 4)
  const int j = mw >> 2;             // weight tile
  const int r = quad * 32 + lane;    // tile row = tensor-memory lane
  const uint32_t tq = sm.tmem_base + ((uint32_t)(quad * 32) << 16) +
                      (uint32_t)(kFp8AccBufs * sh.acc_cols + j * (kFp8AStageCols / 2));
  const int swz = r & 7;
  int q = 0, as = 0;
  uint32_t qph = 0u, asph = 0u;
  for (;;) {
    const long long t0 = tclock<kTrace>();
    if (!warp_wait(&sm.cq_full[q], qph, p, lane, 64)) return;
    const int slot = sm.cq_slot[q];
    const uint32_t par = sm.cq_par[q], fpar = sm.cq_fpar[q];
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.cq_empty[q]);  // the entry is read
    if (++q == kCq) {
      q = 0;
      qph ^= 1u;
    }
    if (slot < 0) {  // the end, in the next A stage once the MMAs left it
      if (!warp_wait(&astage_empty(sm)[as], asph ^ 1u, p, lane, 64)) return;
      if (mw == 0 && lane == 0) sm.ahdr[as].kind = HK_END;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.conv_bar[as]);
      return;
    }
    if (!IDX_OK(p, slot < sh.nst)) return;
    // the header was written before the queue entry: the tile's scale loads while the
    // codes are still in flight
    const StageHeader hd = sm.hdr[slot];
    const bool conv = j < (hd.info & 3);
    float sv = 0.0f;
    if (conv) {
      const bool down = (hd.info & kTcInfoFp8Down) != 0;
      const float* sa = down ? p.sc_down : (j ? p.sc_up : p.sc_gate);
      sv = __ldg(sa + hd.wrow + (down && j ? p.I / kTcRows : 0));
    }
    if (!warp_wait(&sm.wfull[slot], par, p, lane, 64)) return;
    if (!warp_wait(&sm.full[slot], fpar, p, lane, 64)) return;                // its activations
    if (!warp_wait(&astage_empty(sm)[as], asph ^ 1u, p, lane, 64)) return;  // the A stage is free
    const long long t1 = tclock<kTrace>();
    c_wait += (unsigned long long)(t1 - t0);
    {  // the activations of both atoms (n rows each, the second at +NA x 128 bytes), as laid out
      const int n = ((hd.info >> 2) & 7) * kTcActRows;
      const uint8_t* src = ring + slot * sh.slot_bytes + 2 * kTcTileBytes;
      uint8_t* dst = actring + as * fp8_act_stage_bytes(sh.NA);
      const int chunks = n * (kTcAtomK * 2 / 16);  // 16-byte chunks per atom
      for (int i = mw * 32 + lane; i < 2 * chunks; i += kMacThreads) {
        const int a = i >= chunks ? 1 : 0, c = i - a * chunks;
        const int off = a * sh.NA * kTcAtomK * 2 + c * 16;
        *reinterpret_cast<uint4*>(dst + off) = *reinterpret_cast<const uint4*>(src + off);
      }
    }
    if (conv) {
      tc_fence_after();
      const uint8_t* sbase = ring + slot * sh.slot_bytes;
      const uint32_t sc = scale_bf16x2(sv);
      const uint8_t* row = sbase + j * kFp8TileBytes + r * (2 * kTcAtomK);
      const uint32_t col = (uint32_t)(as * kFp8AStageCols);
#pragma unroll
      for (int h = 0; h < 2; ++h) {  // codes 64 h .. 64 h + 63
        uint4 v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) v[c] = *reinterpret_cast<const uint4*>(row + (((4 * h + c) ^ swz) << 4));
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t w[4] = {v[c].x, v[c].y, v[c].z, v[c].w};
          uint32_t o[8];
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            e4m3x4_to_bf16x2x2(w[t], o[2 * t], o[2 * t + 1]);
            o[2 * t] = mul_bf16x2(o[2 * t], sc);
            o[2 * t + 1] = mul_bf16x2(o[2 * t + 1], sc);
          }
          tmem_st8(tq + col + (uint32_t)(8 * (4 * h + c)), o);  // K elements 16 (4h + c) .. + 15
        }
      }
      tmem_st_wait();
    }
    if (mw == 0 && lane == 0) sm.ahdr[as] = hd;
    fence_proxy_async_shared();  // the copied activations, then the tensor cores' reads
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&sm.cdone[slot]);  // the slot is free
      mbar_arrive(&sm.conv_bar[as]);
    }
    if (++as == sh.nas) {
      as = 0;
      asph ^= 1u;
    }
    c_work += (unsigned long long)(tclock<kTrace>() - t1);
  }
}

// ---- tensor-core path: MMA warp --------------------------------------------------------------------

// One elected lane issues, per stage, 4 K-steps of 16 for each weight tile into the
// unit's accumulator buffer, then commits the stage's slot back to the producer
// (the slot is free once those MMAs have read it). At a unit's last stage the buffer
// is handed to the epilogue warps: one commit arrive (the MMAs are complete) plus one
// plain arrive that publishes the unit id.
template <bool kTrace, bool kFp8 = false>
__device__ void mma_warp(const Params& p, Smem& sm, uint8_t* ring, int lane, uint8_t* aring = nullptr) {
  const uint32_t tmem = sm.tmem_base;
  int slot = 0;
  uint32_t phase = 0;
  int abuf = 0;
  uint32_t aphase = 0;
  bool issued = false;
  bool amode = false;  // FP8: the stages come from the tensor-memory A stages (after HK_SWITCH)
  int as = 0;          // FP8: the next A stage and its conv_bar parity
  uint32_t asph = 0u;
  unsigned long long c_full = 0, c_acc = 0, c_st = 0, c_issue = 0, c_conv = 0;
  const long long tloop0 = tclock<kTrace>();
  for (;;) {
    StageHeader hd;
    if (!amode) {
      const long long t0 = tclock<kTrace>();
      const bool got = warp_wait(&sm.full[slot], phase, p, lane);
      c_full += (unsigned long long)(tclock<kTrace>() - t0);
      if (!got) break;
      hd = sm.hdr[slot];
      if (kFp8 && hd.kind == HK_SWITCH) {  // the slot carries no tiles; the A stages follow
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
        __syncwarp();
        if (++slot == sm.sh.nst) {
          slot = 0;
          phase ^= 1u;
        }
        amode = true;
        continue;
      }
    } else {  // the converters filled A stage `as` (weights in tensor memory, activations beside)
      const long long t0 = tclock<kTrace>();
      const bool got = warp_wait(&sm.conv_bar[as], asph, p, lane, 64);
      c_conv += (unsigned long long)(tclock<kTrace>() - t0);
      if (!got) break;
      hd = sm.ahdr[as];
    }
    if (hd.kind == HK_END) {
      if (lane == 0) trace_stamp<kTrace>(p, TR_MAC_END);
      break;
    }
    const int info = hd.info;
    const bool first = (info & kTcInfoFirst) != 0;
    const bool last = (info & kTcInfoLast) != 0;
    if (first) {
      const long long t0 = tclock<kTrace>();
      const bool got = warp_wait(&sm.acc_empty[abuf], aphase ^ 1u, p, lane);
      c_acc += (unsigned long long)(tclock<kTrace>() - t0);
      if (!got) break;
    }
    tc_fence_after();
    const long long ti0 = tclock<kTrace>();
    if (lane == 0) {
      const int nbox = info & 3;
      const uint32_t idesc = idesc_bf16_m128((uint32_t)((info >> 2) & 7) * kTcActRows);
      const uint32_t acols = kFp8 ? (uint32_t)sm.sh.acc_cols : (uint32_t)kTcAccCols;
      const uint32_t t0 = tmem + abuf * acols;
      if (kFp8 && amode) {
        // one 128-column K block: 8 K steps of A from tensor memory; the activations of the
        // two atoms beside the A stage, the second at +NA x 128 bytes
        const uint32_t a0 = tmem + kFp8AccBufs * acols + (uint32_t)(as * kFp8AStageCols);
        const uint32_t abase = smem_u32(aring + as * fp8_act_stage_bytes(sm.sh.NA));
        const uint64_t da = sw128_desc(abase);
        const uint64_t da1 = sw128_desc(abase + (uint32_t)(sm.sh.NA * kTcAtomK * 2));
#pragma unroll
        for (int ks = 0; ks < 2 * kTcAtomK / 16; ++ks) {
          const uint32_t accum = (first && ks == 0) ? 0u : 1u;
          const uint64_t db = (ks < 4 ? da : da1) + (uint64_t)(2 * (ks & 3));
          tc_mma_bf16_ta(t0, a0 + (uint32_t)(8 * ks), db, idesc, accum);
          if (nbox == 2) tc_mma_bf16_ta(t0 + acols / 2, a0 + (uint32_t)(kFp8AStageCols / 2 + 8 * ks), db, idesc, accum);
        }
        tc_commit(&astage_empty(sm)[as]);
      } else {
        const uint32_t sbase = smem_u32(ring + slot * sm.sh.slot_bytes);
        const uint64_t dw0 = sw128_desc(sbase);
        const uint64_t dw1 = sw128_desc(sbase + kTcTileBytes);
        const uint64_t da = sw128_desc(sbase + 2 * kTcTileBytes);
#pragma unroll
        for (int ks = 0; ks < kTcAtomK / 16; ++ks) {
          const uint32_t accum = (first && ks == 0) ? 0u : 1u;
          tc_mma_bf16(t0, dw0 + (uint64_t)(2 * ks), da + (uint64_t)(2 * ks), idesc, accum);
          if (nbox == 2) tc_mma_bf16(t0 + acols / 2, dw1 + (uint64_t)(2 * ks), da + (uint64_t)(2 * ks), idesc, accum);
        }
        tc_commit(&sm.empty[slot]);
      }
      if (last) {
        sm.acc_unit[abuf] = hd.unit;
        tc_commit(&sm.acc_full[abuf]);
        mbar_arrive(&sm.acc_full[abuf]);
      }
    }
    issued = true;
    __syncwarp();
    c_issue += (unsigned long long)(tclock<kTrace>() - ti0);
    ++c_st;
    if (last) {
      if (++abuf == (kFp8 ? kFp8AccBufs : kTcAccBufs)) {
        abuf = 0;
        aphase ^= 1u;
      }
    }
    if (kFp8 && amode) {
      if (++as == sm.sh.nas) {
        as = 0;
        asph ^= 1u;
      }
    } else if (++slot == sm.sh.nst) {
      slot = 0;
      phase ^= 1u;
    }
  }
  if (lane == 0 && kTrace) {
    trace_put<kTrace>(p, TR_MAC_LOOP_CYC, (unsigned long long)(tclock<kTrace>() - tloop0));
    trace_put<kTrace>(p, TR_MAC_WAIT_FULL_CYC, c_full);
    trace_put<kTrace>(p, TR_MMA_WAIT_CONV_CYC, c_conv);
    trace_put<kTrace>(p, TR_MAC_WAIT_RB_CYC, c_acc);
    trace_put<kTrace>(p, TR_MAC_COMPUTE_CYC, c_issue);
    trace_put<kTrace>(p, TR_MAC_STAGES, c_st);
  }
  // stop the epilogue warps (bounded)
  if (warp_wait(&sm.acc_empty[abuf], aphase ^ 1u, p, lane)) {
    if (lane == 0) {
      sm.acc_unit[abuf] = -1;
      mbar_arrive(&sm.acc_full[abuf]);
      mbar_arrive(&sm.acc_full[abuf]);
    }
  }
  __syncwarp();
  // every MMA this warp issued completes before the CTA gives up its shared and tensor
  // memory. MMAs that never complete are reported; the tensor memory is still freed
  // (a CTA that kept it would leave its SM's next allocation waiting without bound).
  if (issued && lane == 0) {
    tc_commit(&sm.mma_bar);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&sm.mma_bar, 0u)) {
      if (globaltimer_ns() - t0 > 50000000ull) {
        record_abort(p, MOE_ERR_TIMEOUT);
        break;
      }
    }
  }
  __syncwarp();
}

// ---- tensor-core path: epilogue warps --------------------------------------------------------------

// Rendezvous of the 4 epilogue warps (an mbarrier with bounded waits, so a warp that
// gives up never leaves the others blocked).
__device__ __forceinline__ bool epi_sync(Smem& sm, uint32_t& phase, const Params& p, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(&sm.epi_bar);
  const bool ok = warp_wait(&sm.epi_bar, phase, p, lane, 0);
  phase ^= 1u;
  return ok;
}

// Loads accumulator columns [j0, j0 + 16) of both tiles of the buffer (lane quadrant of
// the calling warp). `two` is warp-uniform.
// Columns j0 .. j0 + 15 of tile 0 (v0) and, if two, of tile 1 (v1, `half` columns on).
__device__ __forceinline__ void tmem_cols16(uint32_t ta, int j0, bool two, uint32_t (&v0)[16], uint32_t (&v1)[16],
                                            uint32_t half = kTcAccCols / 2) {
  tmem_ld16(ta + (uint32_t)j0, v0);
  if (two) tmem_ld16(ta + half + (uint32_t)j0, v1);
  tmem_ld_wait();
  tmem_regs_after_wait(v0);
  if (two) tmem_regs_after_wait(v1);
}

// The fix-up of a gate/up tile whose splits are all done: fixed split order, so the
// sums do not depend on which split finished last. Thread et (0..127) owns tile row et.
__device__ void fixup_tc(const Params& p, const Smem& sm, const UnitDesc& d, int et) {
  const Shape& sh = sm.sh;
  const Sched& sc = sm.sc;
  if (d.type == UT_SHARED) {
    for (int b = 0; b < sh.B; ++b) {
      float g = 0.0f, u = 0.0f;
      for (int sp = 0; sp < d.nsplit; ++sp) {
        const float* src = p.spart + (((size_t)sp * sh.B + b) * sh.ST + d.tile) * (2 * kTcRows);
        g += __ldcg(src + et);
        u += __ldcg(src + kTcRows + et);
      }
      p.hs[(size_t)b * p.Is + d.tile * kTcRows + et] = f2bf(silu(g) * u);
    }
  } else {
    const int i = sc.pair_slot[d.pair];
    const int r0 = sc.slot_base[i], cnt = sc.slot_cnt[i];
    for (int j = 0; j < cnt; ++j) {
      if (!IDX_OK(p, (unsigned)(r0 + j) < (unsigned)sc.S && (unsigned)sc.S <= p.cap_slots)) break;
      float g = 0.0f, u = 0.0f;
      for (int sp = 0; sp < d.nsplit; ++sp) {
        const float* src = p.epart + (((size_t)sp * sc.S + r0 + j) * sh.IT + d.tile) * (2 * kTcRows);
        g += __ldcg(src + et);
        u += __ldcg(src + kTcRows + et);
      }
      p.he[(size_t)(r0 + j) * p.I + d.tile * kTcRows + et] = f2bf(silu(g) * u);
    }
  }
}

// Rows rows[0..n) of down tile pair t once each has all its k expert contributions and
// the shared one: y = bf16(x + s + sum_j w_j d_j), the shared part first, then the
// row's choices in top-k order. Down partial rows: the shared expert's token row b at
// b, expert slot row r at B + r. 64 threads cover a row's 256 features four at a
// time (128-bit loads), two rows per pass. A step over an expert range (y_part set)
// sums the row's choices among its experts (slot_of >= 0) and writes the fp32 partial,
// with x + s only when ep_rs.
template <bool kEp>
__device__ void combine_rows_tc(const Params& p, const Smem& sm, int t, const int16_t* rows, int n, int et) {
  const Shape& sh = sm.sh;
  const Sched& sc = sm.sc;
  const int h = t * 2 * kTcRows + 4 * (et & 63);
  if (h >= p.H) return;
  for (int ci = et >> 6; ci < n; ci += 2) {
    const int b = rows[ci];
    if (!IDX_OK(p, b < sh.B)) continue;
    const int16_t* so = &sc.slot_of[b * sh.k];
#ifdef MOE_BOUNDS_CHECK
    bool bad = false;
    for (int j = 0; j < sh.k; ++j) bad = bad || ((!kEp || so[j] >= 0) && (unsigned)so[j] >= (unsigned)sc.S);
    if (!IDX_OK(p, !bad)) continue;
#endif
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    if (!kEp || p.ep_rs) acc = __ldcg(reinterpret_cast<const float4*>(p.dpart + (size_t)b * p.H + h));
    for (int j0 = 0; j0 < sh.k; j0 += 8) {
      float4 v[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
        if (j0 + jj < sh.k && (!kEp || so[j0 + jj] >= 0))
          v[jj] = __ldcg(reinterpret_cast<const float4*>(p.dpart + (size_t)(sh.B + so[j0 + jj]) * p.H + h));
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (j0 + jj < sh.k && (!kEp || so[j0 + jj] >= 0)) {
          const float w = sc.w_of[so[j0 + jj]];
          acc.x = fmaf(w, v[jj].x, acc.x);
          acc.y = fmaf(w, v[jj].y, acc.y);
          acc.z = fmaf(w, v[jj].z, acc.z);
          acc.w = fmaf(w, v[jj].w, acc.w);
        }
      }
    }
    if (kEp && p.y_part) {  // the fp32 partial of a step over an expert range
      if (p.ep_rs) {
        const uint2 xv = __ldcg(reinterpret_cast<const uint2*>(p.x + (size_t)b * p.H + h));
        acc.x += bf2f(xv.x & 0xFFFFu);
        acc.y += bf2f(xv.x >> 16);
        acc.z += bf2f(xv.y & 0xFFFFu);
        acc.w += bf2f(xv.y >> 16);
      }
      *reinterpret_cast<float4*>(p.y_part + (size_t)b * p.H + h) = acc;
      continue;
    }
    const uint2 xv = __ldcg(reinterpret_cast<const uint2*>(p.x + (size_t)b * p.H + h));
    uint2 yv;
    yv.x = (uint32_t)f2bf(bf2f(xv.x & 0xFFFFu) + acc.x) | ((uint32_t)f2bf(bf2f(xv.x >> 16) + acc.y) << 16);
    yv.y = (uint32_t)f2bf(bf2f(xv.y & 0xFFFFu) + acc.z) | ((uint32_t)f2bf(bf2f(xv.y >> 16) + acc.w) << 16);
    *reinterpret_cast<uint2*>(p.y + (size_t)b * p.H + h) = yv;
  }
}

// The bf16 output of an expert-parallel step once the ranks' fp32 partials are summed.
__global__ void partial_to_bf16_kernel(const float* __restrict__ in, uint16_t* __restrict__ out, long long n) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) out[i] = f2bf(in[i]);
}

// F: the layers of a fused launch (a unit's header names its layer), or nullptr when
// the launch runs the one layer p0.
template <bool kTrace, bool kFp8 = false, bool kEp = false>
__device__ void epilogue_tc(const Params& p0, Smem& sm, int warp_id, int lane, const FusedParams* F = nullptr) {
  const Shape& sh = sm.sh;
  const int quad = warp_id & 3;
  const int row = quad * 32 + lane;                        // accumulator lane = tile row
  const int et = (warp_id - kTcEpiWarp0) * 32 + lane;       // 0..127 for the fix-ups
  const uint32_t tq = sm.tmem_base + ((uint32_t)(quad * 32) << 16);
  int abuf = 0;
  uint32_t aphase = 0, ephase = 0;
  int sched_layer = -1;  // the last layer whose schedule this warp has seen
  unsigned long long c_busy = 0;
  for (;;) {
    if (!warp_wait(&sm.acc_full[abuf], aphase, p0, lane)) break;
    const int hu = sm.acc_unit[abuf];
    if (hu < 0) {
      if (lane == 0 && kTrace && warp_id == kTcEpiWarp0) {
        trace_stamp<kTrace>(p0, TR_EPI_END);
        trace_put<kTrace>(p0, TR_EPI_BUSY_CYC, c_busy);
      }
      break;
    }
    const int layer = hu >> 24, u = hu & 0xFFFFFF;
    const Params& p = F ? F->layer[layer] : p0;
    tc_fence_after();
    const long long tb0 = tclock<kTrace>();
    const Sched& sc = sm.sc;
    const UnitDesc d = decode_unit_tc(sh, sc, u);
    const uint32_t acols = kFp8 ? (uint32_t)sh.acc_cols : (uint32_t)kTcAccCols;  // tile 1 at +acols / 2
    const uint32_t ta = tq + abuf * acols;
    const bool direct = d.nsplit == 1 && (d.type == UT_SHARED || d.type == UT_EXPERT);
    uint32_t v0[16], v1[16];
    switch (d.type) {
      case UT_ROUTER: {
        const int e0 = d.tile * 2 * kTcRows + row, e1 = e0 + kTcRows;
        const bool two = d.tile * 2 * kTcRows + kTcRows < p.E;
        // this split's partial logits; the row owners sum the splits
        float* dst = p.rpart + (size_t)d.split * sh.B * p.E;
        for (int j0 = 0; j0 < sh.B; j0 += 16) {
          tmem_cols16(ta, j0, two, v0, v1, acols / 2);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int b = j0 + jj;
            if (b < sh.B) {
              dst[(size_t)b * p.E + e0] = __uint_as_float(v0[jj]);
              if (two) dst[(size_t)b * p.E + e1] = __uint_as_float(v1[jj]);
            }
          }
        }
        break;
      }
      case UT_SHARED: {
        for (int j0 = 0; j0 < sh.B; j0 += 16) {
          tmem_cols16(ta, j0, true, v0, v1, acols / 2);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int b = j0 + jj;
            if (b < sh.B) {
              const float g = __uint_as_float(v0[jj]), uu = __uint_as_float(v1[jj]);
              if (direct) {
                p.hs[(size_t)b * p.Is + d.tile * kTcRows + row] = f2bf(silu(g) * uu);
              } else {
                float* dst = p.spart + (((size_t)d.split * sh.B + b) * sh.ST + d.tile) * (2 * kTcRows);
                dst[row] = g;
                dst[kTcRows + row] = uu;
              }
            }
          }
        }
        break;
      }
      case UT_EXPERT: {
        // the expert's rows are scattered token columns: one column load per row
        const int i = sc.pair_slot[d.pair];
        const int r0 = sc.slot_base[i];
        int cnt = sc.slot_cnt[i];
        if (!IDX_OK(p, (unsigned)(r0 + cnt) <= (unsigned)sc.S && (unsigned)sc.S <= p.cap_slots)) cnt = 0;
        for (int j0 = 0; j0 < cnt; j0 += 8) {
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int j = j0 + jj < cnt ? j0 + jj : j0;
            uint32_t col = (uint32_t)sc.row_of[r0 + j];
            if (!IDX_OK(p, col < (uint32_t)sh.NA)) col = 0;
            tmem_ld1(ta + col, v0[jj]);
            tmem_ld1(ta + acols / 2 + col, v1[jj]);
          }
          tmem_ld_wait();
          tmem_regs_after_wait(v0);
          tmem_regs_after_wait(v1);
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int j = j0 + jj;
            if (j < cnt) {
              const float g = __uint_as_float(v0[jj]), uu = __uint_as_float(v1[jj]);
              if (direct) {
                p.he[(size_t)(r0 + j) * p.I + d.tile * kTcRows + row] = f2bf(silu(g) * uu);
              } else {
                float* dst = p.epart + (((size_t)d.split * sc.S + r0 + j) * sh.IT + d.tile) * (2 * kTcRows);
                dst[row] = g;
                dst[kTcRows + row] = uu;
              }
            }
          }
        }
        break;
      }
      default: {
        // down: unweighted partial rows of the source (token rows 0..B-1 for the shared
        // expert, B + slot row for an expert), combined per row once all have arrived
        const bool shared = d.type == UT_DOWN_SHARED;
        const int i = shared ? 0 : sc.pair_slot[d.pair];
        const int r0 = shared ? 0 : sh.B + sc.slot_base[i];
        int cnt = shared ? sh.B : sc.slot_cnt[i];
        if (!IDX_OK(p, (unsigned)(r0 + cnt) <= p.cap_dpart_rows)) cnt = 0;
        const int h0 = d.tile * 2 * kTcRows + row, h1 = h0 + kTcRows;
        const bool two = d.tile * 2 * kTcRows + kTcRows < p.H;
        for (int j0 = 0; j0 < cnt; j0 += 16) {
          tmem_cols16(ta, j0, two, v0, v1, acols / 2);
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = j0 + jj;
            if (j < cnt) {
              float* dst = p.dpart + (size_t)(r0 + j) * p.H;
              dst[h0] = __uint_as_float(v0[jj]);
              if (two) dst[h1] = __uint_as_float(v1[jj]);
            }
          }
        }
        break;
      }
    }
    // accumulator buffer back to the MMA warp
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.acc_empty[abuf]);
    if (++abuf == (kFp8 ? kFp8AccBufs : kTcAccBufs)) {
      abuf = 0;
      aphase ^= 1u;
    }
    if (d.type == UT_DOWN_SHARED || d.type == UT_DOWN_EXPERT) {
      // count this source in for each of its rows; the unit that brings a row's last
      // contribution (k experts + the shared expert) combines that row of the tile
      __threadfence();
      if (!epi_sync(sm, ephase, p, lane)) break;
      const bool shared = d.type == UT_DOWN_SHARED;
      const bool ranged = kEp && (p.ep_e0 > 0 || p.ep_e1 < p.E);  // a step over an expert range
      if (ranged && shared && sched_layer < layer) {
        // its rows' contribution counts come from the schedule, which a shared-expert
        // tile can precede (this CTA's router units, queued earlier, are done)
        if (!warp_wait(&sm.sched_bar, (uint32_t)(layer & 1), p, lane)) break;
        sched_layer = layer;
      }
      const int i = shared ? 0 : sc.pair_slot[d.pair];
      const int cnt = shared ? sh.B : sc.slot_cnt[i];
      if (et < cnt &&
          IDX_OK(p, shared || ((unsigned)(sc.slot_base[i] + et) < (unsigned)kMaxSlots &&
                               sc.row_of[sc.slot_base[i] + et] < sh.B))) {
        const int b = shared ? et : sc.row_of[sc.slot_base[i] + et];
        // the row's contributions: the shared expert and its choices among this step's experts
        int kloc = sh.k;
        if (ranged) {
          kloc = 0;
          for (int j = 0; j < sh.k; ++j) kloc += sc.slot_of[b * sh.k + j] >= 0 ? 1 : 0;
        }
        uint32_t* tix = &p.row_tix[d.tile * sh.B + b];
        const uint32_t old = atom_add_acq_rel(tix, 1u);
        if (old == (uint32_t)kloc) {
          st_relaxed_gpu(tix, 0u);
          const int slot = atomicAdd(&sm.ncomb, 1);
          if (IDX_OK(p, slot < kTcMaxN)) sm.comb_rows[slot] = (int16_t)b;
        }
      }
      if (!epi_sync(sm, ephase, p, lane)) break;
      const int ncomb = sm.ncomb < kTcMaxN ? sm.ncomb : kTcMaxN;
      if (ncomb > 0) {
        // a shared-expert tile can complete a row before this CTA's schedule exists
        if (sched_layer < layer) {
          if (!warp_wait(&sm.sched_bar, (uint32_t)(layer & 1), p, lane)) break;
          sched_layer = layer;
        }
        combine_rows_tc<kEp>(p, sm, d.tile, sm.comb_rows, ncomb, et);
        if (p.rows_out) __threadfence();  // the rows' outputs, then their completion counts
        if (!epi_sync(sm, ephase, p, lane)) break;
        if (p.rows_out && et < ncomb) red_release_add(&p.rows_out[sm.comb_rows[et]], 1u);
        if (et == 0) sm.ncomb = 0;  // ordered before the next unit's list by its first rendezvous
      }
    } else {
      bool finished = direct || d.type == UT_ROUTER;
      if (!finished) {
        // split-K gate/up tile: count this split in, the last one does the fix-up
        __threadfence();
        if (!epi_sync(sm, ephase, p, lane)) break;
        if (et == 0) {
          const uint32_t old = atom_add_acq_rel(&p.tickets[d.ticket], 1u);
          const int last = old == (uint32_t)(d.nsplit - 1);
          if (last) st_relaxed_gpu(&p.tickets[d.ticket], 0u);
          sm.epi_last = last;
        }
        if (!epi_sync(sm, ephase, p, lane)) break;
        finished = sm.epi_last != 0;
        if (finished) fixup_tc(p, sm, d, et);
      }
      if (finished) {
        fence_proxy_async_global();
        __threadfence();
        if (!epi_sync(sm, ephase, p, lane)) break;
        if (et == 0) red_release_add(done_counter(p, d), 1u);
      }
    }
    c_busy += (unsigned long long)(tclock<kTrace>() - tb0);
  }
}

// ---- the kernel ----------------------------------------------------------------------------------

template <bool kTrace, bool kTC, bool kFp8 = false, bool kEp = false>
__global__ void __launch_bounds__(kTC ? kTcThreads : kThreads, 1)
    moe_decode_layer_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(ring + (kTC ? kTcRingBytes : kCcRingBytes));
  constexpr int kNst = kTC ? kTcStagesMax : kStages;  // barriers initialised (the TC ring uses sh.nst)
  const int tid = threadIdx.x;
  const int warp_id = tid / 32;
  const int lane = tid % 32;

  if (tid == 0) {
    for (int s = 0; s < kNst; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kTC ? 1 : kMacWarps);
    }
    if constexpr (kTC) {
      for (int b = 0; b < kTcAccBufs; ++b) {
        mbar_init(&sm.acc_full[b], 2);
        mbar_init(&sm.acc_empty[b], kTcEpiWarps);
      }
      mbar_init(&sm.mma_bar, 1);
      mbar_init(&sm.epi_bar, kTcEpiWarps);
      for (int s = 0; s < kTcStagesMax; ++s) {
        mbar_init(&sm.conv_bar[s], kMacWarps);
        mbar_init(&sm.wfull[s], 1);
        mbar_init(&sm.cdone[s], kMacWarps);
      }
      for (int a = 0; a < kFp8AStagesMax; ++a) mbar_init(&astage_empty(sm)[a], 1);
      for (int q = 0; q < kCq; ++q) {
        mbar_init(&sm.cq_full[q], 1);
        mbar_init(&sm.cq_empty[q], kMacWarps);  // every converter warp reads every entry
      }
      make_shape_tc(p, sm.sh);
    } else {
      for (int b = 0; b < kRB; ++b) {
        mbar_init(&sm.rb_full[b], kMacWarps);
        mbar_init(&sm.rb_empty[b], 1);
      }
      make_shape(p, sm.sh);
    }
    mbar_init(&sm.sched_bar, 1);
    mbar_init(&sm.mac_bar, kMacWarps);
    sm.ncomb = 0;
    for (int w = 0; w < kMaxSlots / 32; ++w) sm.known_done[w] = 0u;
    if (kTrace) {
      for (int t = 0; t < kTraceSlots; ++t) p.trace[(size_t)blockIdx.x * kTraceSlots + t] = 0ull;
      trace_stamp<kTrace>(p, TR_START);
      trace_clk<kTrace>(p, TR_START_CLK);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if constexpr (kTC) {
    if (warp_id == kTcMmaWarp) {
      tmem_alloc(&sm.tmem_base, kTmemCols);
      tmem_relinquish();
    }
    tc_fence_before();
  }
  __syncthreads();
  if constexpr (kTC) tc_fence_after();
  if (tid == 0) trace_stamp<kTrace>(p, TR_ROLES);
  uint8_t* const aring = ring;                            // FP8: the A stages' activations
  if constexpr (kFp8) ring += fp8_actbuf_bytes(sm.sh.NA);  // FP8: the slots follow them

  if (warp_id == 0) {
    Producer pr(p, sm, lane, sm.sh.nst);
    if constexpr (kTC) producer_tc<kTrace, kFp8, kEp>(pr, ring);
    else producer_cc<kTrace>(pr, ring);
  } else if (warp_id <= kMacWarps) {
    if constexpr (kTC) {
      // RMSNorm of this CTA's rows, then the routing schedule (the MMA and epilogue
      // warps keep the router and shared-expert tiles moving meanwhile)
      const int mw = warp_id - 1;
      uint32_t mphase = 0;
      const uint32_t tag = choice_tag(p);
      bool ok = normalise_rows<kTrace>(p, sm, mw, lane, mphase);
      if (ok) ok = route_rows_tc<kTrace>(p, sm, mw, lane, mphase, tag);
      if (ok && (int)blockIdx.x >= p.B && p.B > 1) {
        // a CTA that owns no row warms the schedule code (a short dry pass) in the gap
        // between the router units finishing and the rows' choices being published
        if (mw == 0) {
          int r = 1;
          if (lane == 0) r = wait_counter(&p.ctr[CTR_ROUTER], (uint32_t)sm.sh.router_target, p) ? 1 : 0;
          r = __shfl_sync(0xffffffffu, r, 0);
          if (lane == 0) sm.bcast = r;
        }
        ok = mac_sync(sm, mphase, p, lane) && sm.bcast;
        if (ok) ok = build_schedule_tc<kTrace, kEp>(p, sm, mw, lane, mphase, true);
      }
      if (ok) ok = p.B == 1 ? build_schedule_b1<kTrace, kEp>(p, sm, mw, lane, mphase, tag)
                            : build_schedule_tc<kTrace, kEp>(p, sm, mw, lane, mphase, false);
      if (mw == 0 && lane == 0 && ok) mbar_arrive(&sm.sched_bar);
      if constexpr (kFp8) convert_fp8_stages<kTrace>(p, sm, ring, aring, mw, lane, ok);
    } else {
      mac_warps_cc<kTrace>(p, sm, ring, warp_id - 1, lane);
    }
  } else if constexpr (!kTC) {
    epilogue_cc<kTrace>(p, sm, lane);
  } else if (warp_id == kTcMmaWarp) {
    mma_warp<kTrace, kFp8>(p, sm, ring, lane, aring);
  } else {
    epilogue_tc<kTrace, kFp8, kEp>(p, sm, warp_id, lane);
  }

  if constexpr (kTC) tc_fence_before();
  __syncthreads();
  if constexpr (kTC) {
    if (warp_id == kTcMmaWarp) {
      tc_fence_after();
      tmem_dealloc(sm.tmem_base, kTmemCols);
    }
  }
  if (tid == 0) {
    trace_stamp<kTrace>(p, TR_EXIT);
    __threadfence();
    const uint32_t done = atom_add_acq_rel(&p.gctr[CTR_EXIT], 1u);
    if (done == gridDim.x - 1) {
      // last CTA out: reset this step's counters for the next launch
      const bool aborted = ld_relaxed_gpu(&p.gctr[CTR_ABORT]) != 0u;
      if (aborted) {
        for (unsigned t = 0; t < p.max_tiles; ++t) p.tickets[t] = 0u;
        for (int t = 0; t < kMaxSlots; ++t) p.pair_done[t] = 0u;
        for (unsigned t = 0; t < p.row_tix_count; ++t) p.row_tix[t] = 0u;
      } else {
        for (int t = 0; t < sm.sc.P; ++t) p.pair_done[t] = 0u;
      }
      for (int c = 0; c < CTR_COUNT; ++c)
        if (c != CTR_EPOCH) p.ctr[c] = 0u;
      p.ctr[CTR_EPOCH] += 1u;  // the next launch's choices carry a new tag
      __threadfence();
    }
  }
}

// ---- several layers in one launch (tensor-core path) ---------------------------------------------
//
// Layer l + 1 follows layer l inside the same persistent launch: a CTA whose producer
// has drawn the last of layer l's units moves on to layer l + 1's queue (its router and
// shared-expert tiles arm their weight stages while layer l drains); each output row of
// layer l counts its
// combined tile pairs, and the CTA that owns row b normalises it for layer l + 1 once all
// have arrived. Every layer keeps its own counters, completion flags and choice tags;
// the activation buffers are shared, since a layer writes them only after the previous
// layer's output is complete everywhere, which means no unit of that layer is left.
// The per-layer kernel count of the pages' decode path (page post.smzdm.com/p/a6zppe4g,
// section "改了什么：每层 23 个 kernel 砍到 13 个") becomes one launch per step.
template <bool kTrace>
__global__ void __launch_bounds__(kTcThreads, 1) moe_decode_fused_kernel(const __grid_constant__ FusedParams F) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~uintptr_t(1023));
  Smem& sm = *reinterpret_cast<Smem*>(ring + kTcRingBytes);
  const Params& p0 = F.layer[0];
  const int L = F.L;
  const int tid = threadIdx.x;
  const int warp_id = tid / 32;
  const int lane = tid % 32;

  if (tid == 0) {
    for (int s = 0; s < kTcStagesMax; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < kTcAccBufs; ++b) {
      mbar_init(&sm.acc_full[b], 2);
      mbar_init(&sm.acc_empty[b], kTcEpiWarps);
    }
    mbar_init(&sm.mma_bar, 1);
    mbar_init(&sm.epi_bar, kTcEpiWarps);
    make_shape_tc(p0, sm.sh);  // every layer of the stack has the same shape
    mbar_init(&sm.sched_bar, 1);  // one phase per layer
    mbar_init(&sm.mac_bar, kMacWarps);
    sm.ncomb = 0;
    for (int w = 0; w < kMaxSlots / 32; ++w) sm.known_done[w] = 0u;
    if (kTrace) {
      for (int l = 0; l < L; ++l)
        for (int t = 0; t < kTraceSlots; ++t) F.layer[l].trace[(size_t)blockIdx.x * kTraceSlots + t] = 0ull;
      trace_stamp<kTrace>(p0, TR_START);
      trace_clk<kTrace>(p0, TR_START_CLK);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp_id == kTcMmaWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) trace_stamp<kTrace>(p0, TR_ROLES);

  if (warp_id == 0) {
    RingState st{0, 0u, 0u, 0u};
    for (int l = 0; l < L; ++l) {
      Producer pr(F.layer[l], sm, lane, sm.sh.nst);
      pr.slot = st.slot;
      pr.phase = st.phase;
      pr.pend_mask = st.pend_mask;
      pr.pend_parity = st.pend_parity;
      const bool ok = producer_tc<kTrace>(pr, ring, l == L - 1);
      st = RingState{pr.slot, pr.phase, pr.pend_mask, pr.pend_parity};
      if (!ok) break;  // the stop header and the drain are done
    }
  } else if (warp_id <= kMacWarps) {
    const int mw = warp_id - 1;
    uint32_t mphase = 0;
    for (int l = 0; l < L; ++l) {
      const Params& p = F.layer[l];
      const uint32_t tag = choice_tag(p);
      bool ok = normalise_rows<kTrace>(p, sm, mw, lane, mphase);
      if (ok) ok = route_rows_tc<kTrace>(p, sm, mw, lane, mphase, tag);
      if (ok && (int)blockIdx.x >= p.B && p.B > 1) {
        if (mw == 0) {
          int r = 1;
          if (lane == 0) r = wait_counter(&p.ctr[CTR_ROUTER], (uint32_t)sm.sh.router_target, p) ? 1 : 0;
          r = __shfl_sync(0xffffffffu, r, 0);
          if (lane == 0) sm.bcast = r;
        }
        ok = mac_sync(sm, mphase, p, lane) && sm.bcast;
        if (ok) ok = build_schedule_tc<kTrace>(p, sm, mw, lane, mphase, true);
      }
      if (ok) ok = p.B == 1 ? build_schedule_b1<kTrace>(p, sm, mw, lane, mphase, tag)
                            : build_schedule_tc<kTrace>(p, sm, mw, lane, mphase, false);
      if (mw == 0 && lane == 0 && ok) mbar_arrive(&sm.sched_bar);
      if (!ok) break;
    }
  } else if (warp_id == kTcMmaWarp) {
    mma_warp<kTrace>(p0, sm, ring, lane);
  } else {
    epilogue_tc<kTrace>(p0, sm, warp_id, lane, &F);
  }

  tc_fence_before();
  __syncthreads();
  if (warp_id == kTcMmaWarp) {
    tc_fence_after();
    tmem_dealloc(sm.tmem_base, kTmemCols);
  }
  if (tid == 0) {
    trace_stamp<kTrace>(p0, TR_EXIT);
    __threadfence();
    const uint32_t done = atom_add_acq_rel(&p0.gctr[CTR_EXIT], 1u);
    sm.bcast = done == gridDim.x - 1 ? 1 : 0;
  }
  __syncthreads();
  if (sm.bcast) {
    // last CTA out: every layer's counters, completion flags and row counts start at zero
    // for the next launch (and the shared tickets, which an aborted step may leave set)
    const bool aborted = ld_relaxed_gpu(&p0.gctr[CTR_ABORT]) != 0u;
    for (int l = 0; l < L; ++l) {
      const Params& p = F.layer[l];
      for (int t = tid; t < kMaxSlots; t += kTcThreads) p.pair_done[t] = 0u;
      if (p.rows_out)
        for (int t = tid; t < p.B; t += kTcThreads) p.rows_out[t] = 0u;
      if (tid < CTR_COUNT && !(l == 0 && tid == CTR_EPOCH)) p.ctr[tid] = 0u;
    }
    if (aborted) {
      for (unsigned t = tid; t < p0.max_tiles; t += kTcThreads) p0.tickets[t] = 0u;
      for (unsigned t = tid; t < p0.row_tix_count; t += kTcThreads) p0.row_tix[t] = 0u;
    }
    __syncthreads();
    if (tid == 0) {
      p0.gctr[CTR_EPOCH] += 1u;  // the next launch's choices carry new tags
      __threadfence();
    }
  }
}

size_t smem_bytes() { return kCcRingBytes + sizeof(Smem) + 1024; }
int threads_per_cta() { return kThreads; }
const void* kernel_fn() { return reinterpret_cast<const void*>(&moe_decode_layer_kernel<false, false>); }
const void* kernel_fn_trace() { return reinterpret_cast<const void*>(&moe_decode_layer_kernel<true, false>); }
size_t tc_smem_bytes() { return kTcRingBytes + sizeof(Smem) + 1024; }
int tc_threads_per_cta() { return kTcThreads; }
const void* tc_kernel_fn() { return reinterpret_cast<const void*>(&moe_decode_layer_kernel<false, true>); }
const void* tc_kernel_fn_trace() { return reinterpret_cast<const void*>(&moe_decode_layer_kernel<true, true>); }
int launch_partial_to_bf16(const float* in, uint16_t* out, long long n, int sms, cudaStream_t stream) {
  long long blocks = (n + 255) / 256;
  if (blocks > 4LL * sms) blocks = 4LL * sms;
  if (blocks < 1) blocks = 1;
  partial_to_bf16_kernel<<<(unsigned)blocks, 256, 0, stream>>>(in, out, n);
  return (int)cudaGetLastError();
}
const void* tc_ep_kernel_fn() { return reinterpret_cast<const void*>(&moe_decode_layer_kernel<false, true, false, true>); }
const void* tc_ep_kernel_fn_trace() {
  return reinterpret_cast<const void*>(&moe_decode_layer_kernel<true, true, false, true>);
}
const void* tc_fp8_kernel_fn() { return reinterpret_cast<const void*>(&moe_decode_layer_kernel<false, true, true>); }
const void* tc_fp8_kernel_fn_trace() {
  return reinterpret_cast<const void*>(&moe_decode_layer_kernel<true, true, true>);
}
const void* fused_kernel_fn() { return reinterpret_cast<const void*>(&moe_decode_fused_kernel<false>); }
const void* fused_kernel_fn_trace() { return reinterpret_cast<const void*>(&moe_decode_fused_kernel<true>); }

}  // namespace moe
