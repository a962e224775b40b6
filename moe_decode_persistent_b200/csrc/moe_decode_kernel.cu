// moe_decode_kernel.cu - the persistent sm_100a kernel of one MoE decode-layer step.
//
// One launch per layer, one CTA per SM (cooperative launch, all CTAs
// co-resident). The pages this follows replace a chain of per-layer kernels by
// one persistent kernel that keeps the GPU streaming (page "Kimi K3推理吞吐提升
// 1.68倍", section "为什么解码阶段适合Megakernel"; page post.smzdm.com/p/a6zppe4g,
// section "改了什么：每层 23 个 kernel 砍到 13 个": 23 -> 13 kernels per layer).
//
// Roles inside a CTA
//   warp 0           producer: takes units of work from a global queue and streams
//                    their weight tiles (2-D TMA boxes of 32 rows x up to 256 K
//                    columns) plus the matching activation rows (1-D bulk copies)
//                    into a kStages-deep shared-memory ring, mbarrier-completed.
//   warps 1..8       consumers: CUDA-core GEMV over each stage (each warp owns 4
//                    weight rows of the box, each lane 8 K columns), fp32
//                    accumulation in registers across the stages of a unit, warp
//                    shuffle reductions, split-K partials and last-arriver fixups.
//
// Units of work (queue order)
//   router    (act group g, tile of 32 experts, K split)      -> logits
//   shared    (act group g, tile of 32 rows of Ws_gate/Ws_up, K split) -> h_s
//   -- every CTA then builds the same routing schedule from the final logits:
//      warp-level top-k per row, softmax over the selected logits, the
//      expert -> rows map and the list of unique experts (each selected expert's
//      weights are streamed once per step however many rows chose it).
//   expert    ((expert, row group) pair, tile of 32 rows of W_gate/W_up, K split) -> h_e
//   down      (tile of 32 output features; split = one shared row group, or up to
//              two (expert, row group) pairs) -> y, combined by the tile's last split
// The shared expert's gate/up units run while the router resolves (page
// post.smzdm.com/p/a6zppe4g, same section: the shared expert moved beside the
// router computation). The next layer's router and shared weights are
// prefetched into L2 by CTAs that run out of work (same section, the last item).
//
// Memory ordering: data produced inside the kernel (normalised rows, logits,
// h, partials) is read only after an acquire on the counter that publishes it,
// and never through the non-coherent path; only static weights are loaded
// ahead of a wait (the pages' review finding: page "vLLM 合併 Kimi K3 專用解碼…",
// section "AI 寫的 GPU 核心 vLLM 怎麼驗證正確"). Every spin-wait is bounded;
// when one runs out the kernel records MOE_ERR_TIMEOUT, all CTAs unwind, drain
// their bulk copies and exit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "kernel_params.h"
#include "moe_decode.h"
#include "ptx.cuh"

namespace moe {

constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = 32 * kConsumerWarps;
constexpr int kThreads = 32 + kConsumerThreads;
constexpr int kRowsPerWarp = kBoxRows / kConsumerWarps;      // 4
constexpr int kBoxBytesMax = kBoxRows * kBoxColsMax * 2;      // 16 KB
constexpr int kActBytesMax = kActGroup * kBoxColsMax * 2;     // 4 KB
constexpr int kSlotBytes = 2 * kBoxBytesMax + kActBytesMax;   // 36 KB
constexpr int kStages = 5;
constexpr int kKSplits = 4;
constexpr uint32_t kConsumerBar = 1;

enum UnitType { UT_ROUTER = 0, UT_SHARED = 1, UT_EXPERT = 2, UT_DOWN_SHARED = 3, UT_DOWN_EXPERT = 4 };
enum HeaderKind { HK_STAGE = 0, HK_SCHED = 1, HK_END = 2 };

struct StageHeader {
  int kind, unit, stage, pad;
};

// Layout constants of one step (identical in every CTA).
struct Shape {
  int B, k, GB;
  int boxH, boxI, boxIs, nkbH, nkbI, nkbIs;
  int RT, ST, IT, DT;
  int RS, SS, ES;
  int NR, NS;
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
};

struct Smem {
  uint8_t ring[kStages][kSlotBytes];
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t sched_bar;
  StageHeader hdr[kStages];
  int abort_flag[2];
  int bcast;
  float red_ss[kConsumerWarps];
  Shape sh;
  Sched sc;
  float red[2][kBoxRows][kActGroup];
  float fin[2][kBoxRows][kActGroup];
  int topk_idx[kMaxSlots];
  float topk_w[kMaxSlots];
  unsigned long long mask[kMaxE];
};

static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "shared memory budget of one CTA");
static_assert(kConsumerThreads / kBoxRows * 8 == 64, "down fixup covers 64 token rows");

struct UnitDesc {
  int type;
  int tile;      // tile within its type
  int ticket;    // global tile id
  int split, nsplit;
  int g;         // row group (router / shared / down-shared)
  int pair;      // expert: the pair; down-expert: first pair
  int npair;     // down-expert
  int kb0;       // first K box
  int nstages;
  int nbox;
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
  atomicExch(&p.ctr[CTR_ABORT], 1u);
}

__device__ __forceinline__ bool abort_seen(const Params& p) {
  return ld_relaxed_gpu(&p.ctr[CTR_ABORT]) != 0u;
}

// Bounded wait on an mbarrier phase (any thread).
__device__ bool wait_mbar(uint64_t* bar, uint32_t parity, const Params& p) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0u) {
      if (abort_seen(p)) return false;
      if (globaltimer_ns() - t0 > p.wait_ns) {
        record_abort(p, MOE_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Bounded wait until *c >= target (acquire). Single thread.
__device__ bool wait_counter(const uint32_t* c, uint32_t target, const Params& p) {
  if (ld_acquire_gpu(c) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(64);
    if (ld_acquire_gpu(c) >= target) return true;
    if (abort_seen(p)) return false;
    if (globaltimer_ns() - t0 > p.wait_ns) {
      record_abort(p, MOE_ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ uint32_t hash32(uint32_t a) {
  a ^= a >> 16;
  a *= 0x7feb352dU;
  a ^= a >> 15;
  a *= 0x846ca68bU;
  a ^= a >> 16;
  return a;
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
  if (u < sh.NR) {
    d.type = UT_ROUTER;
    d.split = u % sh.RS;
    d.tile = (u / sh.RS) % sh.RT;
    d.g = u / (sh.RS * sh.RT);
    d.nsplit = sh.RS;
    d.ticket = d.g * sh.RT + d.tile;
    split_range(sh.nkbH, sh.RS, d.split, d.kb0, d.nstages);
    d.nbox = 1;
  } else if (u < sh.NR + sh.NS) {
    const int v = u - sh.NR;
    d.type = UT_SHARED;
    d.split = v % sh.SS;
    d.tile = (v / sh.SS) % sh.ST;
    d.g = v / (sh.SS * sh.ST);
    d.nsplit = sh.SS;
    d.ticket = sh.GB * sh.RT + d.g * sh.ST + d.tile;
    split_range(sh.nkbH, sh.SS, d.split, d.kb0, d.nstages);
    d.nbox = 2;
  } else if (u < sh.NR + sh.NS + sc.NE) {
    const int v = u - sh.NR - sh.NS;
    d.type = UT_EXPERT;
    d.split = v % sh.ES;
    d.tile = (v / sh.ES) % sh.IT;
    d.pair = v / (sh.ES * sh.IT);
    d.nsplit = sh.ES;
    d.ticket = sh.GB * (sh.RT + sh.ST) + d.pair * sh.IT + d.tile;
    split_range(sh.nkbH, sh.ES, d.split, d.kb0, d.nstages);
    d.nbox = 2;
  } else {
    const int v = u - sh.NR - sh.NS - sc.NE;
    d.tile = v % sh.DT;
    d.split = v / sh.DT;
    d.nsplit = sc.down_splits;
    d.ticket = sh.GB * (sh.RT + sh.ST) + sc.P * sh.IT + d.tile;
    d.kb0 = 0;
    d.nbox = 1;
    if (d.split < sh.GB) {
      d.type = UT_DOWN_SHARED;
      d.g = d.split;
      d.nstages = sh.nkbIs;
    } else {
      d.type = UT_DOWN_EXPERT;
      d.pair = (d.split - sh.GB) * kDownPairsPerSplit;
      d.npair = sc.P - d.pair < kDownPairsPerSplit ? sc.P - d.pair : kDownPairsPerSplit;
      d.nstages = d.npair * sh.nkbI;
    }
  }
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

// Per-stage geometry shared by producer and consumers.
struct StageDesc {
  int box_cols;  // K columns of the boxes of this stage
  int c;         // activation rows
  int pair;      // down-expert: the pair of this stage
  int q;         // down-expert: index of the pair within the unit
  int kb;        // K box index
};

__device__ __forceinline__ StageDesc stage_desc(const Shape& sh, const Sched& sc, const UnitDesc& d,
                                                int st) {
  StageDesc s;
  s.pair = d.pair;
  s.q = 0;
  switch (d.type) {
    case UT_ROUTER:
    case UT_SHARED:
      s.box_cols = sh.boxH;
      s.c = group_rows(sh.B, d.g);
      s.kb = d.kb0 + st;
      break;
    case UT_EXPERT:
      s.box_cols = sh.boxH;
      s.c = pair_rows(sc, d.pair);
      s.kb = d.kb0 + st;
      break;
    case UT_DOWN_SHARED:
      s.box_cols = sh.boxIs;
      s.c = group_rows(sh.B, d.g);
      s.kb = st;
      break;
    default:
      s.q = st / sh.nkbI;
      s.pair = d.pair + s.q;
      s.box_cols = sh.boxI;
      s.c = pair_rows(sc, s.pair);
      s.kb = st % sh.nkbI;
      break;
  }
  return s;
}

// ---- consumer math -----------------------------------------------------------------------------

template <int NBOX, int CP>
__device__ __forceinline__ void mac_stage(const uint8_t* slot, int box_cols, int c,
                                          float (&acc)[2][kRowsPerWarp][kActGroup], int warp,
                                          int lane) {
  const int row_bytes = box_cols * 2;
  const int colb = lane * 16;
  if (colb >= row_bytes) return;
  const uint8_t* act = slot + 2 * kBoxBytesMax;
  float a[CP][8];
#pragma unroll
  for (int j = 0; j < CP; ++j) {
    if (j < c) {
      const uint4 v = *reinterpret_cast<const uint4*>(act + j * row_bytes + colb);
      unpack8(v, a[j]);
    } else {
#pragma unroll
      for (int t = 0; t < 8; ++t) a[j][t] = 0.0f;
    }
  }
#pragma unroll
  for (int m = 0; m < NBOX; ++m) {
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
      const uint4 wv = *reinterpret_cast<const uint4*>(slot + m * kBoxBytesMax +
                                                       (warp + kConsumerWarps * r) * row_bytes + colb);
      float w[8];
      unpack8(wv, w);
#pragma unroll
      for (int j = 0; j < CP; ++j) {
#pragma unroll
        for (int t = 0; t < 8; ++t) acc[m][r][j] = fmaf(w[t], a[j][t], acc[m][r][j]);
      }
    }
  }
}

__device__ __forceinline__ void mac_dispatch(const uint8_t* slot, int nbox, int box_cols, int c,
                                             float (&acc)[2][kRowsPerWarp][kActGroup], int warp,
                                             int lane) {
  if (nbox == 1) {
    if (c <= 1) mac_stage<1, 1>(slot, box_cols, c, acc, warp, lane);
    else if (c <= 2) mac_stage<1, 2>(slot, box_cols, c, acc, warp, lane);
    else mac_stage<1, kActGroup>(slot, box_cols, c, acc, warp, lane);
  } else {
    if (c <= 1) mac_stage<2, 1>(slot, box_cols, c, acc, warp, lane);
    else if (c <= 2) mac_stage<2, 2>(slot, box_cols, c, acc, warp, lane);
    else mac_stage<2, kActGroup>(slot, box_cols, c, acc, warp, lane);
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

// Warp-reduce the accumulators of boxes [0, nbox) into red[m0 + m][row][j] (lane 0 writes).
// `wscale` (nullable) multiplies column j (routing weight of the pair's row j).
__device__ __forceinline__ void reduce_acc(float (&acc)[2][kRowsPerWarp][kActGroup], int nbox,
                                           int c, float (*red)[kBoxRows][kActGroup], int m0,
                                           const float* wscale, int warp, int lane) {
#pragma unroll
  for (int m = 0; m < 2; ++m) {
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r) {
#pragma unroll
      for (int j = 0; j < kActGroup; ++j) {
        if (m >= nbox || j >= c) continue;  // warp-uniform
        float v = acc[m][r][j];
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if (lane == 0) red[m0 + m][warp + kConsumerWarps * r][j] = wscale ? v * wscale[j] : v;
      }
    }
  }
}

// ---- routing schedule (consumer warps, all CTAs) ---------------------------------------------

// Top-k of one row by one warp: the k largest logits, ties to the lower expert index,
// then softmax over the selected logits.
__device__ void warp_topk_row(const Params& p, Smem& sm, int b, int lane) {
  const int E = p.E, k = p.k;
  const int nq = E / 32;
  float v[kMaxE / 32];
  uint32_t taken = 0;
  bool bad = false;
#pragma unroll
  for (int q = 0; q < kMaxE / 32; ++q) {
    if (q < nq) {
      float t = ld_cg_f32(&p.logits[(size_t)b * E + lane + 32 * q]);
      if (!isfinite(t)) {
        bad = true;
        t = -INFINITY;
      }
      v[q] = t;
    } else {
      v[q] = -INFINITY;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) record_error(p, MOE_ERR_NONFINITE);
  int my_idx = 0;
  float my_val = 0.0f;
  for (int j = 0; j < k; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int q = 0; q < kMaxE / 32; ++q) {
      if (q < nq && !((taken >> q) & 1u)) {
        const int e = lane + 32 * q;
        if (bi == 0x7fffffff || v[q] > bv) {
          bv = v[q];
          bi = e;
        }
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (oi != 0x7fffffff && (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi))) {
        bv = ov;
        bi = oi;
      }
    }
    if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
    if (lane == j) {
      my_idx = bi;
      my_val = bv;
    }
  }
  const float mx = __shfl_sync(0xffffffffu, my_val, 0);
  const float ex = lane < k ? expf(my_val - mx) : 0.0f;
  float z = ex;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  if (lane < k) {
    sm.topk_idx[b * k + lane] = my_idx;
    sm.topk_w[b * k + lane] = ex / z;
    atomicOr(&sm.mask[my_idx], 1ull << b);
  }
}

// Builds sm.sc from the final logits. Called by all consumer threads; returns false on abort.
__device__ bool build_schedule(const Params& p, Smem& sm, int ctid, int warp, int lane) {
  const Shape& sh = sm.sh;
  Sched& sc = sm.sc;
  if (ctid == 0) {
    const bool ok = wait_counter(&p.ctr[CTR_ROUTER], (uint32_t)(sh.GB * sh.RT), p);
    sm.bcast = ok ? 1 : 0;
  }
  for (int e = ctid; e < p.E; e += kConsumerThreads) sm.mask[e] = 0ull;
  named_bar_sync(kConsumerBar, kConsumerThreads);
  if (!sm.bcast) return false;
  for (int b = warp; b < p.B; b += kConsumerWarps) warp_topk_row(p, sm, b, lane);
  named_bar_sync(kConsumerBar, kConsumerThreads);
  if (warp == 0) {
    // unique experts in ascending id; rows per expert
    int base = 0;
    for (int e0 = 0; e0 < p.E; e0 += 32) {
      const unsigned long long m = sm.mask[e0 + lane];
      const uint32_t bal = __ballot_sync(0xffffffffu, m != 0ull);
      const int pos = base + __popc(bal & ((1u << lane) - 1u));
      if (m != 0ull) {
        sc.slot_expert[pos] = (int16_t)(e0 + lane);
        sc.slot_cnt[pos] = (int16_t)__popcll(m);
      }
      base += __popc(bal);
    }
    const int U = base;
    // slot bases and (expert, row group) pairs
    int rbase = 0, pbase = 0;
    for (int i0 = 0; i0 < U; i0 += 32) {
      const int i = i0 + lane;
      const int c = i < U ? sc.slot_cnt[i] : 0;
      const int gcount = (c + kActGroup - 1) / kActGroup;
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
      sm.bcast = ((unsigned)sc.total <= p.max_units && tiles <= p.max_tiles) ? 1 : 0;
      if (!sm.bcast) record_abort(p, MOE_ERR_UNSUPPORTED_SHAPE);
    }
  }
  named_bar_sync(kConsumerBar, kConsumerThreads);
  if (!sm.bcast) return false;
  // token rows and routing weights of every slot row (rows ascending within an expert)
  for (int i = ctid; i < sc.U; i += kConsumerThreads) {
    const int e = sc.slot_expert[i];
    unsigned long long m = sm.mask[e];
    int r = sc.slot_base[i];
    while (m) {
      const int b = __ffsll((long long)m) - 1;
      m &= m - 1ull;
      float w = 0.0f;
      for (int j = 0; j < p.k; ++j)
        if (sm.topk_idx[b * p.k + j] == e) w = sm.topk_w[b * p.k + j];
      sc.row_of[r] = (uint8_t)b;
      sc.w_of[r] = w;
      ++r;
    }
  }
  if (blockIdx.x == 0) {
    for (int t = ctid; t < p.B * p.k; t += kConsumerThreads) {
      if (p.dbg_idx) p.dbg_idx[t] = sm.topk_idx[t];
      if (p.dbg_w) p.dbg_w[t] = sm.topk_w[t];
    }
    if (ctid == 0 && p.dbg_nuniq) *p.dbg_nuniq = sc.U;
  }
  named_bar_sync(kConsumerBar, kConsumerThreads);
  return true;
}

// ---- consumer: end of a unit --------------------------------------------------------------------

// Completion counter a finished tile of unit type `type` releases.
__device__ __forceinline__ uint32_t* done_counter(const Params& p, const UnitDesc& d) {
  switch (d.type) {
    case UT_ROUTER: return &p.ctr[CTR_ROUTER];
    case UT_SHARED: return &p.ctr[CTR_HS];
    case UT_EXPERT: return &p.pair_done[d.pair];
    default: return nullptr;
  }
}

__device__ void finish_unit(const Params& p, Smem& sm, const UnitDesc& d, int u, int ctid) {
  const Shape& sh = sm.sh;
  const Sched& sc = sm.sc;
  const bool down = d.type == UT_DOWN_SHARED || d.type == UT_DOWN_EXPERT;
  named_bar_sync(kConsumerBar, kConsumerThreads);  // sm.red complete
  float(*fin)[kBoxRows][kActGroup] = sm.red;
  if (d.nsplit > 1) {
    float* part = p.partial + (size_t)u * kPartialFloats;
    const float* red = &sm.red[0][0][0];
    for (int t = ctid; t < kPartialFloats; t += kConsumerThreads) part[t] = red[t];
    __threadfence();
    named_bar_sync(kConsumerBar, kConsumerThreads);
    if (ctid == 0) {
      const uint32_t old = atom_add_acq_rel(&p.tickets[d.ticket], 1u);
      const bool last = old == (uint32_t)(d.nsplit - 1);
      if (last) st_relaxed_gpu(&p.tickets[d.ticket], 0u);
      sm.bcast = last ? 1 : 0;
    }
    named_bar_sync(kConsumerBar, kConsumerThreads);
    if (!sm.bcast) return;
    __threadfence();
    if (!down) {
      // fixed split order -> deterministic sums
      for (int t = ctid; t < kPartialFloats; t += kConsumerThreads) {
        float s = 0.0f;
        for (int sp = 0; sp < d.nsplit; ++sp)
          s += ld_cg_f32(p.partial + (size_t)unit_of_split(sh, sc, d, sp) * kPartialFloats + t);
        (&sm.fin[0][0][0])[t] = s;
      }
      named_bar_sync(kConsumerBar, kConsumerThreads);
      fin = sm.fin;
    }
  }
  // ---- epilogues ----
  if (d.type == UT_ROUTER) {
    const int c = group_rows(sh.B, d.g);
    for (int t = ctid; t < kBoxRows * c; t += kConsumerThreads) {
      const int row = t / c, j = t % c;
      const int e = d.tile * kBoxRows + row;
      const int b = d.g * kActGroup + j;
      float v = fin[0][row][j];
      if (p.bias) v += p.bias[e];
      p.logits[(size_t)b * p.E + e] = v;
      if (p.dbg_logits) p.dbg_logits[(size_t)b * p.E + e] = v;
    }
  } else if (d.type == UT_SHARED || d.type == UT_EXPERT) {
    const int c = d.type == UT_SHARED ? group_rows(sh.B, d.g) : pair_rows(sc, d.pair);
    for (int t = ctid; t < kBoxRows * c; t += kConsumerThreads) {
      const int row = t / c, j = t % c;
      const float h = silu(fin[0][row][j]) * fin[1][row][j];
      if (d.type == UT_SHARED) {
        const int b = d.g * kActGroup + j;
        p.hs[(size_t)b * p.Is + d.tile * kBoxRows + row] = f2bf(h);
      } else {
        const int r = pair_first_slot_row(sc, d.pair) + j;
        p.he[(size_t)r * p.I + d.tile * kBoxRows + row] = f2bf(h);
      }
    }
  } else {
    // down tile fixup: y = bf16(x + s + sum_e w_e d_e), fixed split / pair / row order.
    // Thread (row, bg) owns output feature `row` of the tile for token rows b = bg (mod 8).
    constexpr int kRes = kConsumerThreads / kBoxRows;  // 8
    const int row = ctid / kRes, bg = ctid % kRes;
    float yacc[64 / kRes];
#pragma unroll
    for (int i = 0; i < 64 / kRes; ++i) yacc[i] = 0.0f;
    for (int sp = 0; sp < d.nsplit; ++sp) {
      const float* part =
          p.partial + (size_t)(sh.NR + sh.NS + sc.NE + sp * sh.DT + d.tile) * kPartialFloats;
      if (sp < sh.GB) {
        const int c = group_rows(sh.B, sp);
        for (int j = 0; j < c; ++j) {
          const int b = sp * kActGroup + j;
          if (b % kRes == bg) yacc[b / kRes] += ld_cg_f32(part + row * kActGroup + j);
        }
      } else {
        const int pr0 = (sp - sh.GB) * kDownPairsPerSplit;
        const int np = sc.P - pr0 < kDownPairsPerSplit ? sc.P - pr0 : kDownPairsPerSplit;
        for (int q = 0; q < np; ++q) {
          const int pr = pr0 + q;
          const int c = pair_rows(sc, pr);
          const int r0 = pair_first_slot_row(sc, pr);
          for (int j = 0; j < c; ++j) {
            const int b = sc.row_of[r0 + j];
            if (b % kRes == bg)
              yacc[b / kRes] += ld_cg_f32(part + q * kBoxRows * kActGroup + row * kActGroup + j);
          }
        }
      }
    }
    const int h = d.tile * kBoxRows + row;
#pragma unroll
    for (int i = 0; i < 64 / kRes; ++i) {
      const int b = i * kRes + bg;
      if (b < sh.B) {
        const float xv = bf2f(p.x[(size_t)b * p.H + h]);
        p.y[(size_t)b * p.H + h] = f2bf(xv + yacc[i]);
      }
    }
  }
  uint32_t* done = done_counter(p, d);
  if (done) {
    fence_proxy_async_global();
    __threadfence();
    named_bar_sync(kConsumerBar, kConsumerThreads);
    if (ctid == 0) red_release_add(done, 1u);
  }
}

// ---- RMSNorm of the rows this CTA publishes ---------------------------------------------------

__device__ void normalise_rows(const Params& p, Smem& sm, int ctid, int warp, int lane) {
  for (int b = blockIdx.x; b < p.B; b += gridDim.x) {
    const uint16_t* xb = p.x + (size_t)b * p.H;
    float ss = 0.0f;
    for (int h = ctid; h < p.H; h += kConsumerThreads) {
      const float v = bf2f(xb[h]);
      ss = fmaf(v, v, ss);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) sm.red_ss[warp] = ss;
    named_bar_sync(kConsumerBar, kConsumerThreads);
    float tot = 0.0f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += sm.red_ss[w];
    const float r = 1.0f / sqrtf(tot / (float)p.H + p.eps);
    for (int h = ctid; h < p.H; h += kConsumerThreads) {
      const float v = bf2f(xb[h]) * r * bf2f(p.gamma[h]);
      p.n[(size_t)b * p.H + h] = f2bf(v);
    }
    fence_proxy_async_global();
    __threadfence();
    named_bar_sync(kConsumerBar, kConsumerThreads);
    if (ctid == 0 && !((p.flags & kFlagWithholdNReady) && b == 0)) red_release_add(&p.ctr[CTR_NREADY], 1u);
  }
}

// ---- the kernel ----------------------------------------------------------------------------------

__global__ void __launch_bounds__(kThreads, 1) moe_decode_layer_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp_id = tid / 32;
  const int lane = tid % 32;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init(&sm.sched_bar, 1);
    make_shape(p, sm.sh);
    sm.abort_flag[0] = sm.abort_flag[1] = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const Shape& sh = sm.sh;

  if (warp_id == 0) {
    // =========================== producer warp ===========================
    const uint64_t pol = policy_evict_first();
    if (lane == 0)
      for (int t = 0; t < TM_COUNT; ++t) prefetch_tensormap(&p.tmaps[t]);
    int slot = 0;
    uint32_t phase = 0;
    int last_tx_parity[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) last_tx_parity[s] = -1;
    bool ok = true, sched_ready = false, n_ok = false, hs_ok = false;
    const int pre = sh.NR + sh.NS;
    auto grab = [&]() -> int {
      int v = 0;
      if (lane == 0) v = (int)atom_add_relaxed(&p.ctr[CTR_QUEUE], 1u);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    auto advance = [&]() {
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1u;
      }
    };
    auto wait_bar = [&](uint64_t* bar, uint32_t parity) -> bool {
      int r = 1;
      if (lane == 0) r = wait_mbar(bar, parity, p) ? 1 : 0;
      r = __shfl_sync(0xffffffffu, r, 0);
      __syncwarp();
      return r != 0;
    };
    auto wait_dep = [&](const uint32_t* c, uint32_t target) -> bool {
      int r = 1;
      if (lane == 0) {
        r = wait_counter(c, target, p) ? 1 : 0;
        fence_proxy_async_global();
      }
      return __shfl_sync(0xffffffffu, r, 0) != 0;
    };
    int u = grab();
    while (ok) {
      if (u >= pre && !sched_ready) {
        ok = wait_bar(&sm.empty[slot], phase ^ 1u);
        if (!ok) break;
        last_tx_parity[slot] = -1;  // the slot's previous stage was consumed
        if (lane == 0) {
          sm.hdr[slot].kind = HK_SCHED;
          mbar_arrive(&sm.full[slot]);
        }
        __syncwarp();
        advance();
        ok = wait_bar(&sm.sched_bar, 0u);
        if (!ok) break;
        sched_ready = true;
      }
      if (sched_ready && u >= sm.sc.total) break;
      const UnitDesc d = decode_unit(sh, sm.sc, u);
      const int next_u = grab();
      if ((p.flags & kFlagJitter) && lane == 0) __nanosleep(hash32(blockIdx.x * 7919u + (uint32_t)u) % 3000u);
      for (int st = 0; st < d.nstages && ok; ++st) {
        ok = wait_bar(&sm.empty[slot], phase ^ 1u);
        if (!ok) break;
        const StageDesc s = stage_desc(sh, sm.sc, d, st);
        const uint32_t box_bytes = (uint32_t)(s.box_cols * kBoxRows * 2);
        const uint32_t row_bytes = (uint32_t)(s.box_cols * 2);
        uint8_t* dst = sm.ring[slot];
        uint64_t* fb = &sm.full[slot];
        if (lane == 0) {
          sm.hdr[slot].kind = HK_STAGE;
          sm.hdr[slot].unit = u;
          sm.hdr[slot].stage = st;
          mbar_arrive_expect_tx(fb, (uint32_t)d.nbox * box_bytes + (uint32_t)s.c * row_bytes);
          last_tx_parity[slot] = (int)phase;
          const int x = s.kb * s.box_cols;
          switch (d.type) {
            case UT_ROUTER:
              tma_load_2d(dst, &p.tmaps[TM_WR], x, d.tile * kBoxRows, fb, pol);
              break;
            case UT_SHARED:
              tma_load_2d(dst, &p.tmaps[TM_WSG], x, d.tile * kBoxRows, fb, pol);
              tma_load_2d(dst + kBoxBytesMax, &p.tmaps[TM_WSU], x, d.tile * kBoxRows, fb, pol);
              break;
            case UT_EXPERT: {
              const int e = sm.sc.slot_expert[sm.sc.pair_slot[d.pair]];
              const int row = e * p.I + d.tile * kBoxRows;
              tma_load_2d(dst, &p.tmaps[TM_WG], x, row, fb, pol);
              tma_load_2d(dst + kBoxBytesMax, &p.tmaps[TM_WU], x, row, fb, pol);
              break;
            }
            case UT_DOWN_SHARED:
              tma_load_2d(dst, &p.tmaps[TM_WSD], x, d.tile * kBoxRows, fb, pol);
              break;
            default: {
              const int e = sm.sc.slot_expert[sm.sc.pair_slot[s.pair]];
              tma_load_2d(dst, &p.tmaps[TM_WD], x, e * p.H + d.tile * kBoxRows, fb, pol);
              break;
            }
          }
        }
        // activations: only after the acquire that publishes them
        bool dep_ok = true;
        if (d.type == UT_ROUTER || d.type == UT_SHARED || d.type == UT_EXPERT) {
          if (!n_ok) dep_ok = n_ok = wait_dep(&p.ctr[CTR_NREADY], (uint32_t)p.B);
        } else if (d.type == UT_DOWN_SHARED) {
          if (!hs_ok) dep_ok = hs_ok = wait_dep(&p.ctr[CTR_HS], (uint32_t)(sh.GB * sh.ST));
        } else if (st % sh.nkbI == 0) {
          dep_ok = wait_dep(&p.pair_done[s.pair], (uint32_t)sh.IT);
        }
        if (lane == 0) {
          uint8_t* act = dst + 2 * kBoxBytesMax;
          const int x = s.kb * s.box_cols;
          for (int j = 0; j < s.c; ++j) {
            const uint16_t* src;
            switch (d.type) {
              case UT_ROUTER:
              case UT_SHARED:
                src = p.n + (size_t)(d.g * kActGroup + j) * p.H + x;
                break;
              case UT_EXPERT:
                src = p.n + (size_t)sm.sc.row_of[pair_first_slot_row(sm.sc, d.pair) + j] * p.H + x;
                break;
              case UT_DOWN_SHARED:
                src = p.hs + (size_t)(d.g * kActGroup + j) * p.Is + x;
                break;
              default:
                src = p.he + (size_t)(pair_first_slot_row(sm.sc, s.pair) + j) * p.I + x;
                break;
            }
            bulk_load(act + j * row_bytes, src, row_bytes, fb);
          }
        }
        __syncwarp();
        advance();
        if (!dep_ok) ok = false;
      }
      u = next_u;
    }
    // tell the consumers to stop (bounded)
    if (wait_bar(&sm.empty[slot], phase ^ 1u)) {
      last_tx_parity[slot] = -1;
      if (lane == 0) {
        sm.hdr[slot].kind = HK_END;
        mbar_arrive(&sm.full[slot]);
      }
    }
    __syncwarp();
    // drain: every issued bulk copy must have landed before the CTA exits. A slot's
    // record is the phase of its last TMA stage that no later use of the slot has
    // shown to be complete (only possible after an abort).
    if (lane == 0) {
      for (int s = 0; s < kStages; ++s) {
        if (last_tx_parity[s] < 0) continue;
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&sm.full[s], (uint32_t)last_tx_parity[s])) {
          if (globaltimer_ns() - t0 > 50000000ull) break;
        }
      }
      // L2 prefetch of the next layer's router and shared-expert weights
      for (int r = 0; r < 4; ++r) {
        if (!p.pf_ptr[r] || !p.pf_bytes[r]) continue;
        const unsigned long long tot = p.pf_bytes[r];
        unsigned long long lo = (tot * blockIdx.x / gridDim.x) & ~15ull;
        unsigned long long hi = blockIdx.x + 1 == gridDim.x ? tot : (tot * (blockIdx.x + 1) / gridDim.x) & ~15ull;
        const uint8_t* base = reinterpret_cast<const uint8_t*>(p.pf_ptr[r]);
        for (unsigned long long o = lo; o < hi; o += 65536ull) {
          const unsigned long long n = hi - o < 65536ull ? hi - o : 65536ull;
          if (n >= 16) prefetch_l2_bulk(base + o, (uint32_t)(n & ~15ull));
        }
      }
    }
    __syncwarp();
  } else {
    // =========================== consumer warps ===========================
    const int cw = warp_id - 1;
    const int ctid = tid - 32;
    normalise_rows(p, sm, ctid, cw, lane);
    int slot = 0;
    uint32_t phase = 0;
    int cur_u = -1;
    UnitDesc d;
    d.type = UT_ROUTER;
    d.nstages = 0;
    float acc[2][kRowsPerWarp][kActGroup];
    zero_acc(acc);
    for (uint32_t it = 0;; ++it) {
      if (ctid == 0) sm.abort_flag[it & 1u] = wait_mbar(&sm.full[slot], phase, p) ? 0 : 1;
      named_bar_sync(kConsumerBar, kConsumerThreads);
      if (sm.abort_flag[it & 1u]) break;
      const StageHeader hd = sm.hdr[slot];
      if (hd.kind == HK_END) break;
      if (hd.kind == HK_SCHED) {
        const bool ok = build_schedule(p, sm, ctid, cw, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[slot]);
        if (ctid == 0 && ok) mbar_arrive(&sm.sched_bar);
        if (++slot == kStages) {
          slot = 0;
          phase ^= 1u;
        }
        if (!ok) break;
        continue;
      }
      if (hd.unit != cur_u) {
        cur_u = hd.unit;
        d = decode_unit(sh, sm.sc, cur_u);
        zero_acc(acc);
      }
      const StageDesc s = stage_desc(sh, sm.sc, d, hd.stage);
      mac_dispatch(sm.ring[slot], d.nbox, s.box_cols, s.c, acc, cw, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[slot]);
      if (++slot == kStages) {
        slot = 0;
        phase ^= 1u;
      }
      if (d.type == UT_DOWN_EXPERT) {
        if (hd.stage % sh.nkbI == sh.nkbI - 1) {
          const float* wsc = &sm.sc.w_of[pair_first_slot_row(sm.sc, s.pair)];
          reduce_acc(acc, 1, s.c, sm.red, s.q, wsc, cw, lane);
          zero_acc(acc);
        }
      } else if (hd.stage == d.nstages - 1) {
        reduce_acc(acc, d.nbox, s.c, sm.red, 0, nullptr, cw, lane);
      }
      if (hd.stage == d.nstages - 1) finish_unit(p, sm, d, cur_u, ctid);
    }
  }

  __syncthreads();
  if (tid == 0) {
    __threadfence();
    const uint32_t done = atom_add_acq_rel(&p.ctr[CTR_EXIT], 1u);
    if (done == gridDim.x - 1) {
      // last CTA out: reset this step's counters for the next launch
      const bool aborted = ld_relaxed_gpu(&p.ctr[CTR_ABORT]) != 0u;
      if (aborted) {
        for (unsigned t = 0; t < p.max_tiles; ++t) p.tickets[t] = 0u;
        for (int t = 0; t < kMaxSlots; ++t) p.pair_done[t] = 0u;
      } else {
        for (int t = 0; t < sm.sc.P; ++t) p.pair_done[t] = 0u;
      }
      for (int c = 0; c < CTR_COUNT; ++c) p.ctr[c] = 0u;
      __threadfence();
    }
  }
}

size_t smem_bytes() { return sizeof(Smem) + 1024; }
int threads_per_cta() { return kThreads; }
const void* kernel_fn() { return reinterpret_cast<const void*>(&moe_decode_layer_kernel); }

}  // namespace moe
