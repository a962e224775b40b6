/*
 * moe_decode.h - C ABI of the B200 (sm_100a) persistent MoE decode-layer step.
 *
 * One call of moe_decode_step runs one low-batch decode step (1..64 token rows)
 * of a sparse mixture-of-experts transformer layer as ONE persistent kernel
 * launch per layer: RMSNorm, router logits over all experts, top-k selection
 * with softmax renormalisation, a unique-expert schedule, the shared expert
 * (streamed while the routing resolves), the SwiGLU expert projections
 * (gate/up, SiLU * up, down) over only the selected experts, and the weighted
 * combine with the residual add.
 *
 * The method is the one the Kimi K3 decode pages describe: the per-layer chain
 * of kernels replaced by fused, persistent work (page "Kimi K3推理吞吐提升1.68倍",
 * section "为什么解码阶段适合Megakernel"); 896 experts with 16 active per token
 * (page "vLLM 合併 Kimi K3 專用解碼：官方稱 GB300 快 1.5 到 2 倍，423 tok/s 怎麼核對",
 * section "Kimi K3 專用解碼路徑改了什麼"); a batch-shape switch between small-matrix
 * and split-K kernels, router scores and the shared expert beside the routing (page
 * post.smzdm.com/p/a6zppe4g, section "改了什么：每层 23 个 kernel 砍到 13 个"). The
 * layer's arithmetic is:
 *
 *   n    = bf16(x * rsqrt(mean(x^2) + eps) * gamma)        (fp32)
 *   l[e] = n . W_r[e] (+ bias[e])                         (fp32 accumulate)
 *   S    = top-k of l, ties to the lower expert index;  w = softmax(l[S])
 *   h_e  = bf16(silu(W_g[e] n) * (W_u[e] n));  d_e = W_d[e] h_e
 *   s    = W_sd bf16(silu(W_sg n) * (W_su n))
 *   y    = bf16(x + s + sum_{e in S} w_e d_e)
 *
 * Conventions
 *  - All tensors are row-major. bf16 = IEEE bfloat16 bit patterns.
 *  - Device pointers are owned by the caller; the library never copies or
 *    repacks weights and must not outlive them. The library owns only its
 *    workspace (allocated by moe_decode_create, freed by moe_decode_destroy).
 *  - Every function returns 0 on success or a negative MOE_ERR_* code; nothing
 *    throws, exits or traps across this boundary.
 *  - moe_decode_step is asynchronous on the caller's stream and allocates
 *    nothing. Device-side failures (a bounded wait that ran out, a non-finite
 *    router logit) are recorded in a status word read by moe_decode_get_status
 *    after the stream has been synchronised.
 *  - A handle is not thread-safe: use it from one host thread and one stream at
 *    a time (steps on one handle must not overlap on the GPU).
 */
#ifndef MOE_DECODE_H
#define MOE_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_ERR_INVALID_ARG (-1)        /* null pointer, bad size, batch/top_k out of range */
#define MOE_ERR_UNSUPPORTED_ARCH (-2)   /* device is not sm_100 (B200) */
#define MOE_ERR_UNSUPPORTED_SHAPE (-3)  /* dimensions the kernel does not tile (see create) */
#define MOE_ERR_COOPERATIVE (-4)        /* cooperative launch unsupported or grid not co-resident */
#define MOE_ERR_CUDA (-5)               /* a CUDA runtime/driver call failed */
#define MOE_ERR_TIMEOUT (-6)            /* device status: a bounded wait ran out */
#define MOE_ERR_NONFINITE (-7)          /* device status: a router logit was NaN or infinite
                                           (the tensor-core kernel abandons the step: y undefined) */
#define MOE_ERR_NO_MEMORY (-8)          /* workspace allocation failed */
#define MOE_ERR_BOUNDS (-9)             /* device status, bounds-checked build only: an index
                                           derived from the routing schedule fell outside its
                                           buffer; the access was skipped and the step abandoned */

/* Kernel paths of a step (moe_decode_step_path). */
#define MOE_PATH_CUDA_CORE 0   /* CUDA-core GEMV units of 32 weight rows x 4 token rows */
#define MOE_PATH_TENSOR_CORE 1 /* tcgen05 tiles of 128 weight rows x all token rows, TMEM accumulators */

/* Layer dimensions, fixed at create time.
 *  hidden        H   (multiple of 32; multiple of 256 or at most 256; at most 16384)
 *  n_experts     E   (multiple of 32, at most 1024)
 *  top_k_max     largest k a step may use (1..32, <= E)
 *  inter         I   expert SwiGLU intermediate (multiple of 32; multiple of 256 or <= 256)
 *  shared_inter  Is  shared-expert intermediate (same rule as inter)
 *  max_batch     largest number of token rows per step (1..64)
 *  n_layers      layers run back-to-back by one step (1..8); layer l+1's input is
 *                layer l's output. On the tensor-core path all layers run in ONE
 *                persistent launch: CTAs that run out of layer l's work arm layer
 *                l+1's first weight tiles, and each row of layer l+1 is normalised as
 *                soon as all of its layer-l outputs exist
 *  eps           RMSNorm epsilon */
typedef struct {
  int hidden;
  int n_experts;
  int top_k_max;
  int inter;
  int shared_inter;
  int max_batch;
  int n_layers;
  float eps;
} moe_decode_config;

/* Device pointers of one layer's parameters (bf16 unless noted). All must be
 * 16-byte aligned (router_bias: 4-byte aligned). */
typedef struct {
  const void* gamma;        /* [H] RMSNorm gain */
  const void* w_router;     /* [E][H] */
  const float* router_bias; /* fp32 [E], or NULL for no bias */
  const void* w_gate;       /* [E][I][H] */
  const void* w_up;         /* [E][I][H] */
  const void* w_down;       /* [E][H][I] */
  const void* ws_gate;      /* [Is][H] */
  const void* ws_up;        /* [Is][H] */
  const void* ws_down;      /* [H][Is] */
} moe_decode_layer_weights;

/* Device pointers of one layer whose routed experts are stored in FP8: E4M3 codes
 * (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; largest finite 448) with one
 * power-of-two fp32 scale per 128 x 128 block of each expert matrix. A weight is
 * value(code) * scale of its block, which must be exactly a bf16 value: the layer is
 * then the bf16 layer on those weights. Every scale must be a power of two (either
 * sign) in [2^-117, 2^7], the range in which the kernel's in-register decode is exact;
 * moe_decode_create_fp8 reads the scales once and refuses any other value with
 * MOE_ERR_INVALID_ARG. Router and shared expert stay bf16. All
 * pointers 16-byte aligned (router_bias and the scales 4-byte aligned).
 * (A more aggressive quantisation format is named on page "Kimi K3推理吞吐提升1.68倍",
 * intro, only as what the reported gain did not need; the format here is this
 * library's reading.) */
typedef struct {
  const void* gamma;          /* bf16 [H] */
  const void* w_router;       /* bf16 [E][H] */
  const float* router_bias;   /* fp32 [E] or NULL */
  const uint8_t* w_gate;      /* E4M3 [E][I][H] */
  const float* w_gate_scale;  /* fp32 [E][I/128][H/128] */
  const uint8_t* w_up;        /* E4M3 [E][I][H] */
  const float* w_up_scale;    /* fp32 [E][I/128][H/128] */
  const uint8_t* w_down;      /* E4M3 [E][H][I] */
  const float* w_down_scale;  /* fp32 [E][H/128][I/128] */
  const void* ws_gate;        /* bf16 [Is][H] */
  const void* ws_up;          /* bf16 [Is][H] */
  const void* ws_down;        /* bf16 [H][Is] */
} moe_decode_layer_weights_fp8;

/* Optional per-layer debug outputs of a step (device pointers; any may be NULL). */
typedef struct {
  float* logits;      /* fp32 [B][E]: router logits (bias included) */
  int32_t* topk_idx;  /* int32 [B][k]: selected experts, descending logit, ties to lower index */
  float* topk_w;      /* fp32 [B][k]: softmax weights of the selected experts */
  int32_t* n_unique;  /* int32 [1]: number of distinct experts selected by the batch */
} moe_decode_debug;

typedef struct moe_decode_handle moe_decode_handle;

/* Checks the device (sm_100, cooperative launch, one 1-CTA-per-SM persistent
 * grid), validates the shapes, records the caller's weight pointers for
 * cfg->n_layers layers (array `layers`), builds the TMA descriptors of every
 * weight matrix and allocates the workspace on `device`. On success *out holds
 * a handle owned by the caller (free it with moe_decode_destroy). */
int moe_decode_create(const moe_decode_config* cfg, const moe_decode_layer_weights* layers,
                      int device, moe_decode_handle** out);

/* moe_decode_create for layers with FP8 expert weights (moe_decode_layer_weights_fp8).
 * Every dimension must be a multiple of 128 (MOE_ERR_UNSUPPORTED_SHAPE otherwise):
 * steps of such a handle always take the tensor-core path, one launch per layer, and
 * the expert tiles stream as E4M3 codes (half the bytes of bf16), turned into the bf16
 * MMA operand in shared memory by the CTA's routing warps once the routing is done.
 * Copies the scale arrays to the host once to check them (synchronous on `device`):
 * MOE_ERR_INVALID_ARG for a scale outside the range above or a scale pointer that is
 * not 4-byte aligned, MOE_ERR_CUDA if the copy fails. */
int moe_decode_create_fp8(const moe_decode_config* cfg, const moe_decode_layer_weights_fp8* layers, int device,
                          moe_decode_handle** out);

/* Expert parallelism (one layer): a handle for the experts expert_begin <= e <
 * expert_end of a layer whose routed experts are split over several GPUs, router and
 * shared expert replicated on each (the pages spread the expert work over the GPUs and
 * fold the cross-GPU exchange into the computation: page post.smzdm.com/p/a6zppe4g,
 * section "改了什么：每层 23 个 kernel 砍到 13 个", items "把通信缝进计算" and "MoE
 * 去重"). layers[0] holds the full router (E rows) and shared expert, but w_gate,
 * w_up and w_down hold only this range's experts: [expert_end - expert_begin][I][H]
 * and [..][H][I], local expert i being expert expert_begin + i. cfg->n_layers must
 * be 1 and every dimension a multiple of 128 (the tensor-core kernel; otherwise
 * MOE_ERR_UNSUPPORTED_SHAPE). Steps of the handle go through
 * moe_decode_step_partial. */
int moe_decode_create_ep(const moe_decode_config* cfg, const moe_decode_layer_weights* layers, int device,
                         int expert_begin, int expert_end, moe_decode_handle** out);

/* The partial output of a one-layer step over the handle's experts:
 * y_partial[b] = sum over row b's top-k choices j whose expert the handle covers of
 * w_j E_j(n_b), plus x_b + s_b (the residual and the shared expert) when
 * add_residual_shared is nonzero -- exactly one rank sets it. Every row is written.
 * y_partial: device fp32 [batch][H], 16-byte aligned, owned by the caller. The sum of
 * the ranks' partials (an all-reduce) rounded by moe_decode_partial_to_bf16 is the
 * layer's output. Routing (logits, top-k, softmax) is computed in full on every rank.
 * Arguments as moe_decode_step; MOE_ERR_INVALID_ARG for a handle of several layers, an
 * FP8 handle, or one whose shapes the tensor-core kernel cannot run. A whole-layer
 * handle (moe_decode_create) gives the whole layer's output in fp32. */
int moe_decode_step_partial(moe_decode_handle* h, const void* x_in, float* y_partial, int batch, int top_k,
                            int add_residual_shared, void* stream, const moe_decode_debug* dbg);

/* y_out[i] = bf16(y_partial[i]) (round to nearest even) for i < n, on `device`,
 * asynchronous on `stream`: the output of an expert-parallel step after the
 * all-reduce. Device pointers; y_out 2-byte aligned. */
int moe_decode_partial_to_bf16(const float* y_partial, void* y_out, long long n, int device, void* stream);

/* One decode step over all layers. x_in: device bf16 [batch][H]; y_out: device
 * bf16 [batch][H] (may not alias x_in). 1 <= batch <= max_batch, 1 <= top_k <=
 * top_k_max. stream: a cudaStream_t (NULL = legacy default stream). dbg: NULL or
 * an array of n_layers debug records. Launches one kernel for the whole layer stack
 * on the tensor-core path, one per layer on the CUDA-core path (see
 * moe_decode_step_path); returns MOE_ERR_* for argument errors and launch failures. */
int moe_decode_step(moe_decode_handle* h, const void* x_in, void* y_out, int batch, int top_k,
                    void* stream, const moe_decode_debug* dbg);

/* Same step on HOST buffers: copies x_host (bf16 [batch][H], preferably pinned)
 * to the device, runs the step and copies the result back into y_host, all
 * asynchronous on `stream` (synchronise before reading y_host). Uses staging
 * buffers inside the handle's workspace. */
int moe_decode_step_host(moe_decode_handle* h, const void* x_host, void* y_host, int batch,
                         int top_k, void* stream, const moe_decode_debug* dbg);

/* Reads and clears the device status word of the last completed steps (call
 * after synchronising the stream). *device_status receives MOE_OK or the
 * first device-side MOE_ERR_* recorded. The return value reports whether the
 * read itself succeeded. */
int moe_decode_get_status(moe_decode_handle* h, int* device_status);

/* Number of kernel launches one moe_decode_step of max_batch rows makes: 1 when that
 * step takes the tensor-core path (the whole layer stack in one launch), n_layers on
 * the CUDA-core path. */
int moe_decode_launches_per_step(const moe_decode_handle* h);

/* Sets debug behaviour of later steps (tests only): bit 0 = per-CTA random
 * __nanosleep jitter at unit boundaries; bit 1 = withhold the normalised-row
 * ready signal so that every waiting CTA's bounded wait runs out; bit 2 (honoured
 * by the bounds-checked build, libmoe_decode_checked.so, only) = point row 0's
 * first choice at the first slot row past the schedule (a row inside the
 * workspace), which that build's checks must report as MOE_ERR_BOUNDS. wait_ms is
 * the bound of every device-side wait (default 2000 ms). */
int moe_decode_set_debug(moe_decode_handle* h, unsigned flags, unsigned wait_ms);

/* Per-CTA timeline of later steps (profiling aid). trace: NULL to switch it off,
 * or a device buffer of n_layers * moe_decode_trace_slots(h) uint64 values,
 * 8-byte aligned, owned by the caller. Per layer and CTA, 48 slots: global-timer
 * stamps (ns) of the kernel start, normalised rows acquired, schedule seen, first
 * expert and first down stage issued, last stage issued, last stage consumed, last
 * epilogue, exit; then clock64 sums of the producer's waits for ring slots, for
 * published activations and for queue tickets, MAC warp 0's waits for stages and
 * for result buffers, the epilogue warp's busy time, the number of units, MAC
 * warp 0's arithmetic cycles and stage count, the producer's issue cycles and
 * stage count, MAC warp 0's schedule-building, reduction and total loop
 * cycles, the producer's unit-setup, schedule-wait and total loop cycles, and
 * stamps of the router tiles seen finished, of the schedule built, and of the
 * schedule's top-k, top-k rendezvous and unique-expert steps, of a
 * normalised row published by the CTA, and of the first top-k row's logits
 * loaded and selection done; on the tensor-core kernel also the owned row's
 * top-k chosen (34) and its cycle count (35), the unique experts placed (36),
 * the pairs sorted (37), and clock64 at the kernel start (38): there the
 * routing stamps (slots 26-30, 32-34, 36, 37) are clock64 values of the CTA's
 * SM, comparable with slot 38 of the same CTA only (slot 39 is reserved); then
 * global-timer stamps of the warp roles starting after the set-up rendezvous (40),
 * the producer's first weight tile issued (41), and, on the CTA that owns the
 * first row it normalises, that row's squares summed (42), its sum known to every
 * routing warp (43) and its normalised values stored (44); slots 45-47 are reserved.
 * Traced steps run a separate instance of the kernel whose stamps are global stores
 * on the routing chain: a traced batch-1 step takes several microseconds longer
 * than an untraced one, so the stamps bound the time of each hop from above and
 * step times are compared on untraced steps. */
int moe_decode_set_trace(moe_decode_handle* h, void* trace);

/* uint64 trace slots of one layer (number of CTAs x 48). */
int moe_decode_trace_slots(const moe_decode_handle* h);

/* The batch-shape switch (page post.smzdm.com/p/a6zppe4g, section "改了什么：每层
 * 23 个 kernel 砍到 13 个": small-matrix and split-K kernels chosen by the batch
 * shape). Steps whose batch is at least min_batch run the tensor-core kernel:
 * every weight tile is 128 rows (M) and all token rows of the batch, or all slot
 * rows of one expert, are the MMA's N columns (rounded up to 16), so each selected
 * expert's weights stream once however many rows chose it, and the products
 * accumulate in tensor memory. Smaller batches run the CUDA-core kernel (fp32 FMA
 * GEMV over 4 token rows at a time). min_batch = 0 keeps every step on the
 * CUDA-core kernel. The tensor-core kernel needs hidden, inter, shared_inter and
 * n_experts to be multiples of 128 and max_batch <= 64; for other shapes every
 * step takes the CUDA-core kernel whatever min_batch says. Default min_batch: 1
 * (the tensor-core kernel measured faster at every batch size, batch 1 included).
 * Returns MOE_ERR_INVALID_ARG for a null handle or a negative min_batch. */
int moe_decode_set_tc_min_batch(moe_decode_handle* h, int min_batch);

/* The path a step of `batch` rows takes on this handle: MOE_PATH_CUDA_CORE or
 * MOE_PATH_TENSOR_CORE (MOE_ERR_INVALID_ARG for a null handle or a batch outside
 * 1..max_batch). */
int moe_decode_step_path(const moe_decode_handle* h, int batch);

/* The same decode step for callers that cannot allocate device memory: code on a
 * path where cudaMalloc is not allowed (inside a framework or plugin that owns
 * all device memory, an allocator callback, a process whose memory budget is
 * fixed up front). It takes no handle and allocates nothing; its scratch is one
 * device array of about 16.7 MB inside this library, which every GPU that loads
 * the library holds until the process exits. The pages have no counterpart to
 * this entry point.
 *  - Limits: batch <= 4, top_k <= 16, hidden <= 7168, n_experts <= 1024, inter <=
 *    1024, shared_inter <= 2048, n_layers <= 2 (cfg->max_batch and top_k_max are
 *    not used); beyond them it returns MOE_ERR_UNSUPPORTED_SHAPE.
 *  - cfg, layers, x_in, y_out, batch, top_k and stream mean what they mean for
 *    moe_decode_create and moe_decode_step; the TMA descriptors are built on
 *    every call and handed to the GPU by value in a kernel launch's parameters
 *    (no host buffer is read after the call returns).
 *  - The first call on a device (the current device) sets up that device: it
 *    looks up the scratch array's device address and the kernel's attributes.
 *  - All calls share the one array and each call clears its counters before it
 *    runs: calls that overlap on the GPU (other streams, other threads) race and
 *    must be serialised by the caller.
 *  - device_status (required; NULL is MOE_ERR_INVALID_ARG): a caller-zeroed,
 *    4-byte aligned device int into which the kernel records the first
 *    device-side MOE_ERR_* of the step (a wait that ran out, a non-finite router
 *    logit; read it after a sync). It is the only place such a failure shows:
 *    the return value covers argument and launch errors only. */
int moe_decode_step_noalloc(const moe_decode_config* cfg, const moe_decode_layer_weights* layers,
                            const void* x_in, void* y_out, int batch, int top_k, void* stream,
                            int* device_status);

void moe_decode_destroy(moe_decode_handle* h);

const char* moe_decode_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* MOE_DECODE_H */
