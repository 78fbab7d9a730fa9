/*
 * mono_ffn — one persistent launch per layer for the FFN half of a
 * DeepSeek-V4.1-style decoder layer at decode batch sizes (1-8 rows), on
 * NVIDIA B200 (sm_100a).
 *
 * What one step computes, per row r of hc_in [rows][S=4][H] (the layer as the
 * pages state it):
 *   1. mHC pre: rho = 1/sqrt(mean over the flattened 4H row of X^2 + eps);
 *      mix = rho * (X_flat @ mix_w) -> 24 values: pre = sigmoid + 1e-6 (4),
 *      post = 2 sigmoid (4), comb = 20-iteration Sinkhorn of exp over the
 *      4x4 logits (row-major (i, j) at column 8 + 4 i + j).
 *      (SGLang "[DeepSeek-V4] Add mhc_fused_post_pre kernel", Motivation:
 *      pre-norm GEMM partials + RMS square-sum partials, finalised together;
 *      ds4 "v41: fuse the single-box decode glue", HC fusion commit.)
 *   2. collapse a = sum_s pre_s X_s -> bf16; weighted RMSNorm
 *      n = a / sqrt(mean a^2 + eps) * norm_w -> bf16.  (ds4 page, HC fusion
 *      commit: the collapse weighted by pre and the weighted RMSNorm, each
 *      rounded to bf16.)
 *   3. router select: fp32 logits n @ router_w; score = sqrt(softplus);
 *      sel = score + bias (selection only); canonical top-k by (sel desc,
 *      index asc); weight = score / max(sum, clamp) * route_scale.  (ds4
 *      page, MoE fusion: "Mega-Gate" router select.)
 *   4. shared expert (slot E) and the k routed experts: g, u = n @ gate^T,
 *      n @ up^T -> bf16; act = silu(g) * u; d = act @ down^T.  (ds4 page,
 *      MoE fusion; vLLM "[ROCm][Perf][GLM-5] Fused sparse-layer decode via
 *      AITER MonoKernel", Weights: shared expert in the last slot.)
 *   5. y = bf16(sum_j w_j d_j + d_shared); out_i = bf16(sum_j comb_ij X_j +
 *      post_i y).  (ds4 page: the routed + shared sum rounded to bf16 and
 *      folded into the tail's expand.)
 * The bf16 roundings apply when round_bf16 is set; an fp32 configuration
 * keeps every value in fp32.
 *
 * With n_layers > 1 a step runs a chain: layer l's post/comb expand is
 * deferred and fused into layer l+1's opening pass (which writes the
 * residual streams and the mix partials together), and the last layer's
 * expand is closed at its own tail — one launch per layer (SGLang page,
 * Modifications: cross-layer fusion, final post deferred to the model tail).
 *
 * Conventions for every entry point:
 *   - Return 0 on success or a negative MONO_ERR_* code; mono_ffn_last_error
 *     then holds every reason, newline-separated.
 *   - Device pointers are CUDA device addresses on the plan's device; the
 *     caller keeps ownership and they must not be freed while in use.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).
 *   - Nothing traps on the device: a wait that exceeds the plan's timeout
 *     records an error word that mono_ffn_query_error reports.
 */
#ifndef MONO_FFN_H
#define MONO_FFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* element formats */
enum {
  MONO_F32 = 0,          /* IEEE binary32 */
  MONO_BF16 = 1,         /* bfloat16 */
  MONO_FP8E4M3_B128 = 2, /* e4m3fn codes + one fp32 scale per 1 x 128 block along the input dimension */
  MONO_MXFP4 = 3         /* e2m1 codes, two per byte (even element low nibble) + one e8m0 scale per 32 inputs */
};

/* error codes */
enum {
  MONO_OK = 0,
  MONO_ERR_INVALID_ARG = -1,
  MONO_ERR_UNSUPPORTED_ARCH = -2,
  MONO_ERR_NOT_CORESIDENT = -3,
  MONO_ERR_OOM = -4,
  MONO_ERR_NOT_PACKED = -5,
  MONO_ERR_CUDA = -6,
  MONO_ERR_DEVICE_TIMEOUT = -7,
  MONO_ERR_DEVICE_ABORTED = -8
};

typedef struct {
  int hidden;       /* H; multiple of 128 (FP8) / 32 (MXFP4) / 8 (bf16) / 4 (fp32) */
  int hc;           /* S, hyper-connection streams; must be 4 */
  int n_routed;     /* E routed experts, <= 1024 */
  int top_k;        /* k, 1 <= k <= min(E, 16) */
  int inter;        /* I, SwiGLU intermediate size, same multiple rule as H */
  int max_rows;     /* largest rows a step may pass, 1..8 */
  int n_layers;     /* layers chained per step (>= 1) */
  int hc_dtype;     /* MONO_F32 | MONO_BF16: hc_in / hc_out */
  int norm_dtype;   /* MONO_F32 | MONO_BF16: norm weight */
  int expert_dtype; /* any format above; the shared expert uses the same */
  int round_bf16;   /* 1: bf16 rounding after collapse, norm, gate/up, routed+shared sum */
  float rms_eps;    /* 1e-6 */
  float pre_eps;    /* 1e-6 */
  float post_mult;  /* 2.0 */
  float route_scale;/* 2.5 */
  float denom_clamp;/* lower clamp of the selected-score sum, e.g. 1e-20 */
  int sinkhorn_iters; /* 20 */
  unsigned wait_timeout_us; /* bound of every device-side wait; 0 = 250000 */
  int device;       /* CUDA device ordinal */
  int grid;         /* persistent CTAs; 0 = one per SM */
  int dense;        /* 1: a dense layer: no router; its SwiGLU MLP of width (n_routed + 1) * inter is
                       the n_routed + 1 slots in slot order, run as expert-shaped slices each taken
                       with weight 1 (vLLM MonoKernel page, Weights); top_k must equal n_routed, and
                       router_w / router_bias may be NULL at packing */
  int act_mx8;      /* 1: MXFP8 activations for MXFP4 experts (vLLM MonoKernel page, Numerics): n and the
                       SwiGLU output are quantised to e4m3 with one e8m0 scale per 32 values (OCP MX rule)
                       before each expert matvec, which then runs as one block-scaled e2m1 x e4m3 MMA
                       term; MXFP4 experts on the tensor-core path only (round_bf16, hidden and inter
                       multiples of 128, hidden and inter <= 5120).  0: weight-only dequantisation */
} mono_ffn_config;

/* One layer's weights, device pointers in logical (caller) layouts, read only
 * during mono_ffn_pack_weights:
 *   mix_w       fp32 [S*H][2S + S*S], row s*H + h; columns [pre | post | comb (i,j) at 2S + S i + j]
 *   norm_w      [H] in norm_dtype
 *   router_w    fp32 [H][E] (logits = n @ router_w)
 *   router_bias fp32 [E]
 *   w_gate, w_up  [E+1][I][H] expert codes (output-major; MXFP4: [E+1][I][H/2] bytes)
 *   w_down        [E+1][H][I]                          (MXFP4: [E+1][H][I/2] bytes)
 *   s_gate, s_up  scales [E+1][I][H/128] fp32 (FP8) or [E+1][I][H/32] e8m0 bytes (MXFP4); NULL otherwise
 *   s_down        scales [E+1][H][I/128] or [E+1][H][I/32]
 * Slot E (the last) is the shared expert. */
typedef struct {
  const float* mix_w;
  const void* norm_w;
  const float* router_w;
  const float* router_bias;
  const void* w_gate;
  const void* w_up;
  const void* w_down;
  const void* s_gate;
  const void* s_up;
  const void* s_down;
} mono_ffn_layer_weights;

/* Optional device outputs of one layer's intermediate values (any pointer may
 * be NULL), written by every later step until replaced:
 *   mix [R][24] fp32 (after the rho scale), pre [R][4], post [R][4], comb [R][16] fp32,
 *   n [R][H] fp32 (after its rounding), logits [R][E] fp32, idx [R][k] int32
 *   (selection order), w [R][k] fp32, y [R][H] fp32 (routed + shared after its rounding),
 *   x [R][4][H] fp32: the residual streams the layer read (in a chain, the
 *   previous layer's expand as this layer materialised it). */
typedef struct {
  float* mix;
  float* pre;
  float* post;
  float* comb;
  float* n;
  float* logits;
  int* idx;
  float* w;
  float* y;
  float* x;
} mono_ffn_taps;

typedef struct {
  int code;   /* 0, MONO_ERR_DEVICE_TIMEOUT or MONO_ERR_DEVICE_ABORTED */
  int stage;  /* where the first failing wait was (MONO_STAGE_*) */
  int cta;    /* the CTA that recorded it */
  int layer;  /* the layer slot */
} mono_ffn_status;

enum {
  MONO_STAGE_MIX = 1,     /* mix partials of all CTAs */
  MONO_STAGE_LOGITS = 2,  /* router logits of all CTAs */
  MONO_STAGE_LISTS = 3,   /* this CTA's top-k / work lists */
  MONO_STAGE_ACT = 4,     /* SwiGLU activations of all CTAs */
  MONO_STAGE_RING = 5,    /* a weight-ring stage (TMA completion or slot release) */
  MONO_STAGE_Y = 6,       /* expert outputs of all CTAs (tensor-core kernel) */
  MONO_STAGE_COLLAPSE = 7 /* collapsed h-slices of all CTAs */
};

typedef struct {
  int grid;                 /* CTAs per launch */
  int threads;              /* threads per CTA */
  int smem_bytes;           /* dynamic shared memory per CTA */
  int ring_stages;          /* weight-ring depth */
  int ring_slot_bytes;      /* bytes per ring stage */
  int64_t expert_bytes;     /* packed bytes of one expert slot (gate + up + down + scales) */
  int64_t dense_bytes;      /* mix + router + bias + norm bytes per layer */
  int64_t packed_bytes;     /* all plan-owned packed weights */
  int64_t scratch_bytes;    /* plan-owned scratch (partials, logits, activations, pending state, sync) */
} mono_ffn_info;

typedef struct mono_ffn_plan_s mono_ffn_plan_t;

/* Validate cfg, check the device (sm_100a, co-residency of the persistent
 * grid) and allocate the plan: packed-weight storage for n_layers layers,
 * scratch, per-layer sync words and the error word.  Every refusal reason
 * is listed in mono_ffn_last_error(NULL) when *out is not created. */
int mono_ffn_plan(const mono_ffn_config* cfg, mono_ffn_plan_t** out);

/* Repack one layer's weights (logical layouts above) into the plan's kernel
 * layout, router transposed to [E][H].  A one-time conversion (vLLM
 * MonoKernel page, Weights: the weights are packed one time).  Expert layouts:
 *   - bf16 on the tensor cores (hidden, inter multiples of 128): blocks of 128
 *     rows of K-major core matrices, gate and up interleaved per row group;
 *   - FP8 / MXFP4 on the tensor cores (bf16-rounded layers, multiples of 128):
 *     units of 128 rows x 128 inputs, 16-byte chunk j of row i at [j][i];
 *     FP8 block scales in arrays of their own; MXFP4 with the sign bits moved
 *     inside each 32-bit word of 8 codes, each block's exponent stored
 *     relative to its row's largest minus 6, and 2^(that reference) per row
 *     in arrays of their own;
 *   - otherwise rows cut into contraction chunks with their block scales
 *     interleaved, gate and up chunks of a channel adjacent.
 * Asynchronous on `stream`; the inputs may be freed after the stream reaches
 * this point.  MXFP4 on the tensor cores first reads the scale codes
 * (synchronising `stream`) and refuses code 255 (NaN) with
 * MONO_ERR_INVALID_ARG. */
int mono_ffn_pack_weights(mono_ffn_plan_t* plan, int layer, const mono_ffn_layer_weights* w, void* stream);

/* Run one step: n_layers persistent launches on `stream`.  hc_in, hc_out:
 * device [rows][S][H] in hc_dtype; they must not overlap.  rows == 0 is a
 * no-op; rows > max_rows is MONO_ERR_INVALID_ARG.  Allocates nothing and does
 * not synchronise the host. */
int mono_ffn_step(mono_ffn_plan_t* plan, int rows, const void* hc_in, void* hc_out, void* stream);

/* One step at a fixed launch width with padding rows (vLLM "[ROCm][Perf]
 * [GLM-5] Fused sparse-layer decode via AITER MonoKernel", when the path
 * runs: batches are padded to the captured widths and pad rows carry a slot
 * below zero).  row_slot: device int32 [width]; row r is a padding row when
 * row_slot[r] < 0: its hc_in is never used (it may hold anything, NaN
 * included), it selects no expert (no weight bytes are read for it) and its
 * hc_out is left as it was.  Live rows compute exactly as in mono_ffn_step.
 * So one width (a CUDA graph captured at 1, 2, 4 or 8 rows) serves every
 * batch up to it.  width == 0 is a no-op; width > max_rows or overlapping
 * hc_in / hc_out is MONO_ERR_INVALID_ARG.  Asynchronous; allocates nothing. */
int mono_ffn_step_padded(mono_ffn_plan_t* plan, int width, const int* row_slot, const void* hc_in, void* hc_out,
                         void* stream);

/* One step opened by the attention sublayer's pending post / expand (the
 * within-layer boundary: SGLang "[DeepSeek-V4] Add mhc_fused_post_pre
 * kernel", Modifications: the attention sublayer's hc_post fused with the
 * FFN's hc_pre inside one layer):
 * for each row r the FFN's residual streams are
 *   X_i = round(sum_j attn_comb[r][i][j] x_attn[r][j] + attn_post[r][i] y_attn[r])
 * (round = to hc_dtype), materialised in the opening pass together with the
 * mix products, then the layer (and, with n_layers > 1, the chain) as in
 * mono_ffn_step.  So a caller hands over exactly what the attention sublayer
 * leaves pending instead of closing its expand in a kernel of its own.
 *   x_attn   [rows][S][H] hc_dtype: the residual streams before the attention sublayer
 *   attn_post [rows][S] fp32, attn_comb [rows][S][S] fp32 (row-major (i, j))
 *   y_attn   [rows][H] hc_dtype: the attention sublayer's output
 *   hc_out   [rows][S][H] hc_dtype; must not overlap any input
 * All device memory on the plan's device, caller-owned.  rows == 0 is a
 * no-op; rows > max_rows or overlapping buffers are MONO_ERR_INVALID_ARG.
 * Asynchronous; allocates nothing. */
int mono_ffn_step_pending(mono_ffn_plan_t* plan, int rows, const void* x_attn, const float* attn_post,
                          const float* attn_comb, const void* y_attn, void* hc_out, void* stream);

/* The same step with HOST buffers: copies hc_in (pinned or pageable host
 * memory) to the plan's device staging buffer, runs the step, copies the
 * result back to hc_out and synchronises `stream`. */
int mono_ffn_step_host(mono_ffn_plan_t* plan, int rows, const void* hc_in_host, void* hc_out_host, void* stream);

/* Register (or clear, with NULL) the intermediate-value outputs of a layer. */
int mono_ffn_set_taps(mono_ffn_plan_t* plan, int layer, const mono_ffn_taps* taps);

/* Synchronise the plan's device, read the device error word into *st (may be
 * NULL) and, if a wait failed, reset the sync state so the next step starts
 * clean.  Returns 0 or the recorded MONO_ERR_DEVICE_* code. */
int mono_ffn_query_error(mono_ffn_plan_t* plan, mono_ffn_status* st);

/* Shapes and sizes the plan chose. */
int mono_ffn_get_info(const mono_ffn_plan_t* plan, mono_ffn_info* info);

/* Stage timestamps for profiling: with buf != NULL (device memory of
 * n_layers * grid * 32 uint64), every CTA of layer l writes %globaltimer (ns)
 * at its stage boundaries to buf[(l * grid + cta) * 32 + point]:
 * 0 start, 1 mix partials published, 2 mix totals seen, 3 n ready,
 * 4 router logits published, 5 top-k lists ready, 6 shared gate/up done,
 * 7 routed gate/up done, 8 activations seen (tensor-core kernel: the first
 * down expert's), 9 down projections done,
 * 10 end, 11 producer saw the lists, 12 producer issued every copy;
 * tensor-core kernel also: 13 first routed gate/up stage arrived, 14 routed
 * gate/up MMAs issued, 15 first down operand ready, 16 every MMA issued,
 * 18 first routed copy issued, 19 first down
 * copy issued, 20 first shared gate/up tile read; both: 21 logits counter
 * complete, 22 top-k done, 23 pre/post ready, 24 every CTA's collapsed
 * slice seen, 25 router dot products done, 26 top-k inputs loaded, 27 this
 * CTA's collapsed slice published, 28 mix inputs in shared memory; all
 * kernels: 17 mix partials computed, 29 every slice of the collapse in
 * shared memory, 30 n normalised.
 * The tensor-core kernel stores its SM id (not a time) at point 31.
 * Points a kernel does not reach stay as they were.
 * NULL turns it off (the default). */
int mono_ffn_set_trace(mono_ffn_plan_t* plan, unsigned long long* buf);

/* Fault injection for tests (no GPU fault: every wait is bounded).  CTA
 * `cta` (-1 = none) withholds its arrival at one grid stage, so the other
 * CTAs' bounded waits there expire and mono_ffn_query_error reports
 * MONO_ERR_DEVICE_TIMEOUT with that stage:
 *   MONO_STAGE_MIX, MONO_STAGE_COLLAPSE, MONO_STAGE_LOGITS: the prologue's
 *     grid stages;
 *   MONO_STAGE_ACT: the CUDA-core kernel's activation counter; on the
 *     tensor-core kernels the per-expert activation count of the shared
 *     expert's first gate/up block (withheld by whichever CTA completes that
 *     block; `cta` only enables it);
 *   MONO_STAGE_Y: the expert-output counter (tensor-core kernels only).
 * Other stages, or cta >= grid, are MONO_ERR_INVALID_ARG.  Stays in force
 * until called with cta = -1. */
int mono_ffn_debug_skip_arrival(mono_ffn_plan_t* plan, int cta, int stage);

/* Race detection for tests: with max_ns > 0 (at most 100000) every thread
 * that publishes a grid-visible arrival (the stage counters, the split-block
 * arrivals of the tensor-core kernels, the per-expert activation counts)
 * first sleeps a pseudo-random hash(CTA, step, point) % max_ns
 * nanoseconds, so the order in which CTAs arrive changes from step to step;
 * results must not change.  0 turns it off (the default). */
int mono_ffn_debug_jitter(mono_ffn_plan_t* plan, unsigned max_ns);

/* Router select without a plan and without allocating anything.
 *
 * No counterpart on the pages: their router stage lives inside the fused
 * layer kernel.  This is a standalone variant of that stage (the router
 * logits, sqrt(softplus) scores, selection bias, canonical top-k and the
 * normalised, scaled weights; ds4 "v41: fuse the single-box decode glue",
 * the router "Mega-Gate" commit), for callers that cannot allocate device
 * memory when they need a routing decision: a serving engine that reserves
 * all device memory up front, or code between captured graph segments that
 * must not reach the allocator.  Its scratch is a fixed static device array,
 * so no call allocates (no cudaMalloc, no library allocation).
 *
 *   n          [rows][hidden] device, bf16 (n_bf16 = 1) or fp32, the normed rows
 *   router_w   [hidden][n_routed] fp32 device (logits = n @ router_w)
 *   router_bias[n_routed] fp32 device, added for selection only
 *   idx        [rows][top_k] int32 device, out: selected experts in order
 *   w          [rows][top_k] fp32 device, out: score / max(sum, denom_clamp) * route_scale
 *   stream     cudaStream_t (NULL = legacy default stream)
 *
 * Limits (the size of the static scratch): rows <= 8, n_routed <= 1024,
 * top_k <= 16 (and <= n_routed).  Anything beyond is refused with
 * MONO_ERR_INVALID_ARG and every reason in mono_ffn_last_error(NULL);
 * rows == 0 is a no-op.  Asynchronous: errors of the running kernel show up
 * on the stream.
 *
 * Scratch: 256 KB of partial logits, which need no initial value, and one
 * arrival counter, which must be zero when a call starts.  It is zero from
 * static initialisation and every call leaves it at zero.  Calls that overlap
 * in time on one device (other streams, other threads) share the scratch and
 * race: order them.  The first call on each device looks the scratch address
 * up (cudaGetSymbolAddress, which may load the module); make that first call
 * outside stream capture.  The address is kept for the life of the process:
 * after cudaDeviceReset on a device, do not call this entry point on that
 * device again. */
int mono_ffn_route_noalloc(int rows, int hidden, int n_routed, int top_k, const void* n, int n_bf16,
                           const float* router_w, const float* router_bias, float route_scale, float denom_clamp,
                           int* idx, float* w, void* stream);

/* Every reason of the last failure on this plan (or, for plan == NULL, of
 * the last failed mono_ffn_plan or mono_ffn_route_noalloc call on this
 * thread). */
const char* mono_ffn_last_error(const mono_ffn_plan_t* plan);

void mono_ffn_destroy(mono_ffn_plan_t* plan);

/* ABI version of this header. */
int mono_ffn_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif
