/*
 * CPU oracle of the fused decode FFN half-layer — TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, op-by-op statement of what one FFN half-layer of a
 * DeepSeek-V4.1-style decoder computes at decode time: the mHC
 * (hyper-connection) post->pre boundary, the weighted RMSNorm, the router
 * select, the shared and routed SwiGLU experts, the routed+shared sum and the
 * next mHC expand.  Accumulation is in double; values are rounded to bf16 /
 * fp32 only at the points the layer defines.  Only tests, the smoke check and
 * the benchmark's CPU-baseline leg may load this library; the product path
 * never does.
 *
 * Sources (web pages on the method; cited by page title and section):
 *  - ds4 "v41: fuse the single-box decode glue (HC, MoE, attention)", PR
 *    description, "What" and the HC / MoE fusion commits: hyper-connection
 *    norm + mix matvec, split/sinkhorn, pre-weighted collapse + BF16 +
 *    weighted RMSNorm + BF16, post/comb expand + BF16; router "Mega-Gate":
 *    fp32 logits matvec, sqrt(softplus), bias for selection, canonical
 *    (score desc, idx asc) top-k, normalised weights with clamp, division and
 *    scale as separately rounded ops; shared expert gate/up rounded to BF16
 *    before SwiGLU; block = bf16(routed + shared).
 *  - SGLang "[DeepSeek-V4] Add mhc_fused_post_pre kernel", "Motivation" and
 *    "Modifications": the mix as pre-norm GEMM partials and RMS square-sum
 *    partials finalised together; the previous layer's hc_post fused with the
 *    next hc_pre and the final post closed at the model tail.
 *  - vLLM "[ROCm][Perf][GLM-5] Fused sparse-layer decode via AITER
 *    MonoKernel", "Weights": shared expert stored in the last expert slot.
 *  - The layer configuration this build targets: 4 HC streams, mix width 24
 *    (4 pre, 4 post, 16 comb), pre = sigmoid + 1e-6, post = 2 sigmoid, comb =
 *    20-iteration Sinkhorn of exp over 4x4, RMSNorm eps 1e-6, route scale 2.5,
 *    bf16 rounding after the collapse, after the norm, on gate/up and on the
 *    routed+shared sum; FP8 e4m3 1x128 and MXFP4 (e2m1, 32-blocks, e8m0)
 *    weight formats.
 */
#ifndef MONO_ORACLE_H
#define MONO_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_FP8 = 2, ORC_MXFP4 = 3 };

typedef struct {
  int hidden;   /* H */
  int hc;       /* S, hyper-connection streams (4) */
  int n_routed; /* E */
  int top_k;    /* k */
  int inter;    /* I, SwiGLU intermediate */
  int rows;     /* R */
  int hc_dtype;   /* ORC_F32 | ORC_BF16: hc_in / hc_out element type */
  int norm_dtype; /* ORC_F32 | ORC_BF16: norm weight element type */
  int w_dtype;    /* expert weight format */
  int round_bf16; /* 1: round to bf16 after collapse, after norm, gate/up, routed+shared sum */
  int sinkhorn_iters;
  double rms_eps, pre_eps, post_mult, route_scale, denom_clamp;
  int dense;      /* 1: no router; a dense SwiGLU MLP of width (E + 1) I over all slots (top_k = E) */
  int act_mx8;    /* 1 (MXFP4 experts only): activations quantised to MXFP8 before each expert matvec */
} orc_cfg;

/* Logical layouts (row-major):
 *   mix_w    [S*H][2S + S*S] fp32, flattened HC index s*H + h; columns
 *            [pre 0..S-1 | post 0..S-1 | comb (i, j) at 2S + S*i + j]
 *   norm_w   [H]
 *   router_w [H][E] fp32 (logits = n @ router_w), router_bias [E] fp32
 *   experts  slot e in [0, E]; slot E is the shared expert.
 *            gate, up [I][H], down [H][I] (output-major, contraction
 *            contiguous).  FP8: e4m3 codes + fp32 scales [out][in/128];
 *            MXFP4: codes [out][in/2] (even element in the low nibble) +
 *            e8m0 scales [out][in/32].  A NULL slot is allowed for an expert
 *            that the routing does not select. */
typedef struct {
  const float* mix_w;
  const void* norm_w;
  const float* router_w;
  const float* router_bias;
  const void* const* w_gate;
  const void* const* w_up;
  const void* const* w_down;
  const void* const* s_gate;
  const void* const* s_up;
  const void* const* s_down;
} orc_weights;

/* Optional per-row outputs of intermediate values; any pointer may be NULL. */
typedef struct {
  double* rho;    /* [R]       1/sqrt(mean X^2 + eps) over the flattened HC row */
  double* mix;    /* [R][2S+S*S] */
  double* pre;    /* [R][S] */
  double* post;   /* [R][S] */
  double* comb;   /* [R][S][S] */
  double* a;      /* [R][H]    collapse (after its rounding) */
  double* n;      /* [R][H]    normed (after its rounding) */
  float* logits;  /* [R][E] */
  float* score;   /* [R][E] */
  float* sel;     /* [R][E] */
  int* idx;       /* [R][k] */
  float* w;       /* [R][k] */
  double* y;      /* [R][H]    routed + shared (after its rounding) */
} orc_taps;

/* One layer: hc_in [R][S][H] -> hc_out [R][S][H] (hc_dtype).  Returns 0, or
 * -(100 + e) if expert slot e is needed but NULL, or -1 on a bad config. */
int orc_layer(const orc_cfg* cfg, const orc_weights* w, const void* hc_in, void* hc_out, orc_taps* taps);

/* Steps up to the routing decision only (taps up to idx / w). */
int orc_route(const orc_cfg* cfg, const orc_weights* w, const void* hc_in, orc_taps* taps);

/* A chain of n_layers layers.  deferred = 0: each layer runs all its steps
 * and its rounded output feeds the next.  deferred = 1: layer l stops after
 * the routed+shared sum, and its post/comb expand runs at the start of layer
 * l+1 in one pass with that layer's mix and square sums; the last layer's
 * expand is closed at the tail. */
int orc_chain(const orc_cfg* cfg, int n_layers, const orc_weights* w, const void* hc_in, void* hc_out,
              int deferred);

/* Within-layer boundary: the attention sublayer's pending post / expand
 * (x_attn [R][S][H] and y_attn [R][H] in hc_dtype, attn_post [R][S] and
 * attn_comb [R][S][S] fp32) closed in this layer's opening pass, then the
 * layer.  x_out (may be NULL): the materialised residual streams. */
int orc_layer_pending(const orc_cfg* cfg, const orc_weights* w, const void* x_attn, const float* attn_post,
                      const float* attn_comb, const void* y_attn, void* hc_out, void* x_out, orc_taps* taps);

/* The expand alone (op by op): x_out_i = sum_j comb_ij x_in_j + post_i y. */
int orc_expand(const orc_cfg* cfg, const void* x_in, const float* post, const float* comb, const void* y,
               void* x_out);

/* Building blocks, exported for the oracle's own pins. */
void orc_sinkhorn(const double* logits, int s, int iters, double* comb);
void orc_topk(const float* sel, int e, int k, int* idx);
double orc_dec_bf16(uint16_t b);
double orc_dec_e4m3(uint8_t b);
double orc_dec_e2m1(uint8_t nibble);
double orc_dec_e8m0(uint8_t b);
uint16_t orc_round_bf16(double x);
void orc_quant_fp8(const float* w, int64_t rows, int64_t cols, uint8_t* q, float* s);
void orc_quant_mxfp4(const float* w, int64_t rows, int64_t cols, uint8_t* q, uint8_t* e);
void orc_quant_mx8(const double* x, int64_t n, double* out, uint8_t* codes, uint8_t* scales);

#ifdef __cplusplus
}
#endif
#endif
