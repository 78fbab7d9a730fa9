/*
 * CPU oracle of the fused decode FFN half-layer — TEST INFRASTRUCTURE ONLY
 * (tests, the smoke check and the benchmark's CPU-baseline leg).  See
 * mono_oracle.h for the sources followed; each step below names the passage it
 * states.  Plain loops, double accumulation, no blocking or fusion beyond what
 * the definition states.  OpenMP only splits independent output channels, each
 * computed by one thread in a fixed order, so results do not depend on the
 * thread count.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared -lm
 */
#include "mono_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define EXPORT __attribute__((visibility("default")))

/* ---------------------------------------------------------------- codecs -- */

/* bf16: the upper 16 bits of an IEEE binary32 */
EXPORT double orc_dec_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* e4m3fn (OCP 8-bit floating point, E4M3): bias 7, no infinities, S.1111.111 is NaN */
EXPORT double orc_dec_e4m3(uint8_t b) {
  int s = (b >> 7) & 1, e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  v = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10);
  return s ? -v : v;
}

/* e2m1 (OCP MX FP4): bias 1, magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 */
EXPORT double orc_dec_e2m1(uint8_t nib) {
  int s = (nib >> 3) & 1, e = (nib >> 1) & 3, m = nib & 1;
  double v = e == 0 ? 0.5 * m : ldexp((double)(2 + m), e - 2);
  return s ? -v : v;
}

/* e8m0 (OCP MX scale): 2^(b - 127), 0xFF is NaN */
EXPORT double orc_dec_e8m0(uint8_t b) {
  if (b == 0xFF) return NAN;
  return ldexp(1.0, (int)b - 127);
}

/* double -> bf16, one rounding to nearest even (8 significant bits, binary32
 * exponent range with subnormals down to 2^-133) */
EXPORT uint16_t orc_round_bf16(double x) {
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x), q, v;
  int ex, qe;
  float f;
  uint32_t u;
  if (isnan(x)) return 0x7FC0;
  if (a == 0.0) return sign;
  if (isinf(x)) return (uint16_t)(sign | 0x7F80);
  frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) */
  qe = ex - 1 - 7;
  if (qe < -133) qe = -133;
  q = ldexp(1.0, qe);
  v = nearbyint(a / q) * q;
  if (v > 3.3895313892515355e38) return (uint16_t)(sign | 0x7F80);
  f = (float)v;
  memcpy(&u, &f, 4);
  return (uint16_t)(sign | ((u >> 16) & 0x7FFF));
}

static double rbf16(double x) { return orc_dec_bf16(orc_round_bf16(x)); }

/* nearest code of a sorted magnitude table, ties to the even code */
static int nearest_even(const double* mag, int n, double a) {
  int lo = 0, hi = n - 1;
  if (a >= mag[n - 1]) return n - 1; /* saturate */
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (mag[mid] <= a) lo = mid; else hi = mid;
  }
  /* mag[lo] <= a < mag[hi], hi == lo + 1 */
  {
    double dl = a - mag[lo], dh = mag[hi] - a;
    if (dl < dh) return lo;
    if (dh < dl) return hi;
    return (lo & 1) ? hi : lo;
  }
}

/* FP8 1x128 block quantiser (the rule the layer's FP8 weights were made with):
 * s = amax / 448 in fp32 (1 when amax = 0), q = e4m3fn(w / s), the quotient
 * rounded to fp32 and then to the nearest e4m3 value (ties to even),
 * saturating at 448. */
EXPORT void orc_quant_fp8(const float* w, int64_t rows, int64_t cols, uint8_t* q, float* s) {
  double mag[127];
  int64_t nb = cols / 128, rb;
  for (int c = 0; c < 127; ++c) mag[c] = orc_dec_e4m3((uint8_t)c);
#pragma omp parallel for schedule(static)
  for (rb = 0; rb < rows * nb; ++rb) {
    const float* src = w + rb * 128;
    float amax = 0.0f, sc;
    for (int i = 0; i < 128; ++i) amax = fmaxf(amax, fabsf(src[i]));
    sc = amax > 0.0f ? (float)((double)amax / 448.0) : 1.0f;
    s[rb] = sc;
    for (int i = 0; i < 128; ++i) {
      float v = (float)((double)src[i] / (double)sc);
      int code = nearest_even(mag, 127, fabs((double)v));
      q[rb * 128 + i] = (uint8_t)(code | (signbit(v) ? 0x80 : 0));
    }
  }
}

/* MXFP8 (e4m3) quantiser of an activation vector, OCP MX v1.0 shared-exponent
 * rule: per block of 32 consecutive values, X = floor(log2 amax) - 8 (8 = the
 * largest e4m3 exponent), clamped to the e8m0 range [-127, 127]; each element
 * becomes the e4m3 value nearest to x / 2^X (ties to the even code),
 * saturating at 448, and decodes to that value times 2^X.  An all-zero block
 * keeps scale byte 0 and zero codes.  codes / scales (may be NULL) receive the
 * e4m3 codes and the e8m0 bytes. */
EXPORT void orc_quant_mx8(const double* x, int64_t n, double* out, uint8_t* codes, uint8_t* scales) {
  double mag[127];
  for (int c = 0; c < 127; ++c) mag[c] = orc_dec_e4m3((uint8_t)c);
  for (int64_t b = 0; b < n / 32; ++b) {
    const double* src = x + b * 32;
    double amax = 0.0;
    int X = -127;
    for (int i = 0; i < 32; ++i) amax = fmax(amax, fabs(src[i]));
    if (amax > 0.0) {
      int ex;
      frexp(amax, &ex);
      X = (ex - 1) - 8;
      if (X < -127) X = -127;
      if (X > 127) X = 127;
    }
    if (scales) scales[b] = amax > 0.0 ? (uint8_t)(X + 127) : 0;
    for (int i = 0; i < 32; ++i) {
      const double v = ldexp(src[i], -X);
      const int code = amax > 0.0 ? nearest_even(mag, 127, fabs(v)) : 0;
      const int neg = signbit(v) && code != 0;
      out[b * 32 + i] = (neg ? -1.0 : 1.0) * ldexp(mag[code], X);
      if (codes) codes[b * 32 + i] = (uint8_t)(code | (neg ? 0x80 : 0));
    }
  }
}

/* MXFP4 quantiser (OCP MX v1.0 shared-exponent rule): per 32-block,
 * X = floor(log2 amax) - 2 (the largest e2m1 exponent), scale byte X + 127
 * clamped to [0, 254] (0 when amax = 0); element = e2m1(w / 2^X), the scaled
 * value rounded to fp32 and then to the nearest e2m1 value (ties to even),
 * saturating at 6. */
EXPORT void orc_quant_mxfp4(const float* w, int64_t rows, int64_t cols, uint8_t* q, uint8_t* e) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  int64_t nb = cols / 32, rb;
#pragma omp parallel for schedule(static)
  for (rb = 0; rb < rows * nb; ++rb) {
    const float* src = w + rb * 32;
    float amax = 0.0f;
    int byte = 0;
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(src[i]));
    if (amax > 0.0f) {
      int ex;
      frexp((double)amax, &ex);
      byte = (ex - 1) - 2 + 127;
      if (byte < 0) byte = 0;
      if (byte > 254) byte = 254;
    }
    e[rb] = (uint8_t)byte;
    for (int i = 0; i < 32; i += 2) {
      uint8_t nib[2];
      for (int t = 0; t < 2; ++t) {
        float v = (float)ldexp((double)src[i + t], -(byte - 127));
        int code = nearest_even(mag, 8, fabs((double)v));
        nib[t] = (uint8_t)(code | (signbit(v) ? 8 : 0));
      }
      q[rb * 16 + i / 2] = (uint8_t)(nib[0] | (nib[1] << 4));
    }
  }
}

/* ---------------------------------------------------------------- helpers -- */

static double dec_act(const void* p, int64_t i, int dt) {
  return dt == ORC_BF16 ? orc_dec_bf16(((const uint16_t*)p)[i]) : (double)((const float*)p)[i];
}

static void enc_act(void* p, int64_t i, int dt, double v) {
  if (dt == ORC_BF16) ((uint16_t*)p)[i] = orc_round_bf16(v);
  else ((float*)p)[i] = (float)v;
}

/* one decoded row [in] of an expert matrix stored [out][in] */
static void dec_weight_row(const void* codes, const void* scales, int dt, int64_t row, int64_t in,
                           double* dst) {
  int64_t c;
  switch (dt) {
    case ORC_F32:
      for (c = 0; c < in; ++c) dst[c] = (double)((const float*)codes)[row * in + c];
      break;
    case ORC_BF16:
      for (c = 0; c < in; ++c) dst[c] = orc_dec_bf16(((const uint16_t*)codes)[row * in + c]);
      break;
    case ORC_FP8:
      for (c = 0; c < in; ++c)
        dst[c] = orc_dec_e4m3(((const uint8_t*)codes)[row * in + c]) *
                 (double)((const float*)scales)[row * (in / 128) + c / 128];
      break;
    default: /* ORC_MXFP4 */
      for (c = 0; c < in; ++c) {
        uint8_t byte = ((const uint8_t*)codes)[row * (in / 2) + c / 2];
        uint8_t nib = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
        dst[c] = orc_dec_e2m1(nib) * orc_dec_e8m0(((const uint8_t*)scales)[row * (in / 32) + c / 32]);
      }
      break;
  }
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static double softplus(double x) { return (x > 0.0 ? x : 0.0) + log1p(exp(-fabs(x))); }

/* the MXFP8-activation numerics apply to MXFP4 experts only */
static int mx8_on(const orc_cfg* c) { return c->act_mx8 && c->w_dtype == ORC_MXFP4; }

static int check_cfg(const orc_cfg* c) {
  if (c->hidden <= 0 || c->hc <= 0 || c->n_routed <= 0 || c->top_k <= 0 || c->top_k > c->n_routed ||
      c->inter <= 0 || c->rows < 0)
    return -1;
  if (c->w_dtype == ORC_FP8 && (c->hidden % 128 || c->inter % 128)) return -1;
  if (c->dense && c->top_k != c->n_routed) return -1;
  if (c->w_dtype == ORC_MXFP4 && (c->hidden % 32 || c->inter % 32)) return -1;
  return 0;
}

/* ------------------------------------------------ hyper-connection steps -- */

/* Sinkhorn normalisation of exp(logits) over an s x s matrix: subtract the
 * largest logit (exact up to rounding: it scales every entry alike), then per
 * iteration divide every row by its sum and then every column by its sum. */
EXPORT void orc_sinkhorn(const double* logits, int s, int iters, double* comb) {
  double mx = logits[0];
  for (int i = 1; i < s * s; ++i) mx = fmax(mx, logits[i]);
  for (int i = 0; i < s * s; ++i) comb[i] = exp(logits[i] - mx);
  for (int it = 0; it < iters; ++it) {
    for (int i = 0; i < s; ++i) {
      double t = 0.0;
      for (int j = 0; j < s; ++j) t += comb[i * s + j];
      for (int j = 0; j < s; ++j) comb[i * s + j] /= t;
    }
    for (int j = 0; j < s; ++j) {
      double t = 0.0;
      for (int i = 0; i < s; ++i) t += comb[i * s + j];
      for (int i = 0; i < s; ++i) comb[i * s + j] /= t;
    }
  }
}

/* Canonical top-k: order by (sel descending, expert index ascending). */
EXPORT void orc_topk(const float* sel, int e, int k, int* idx) {
  char* taken = (char*)calloc((size_t)e, 1);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int x = 0; x < e; ++x) {
      if (taken[x]) continue;
      if (best < 0 || sel[x] > sel[best]) best = x; /* strict: a tie keeps the lower index */
    }
    idx[j] = best;
    taken[best] = 1;
  }
  free(taken);
}

/* Per-row state between the steps of one layer. */
typedef struct {
  double rho, mix[64], pre[8], post[8], comb[64];
  double *a, *n, *y;
  float *logits, *score, *sel, *w;
  int* idx;
} row_state;

/* Steps 1-3 of the hyper-connection pre step for one row X [S][H]:
 * the flattened row's RMS factor rho = 1 / sqrt(sum X^2 / (S H) + eps), the
 * mix as rho times the plain matvec X @ mix_w (pre-norm GEMM partials and
 * square sums finalised together), then the split into pre / post / comb. */
static void hc_mix_split(const orc_cfg* c, const orc_weights* w, const double* X, row_state* st) {
  const int S = c->hc, H = c->hidden, M = 2 * c->hc + c->hc * c->hc;
  double ss = 0.0;
  for (int64_t i = 0; i < (int64_t)S * H; ++i) ss += X[i] * X[i];
  st->rho = 1.0 / sqrt(ss / (double)(S * H) + c->rms_eps);
  for (int col = 0; col < M; ++col) {
    double acc = 0.0;
    for (int64_t i = 0; i < (int64_t)S * H; ++i) acc += X[i] * (double)w->mix_w[i * M + col];
    st->mix[col] = st->rho * acc;
  }
  for (int i = 0; i < S; ++i) {
    st->pre[i] = sigmoid(st->mix[i]) + c->pre_eps;
    st->post[i] = c->post_mult * sigmoid(st->mix[S + i]);
  }
  orc_sinkhorn(st->mix + 2 * S, S, c->sinkhorn_iters, st->comb);
}

/* Steps 5-6: pre-weighted collapse a = sum_s pre_s X_s (-> bf16), then the
 * weighted RMSNorm n = a / sqrt(mean a^2 + eps) * w_norm (-> bf16). */
static void collapse_norm(const orc_cfg* c, const orc_weights* w, const double* X, row_state* st) {
  const int S = c->hc, H = c->hidden;
  double ms = 0.0, inv;
  for (int h = 0; h < H; ++h) {
    double acc = 0.0;
    for (int s = 0; s < S; ++s) acc += st->pre[s] * X[(int64_t)s * H + h];
    st->a[h] = c->round_bf16 ? rbf16(acc) : acc;
  }
  for (int h = 0; h < H; ++h) ms += st->a[h] * st->a[h];
  inv = 1.0 / sqrt(ms / (double)H + c->rms_eps);
  for (int h = 0; h < H; ++h) {
    double v = st->a[h] * inv * dec_act(w->norm_w, h, c->norm_dtype);
    st->n[h] = c->round_bf16 ? rbf16(v) : v;
  }
}

/* Steps 7-10, the router select: fp32 logits of n @ router_w; score =
 * sqrt(softplus(logit)) in fp32; sel = score + bias in fp32 (selection only);
 * canonical top-k on sel; weight = score / max(sum of selected scores, clamp)
 * * route_scale, every op rounded to fp32. */
static void route(const orc_cfg* c, const orc_weights* w, row_state* st) {
  const int H = c->hidden, E = c->n_routed, K = c->top_k;
  double den = 0.0;
  float fden;
  for (int e = 0; e < E; ++e) {
    double acc = 0.0;
    for (int h = 0; h < H; ++h) acc += st->n[h] * (double)w->router_w[(int64_t)h * E + e];
    st->logits[e] = (float)acc;
    st->score[e] = (float)sqrt(softplus((double)st->logits[e]));
    st->sel[e] = (float)((double)st->score[e] + (double)w->router_bias[e]);
  }
  orc_topk(st->sel, E, K, st->idx);
  for (int j = 0; j < K; ++j) den += (double)st->score[st->idx[j]];
  fden = (float)den;
  if ((double)fden < c->denom_clamp) fden = (float)c->denom_clamp;
  for (int j = 0; j < K; ++j) {
    float q = (float)((double)st->score[st->idx[j]] / (double)fden);
    st->w[j] = (float)((double)q * c->route_scale);
  }
}

/* Step 11 for one expert slot: g = n @ gate^T, u = n @ up^T (-> bf16),
 * act = g * sigmoid(g) * u, d = act @ down^T.  d is accumulated into dst
 * scaled by wt.  Returns -(100 + e) when the slot's weights are missing. */
static int expert(const orc_cfg* c, const orc_weights* w, int e, const double* n, double wt, double* dst) {
  const int H = c->hidden, I = c->inter;
  double* act;
  double* d;
  int64_t ch;
  if (!w->w_gate[e] || !w->w_up[e] || !w->w_down[e]) return -(100 + e);
  act = (double*)malloc(sizeof(double) * (size_t)I);
  d = (double*)malloc(sizeof(double) * (size_t)H);
  /* MXFP8 activations (vLLM MonoKernel page, Numerics: the kernel quantises
   * the activations to MXFP8 for the MXFP4 experts): n before gate / up,
   * and the SwiGLU output before down, each in blocks of 32 along the
   * contraction */
  double* nq = NULL;
  if (mx8_on(c)) {
    nq = (double*)malloc(sizeof(double) * (size_t)H);
    orc_quant_mx8(n, H, nq, NULL, NULL);
    n = nq;
  }
#pragma omp parallel for schedule(static)
  for (ch = 0; ch < I; ++ch) {
    double* row = (double*)malloc(sizeof(double) * (size_t)H);
    double g = 0.0, u = 0.0;
    dec_weight_row(w->w_gate[e], w->s_gate ? w->s_gate[e] : NULL, c->w_dtype, ch, H, row);
    for (int h = 0; h < H; ++h) g += n[h] * row[h];
    dec_weight_row(w->w_up[e], w->s_up ? w->s_up[e] : NULL, c->w_dtype, ch, H, row);
    for (int h = 0; h < H; ++h) u += n[h] * row[h];
    if (c->round_bf16) {
      g = rbf16(g);
      u = rbf16(u);
    }
    act[ch] = g * sigmoid(g) * u;
    free(row);
  }
  if (mx8_on(c)) orc_quant_mx8(act, I, act, NULL, NULL);
#pragma omp parallel for schedule(static)
  for (ch = 0; ch < H; ++ch) {
    double* row = (double*)malloc(sizeof(double) * (size_t)I);
    double acc = 0.0;
    dec_weight_row(w->w_down[e], w->s_down ? w->s_down[e] : NULL, c->w_dtype, ch, I, row);
    for (int i = 0; i < I; ++i) acc += act[i] * row[i];
    d[ch] = acc;
    free(row);
  }
  for (int h = 0; h < H; ++h) dst[h] += wt * d[h];
  free(act);
  free(d);
  free(nq);
  return 0;
}

/* Step 12: y = sum_j w_j d_j + d_shared (-> bf16). */
static int moe(const orc_cfg* c, const orc_weights* w, row_state* st) {
  const int H = c->hidden, E = c->n_routed, K = c->top_k;
  int rc;
  double* acc = (double*)calloc((size_t)H, sizeof(double));
  for (int j = 0; j < K; ++j) {
    rc = expert(c, w, st->idx[j], st->n, (double)st->w[j], acc);
    if (rc) {
      free(acc);
      return rc;
    }
  }
  rc = expert(c, w, E, st->n, 1.0, acc);
  for (int h = 0; h < H; ++h) st->y[h] = c->round_bf16 ? rbf16(acc[h]) : acc[h];
  free(acc);
  return rc;
}

/* Dense layer: a SwiGLU MLP of width (E + 1) I whose weight rows are the E + 1
 * slots' rows in slot order (gate / up row i = slot i / I, row i % I; down
 * row h = the slots' down rows h side by side), evaluated as ONE MLP:
 * g, u = n W (rounded to bf16 when round_bf16), act = silu(g) u, y = act W_down
 * summed over the whole width, rounded like the routed + shared sum.  No
 * router: the vLLM MonoKernel page ("Weights": a dense layer's MLP runs as
 * six expert-shaped slices) computes this MLP with the same kernel, every
 * slice taken with weight 1. */
static int dense_mlp(const orc_cfg* c, const orc_weights* w, row_state* st) {
  const int H = c->hidden, I = c->inter, E1 = c->n_routed + 1;
  const int64_t W = (int64_t)E1 * I;
  double* act;
  int64_t ch;
  for (int e = 0; e < E1; ++e)
    if (!w->w_gate[e] || !w->w_up[e] || !w->w_down[e]) return -(100 + e);
  act = (double*)malloc(sizeof(double) * (size_t)W);
  double* nq = (double*)malloc(sizeof(double) * (size_t)H);
  memcpy(nq, st->n, sizeof(double) * (size_t)H);
  if (mx8_on(c)) orc_quant_mx8(st->n, H, nq, NULL, NULL);
#pragma omp parallel for schedule(static)
  for (ch = 0; ch < W; ++ch) {
    double* row = (double*)malloc(sizeof(double) * (size_t)H);
    const int e = (int)(ch / I), i = (int)(ch % I);
    double g = 0.0, u = 0.0;
    dec_weight_row(w->w_gate[e], w->s_gate ? w->s_gate[e] : NULL, c->w_dtype, i, H, row);
    for (int h = 0; h < H; ++h) g += nq[h] * row[h];
    dec_weight_row(w->w_up[e], w->s_up ? w->s_up[e] : NULL, c->w_dtype, i, H, row);
    for (int h = 0; h < H; ++h) u += nq[h] * row[h];
    if (c->round_bf16) {
      g = rbf16(g);
      u = rbf16(u);
    }
    act[ch] = g * sigmoid(g) * u;
    free(row);
  }
  if (mx8_on(c)) orc_quant_mx8(act, W, act, NULL, NULL);
#pragma omp parallel for schedule(static)
  for (ch = 0; ch < H; ++ch) {
    double* row = (double*)malloc(sizeof(double) * (size_t)W);
    double acc = 0.0;
    for (int e = 0; e < E1; ++e)
      dec_weight_row(w->w_down[e], w->s_down ? w->s_down[e] : NULL, c->w_dtype, ch, I, row + (int64_t)e * I);
    for (int64_t i = 0; i < W; ++i) acc += act[i] * row[i];
    st->y[ch] = c->round_bf16 ? rbf16(acc) : acc;
    free(row);
  }
  for (int j = 0; j < c->top_k; ++j) {   /* the slices, each with weight 1 */
    st->idx[j] = j;
    st->w[j] = 1.0f;
  }
  free(act);
  free(nq);
  return 0;
}

/* Step 13, the hyper-connection post / expand of the next residual streams:
 * out_i = sum_j comb_ij X_j + post_i y, rounded to the hc element type. */
static void expand(const orc_cfg* c, const double* X, const double* comb, const double* post, const double* y,
                   double* out) {
  const int S = c->hc, H = c->hidden;
  for (int i = 0; i < S; ++i)
    for (int h = 0; h < H; ++h) {
      double acc = 0.0;
      for (int j = 0; j < S; ++j) acc += comb[i * S + j] * X[(int64_t)j * H + h];
      acc += post[i] * y[h];
      out[(int64_t)i * H + h] = c->hc_dtype == ORC_BF16 ? rbf16(acc) : (double)(float)acc;
    }
}

static void state_alloc(const orc_cfg* c, row_state* st) {
  st->a = (double*)calloc((size_t)c->hidden, sizeof(double));
  st->n = (double*)calloc((size_t)c->hidden, sizeof(double));
  st->y = (double*)calloc((size_t)c->hidden, sizeof(double));
  st->logits = (float*)calloc((size_t)c->n_routed, sizeof(float));
  st->score = (float*)calloc((size_t)c->n_routed, sizeof(float));
  st->sel = (float*)calloc((size_t)c->n_routed, sizeof(float));
  st->w = (float*)calloc((size_t)c->top_k, sizeof(float));
  st->idx = (int*)calloc((size_t)c->top_k, sizeof(int));
}

static void state_free(row_state* st) {
  free(st->a);
  free(st->n);
  free(st->y);
  free(st->logits);
  free(st->score);
  free(st->sel);
  free(st->w);
  free(st->idx);
}

static void taps_store(const orc_cfg* c, orc_taps* t, int r, const row_state* st, int upto_y) {
  const int S = c->hc, H = c->hidden, E = c->n_routed, K = c->top_k, M = 2 * c->hc + c->hc * c->hc;
  if (!t) return;
  if (t->rho) t->rho[r] = st->rho;
  if (t->mix) memcpy(t->mix + (int64_t)r * M, st->mix, sizeof(double) * M);
  if (t->pre) memcpy(t->pre + (int64_t)r * S, st->pre, sizeof(double) * S);
  if (t->post) memcpy(t->post + (int64_t)r * S, st->post, sizeof(double) * S);
  if (t->comb) memcpy(t->comb + (int64_t)r * S * S, st->comb, sizeof(double) * S * S);
  if (t->a) memcpy(t->a + (int64_t)r * H, st->a, sizeof(double) * H);
  if (t->n) memcpy(t->n + (int64_t)r * H, st->n, sizeof(double) * H);
  if (t->logits) memcpy(t->logits + (int64_t)r * E, st->logits, sizeof(float) * E);
  if (t->score) memcpy(t->score + (int64_t)r * E, st->score, sizeof(float) * E);
  if (t->sel) memcpy(t->sel + (int64_t)r * E, st->sel, sizeof(float) * E);
  if (t->idx) memcpy(t->idx + (int64_t)r * K, st->idx, sizeof(int) * K);
  if (t->w) memcpy(t->w + (int64_t)r * K, st->w, sizeof(float) * K);
  if (upto_y && t->y) memcpy(t->y + (int64_t)r * H, st->y, sizeof(double) * H);
}

/* steps 1-12 for one row; X is the decoded [S][H] row */
static int row_steps(const orc_cfg* c, const orc_weights* w, const double* X, row_state* st, int route_only) {
  hc_mix_split(c, w, X, st);
  collapse_norm(c, w, X, st);
  if (c->dense) return route_only ? 0 : dense_mlp(c, w, st);
  route(c, w, st);
  if (route_only) return 0;
  return moe(c, w, st);
}

static int run_layer(const orc_cfg* c, const orc_weights* w, const void* hc_in, void* hc_out, orc_taps* t,
                     int route_only) {
  const int S = c->hc, H = c->hidden;
  const int64_t SH = (int64_t)S * H;
  int rc = 0;
  double* X;
  double* out;
  row_state st;
  if (check_cfg(c)) return -1;
  X = (double*)malloc(sizeof(double) * (size_t)SH);
  out = (double*)malloc(sizeof(double) * (size_t)SH);
  state_alloc(c, &st);
  for (int r = 0; r < c->rows && !rc; ++r) {
    for (int64_t i = 0; i < SH; ++i) X[i] = dec_act(hc_in, (int64_t)r * SH + i, c->hc_dtype);
    rc = row_steps(c, w, X, &st, route_only);
    taps_store(c, t, r, &st, !route_only && !rc);
    if (rc || route_only) continue;
    expand(c, X, st.comb, st.post, st.y, out);
    for (int64_t i = 0; i < SH; ++i) enc_act(hc_out, (int64_t)r * SH + i, c->hc_dtype, out[i]);
  }
  state_free(&st);
  free(X);
  free(out);
  return rc;
}

EXPORT int orc_layer(const orc_cfg* cfg, const orc_weights* w, const void* hc_in, void* hc_out, orc_taps* taps) {
  return run_layer(cfg, w, hc_in, hc_out, taps, 0);
}

EXPORT int orc_route(const orc_cfg* cfg, const orc_weights* w, const void* hc_in, orc_taps* taps) {
  return run_layer(cfg, w, hc_in, NULL, taps, 1);
}

/* ---------------------------------------------------------------- chains -- */

EXPORT int orc_chain(const orc_cfg* c, int n_layers, const orc_weights* w, const void* hc_in, void* hc_out,
                     int deferred) {
  const int S = c->hc, H = c->hidden, M = 2 * c->hc + c->hc * c->hc;
  const int64_t SH = (int64_t)S * H;
  int rc = 0;
  double* X = (double*)malloc(sizeof(double) * (size_t)SH);
  double* Xn = (double*)malloc(sizeof(double) * (size_t)SH);
  row_state st;
  if (check_cfg(c) || n_layers < 1) {
    free(X);
    free(Xn);
    return -1;
  }
  state_alloc(c, &st);
  for (int r = 0; r < c->rows && !rc; ++r) {
    for (int64_t i = 0; i < SH; ++i) X[i] = dec_act(hc_in, (int64_t)r * SH + i, c->hc_dtype);
    if (!deferred) {
      /* op by op: each layer closes its own expand before the next starts */
      for (int l = 0; l < n_layers && !rc; ++l) {
        rc = row_steps(c, w + l, X, &st, 0);
        if (rc) break;
        expand(c, X, st.comb, st.post, st.y, Xn);
        memcpy(X, Xn, sizeof(double) * (size_t)SH);
      }
    } else {
      /* deferred post: layer l leaves (comb, post, y) pending; layer l+1
       * opens with that expand, materialising its residual streams and, in
       * the same pass over (s, h), its square sum and mix products; the
       * finalisation then scales by rho as in the unfused mix. */
      double pcomb[64], ppost[8];
      double* py = (double*)malloc(sizeof(double) * (size_t)H);
      rc = row_steps(c, w, X, &st, 0);
      for (int l = 1; l < n_layers && !rc; ++l) {
        double ss = 0.0, acc[64];
        memcpy(pcomb, st.comb, sizeof(pcomb));
        memcpy(ppost, st.post, sizeof(ppost));
        memcpy(py, st.y, sizeof(double) * (size_t)H);
        expand(c, X, pcomb, ppost, py, Xn);
        memcpy(X, Xn, sizeof(double) * (size_t)SH);
        for (int64_t i = 0; i < SH; ++i) ss += X[i] * X[i];
        for (int col = 0; col < M; ++col) {
          acc[col] = 0.0;
          for (int64_t i = 0; i < SH; ++i) acc[col] += X[i] * (double)w[l].mix_w[i * M + col];
        }
        st.rho = 1.0 / sqrt(ss / (double)SH + c->rms_eps);
        for (int col = 0; col < M; ++col) st.mix[col] = st.rho * acc[col];
        for (int i = 0; i < S; ++i) {
          st.pre[i] = sigmoid(st.mix[i]) + c->pre_eps;
          st.post[i] = c->post_mult * sigmoid(st.mix[S + i]);
        }
        orc_sinkhorn(st.mix + 2 * S, S, c->sinkhorn_iters, st.comb);
        collapse_norm(c, w + l, X, &st);
        if (c->dense) {
          rc = dense_mlp(c, w + l, &st);
        } else {
          route(c, w + l, &st);
          rc = moe(c, w + l, &st);
        }
      }
      if (!rc) {
        /* the last layer's expand, closed at the tail */
        expand(c, X, st.comb, st.post, st.y, Xn);
        memcpy(X, Xn, sizeof(double) * (size_t)SH);
      }
      free(py);
    }
    if (!rc)
      for (int64_t i = 0; i < SH; ++i) enc_act(hc_out, (int64_t)r * SH + i, c->hc_dtype, X[i]);
  }
  state_free(&st);
  free(X);
  free(Xn);
  return rc;
}

/* ------------------------------------------------- within-layer boundary -- */

/* The attention sublayer's output closed into this FFN's opening pass:
 * X_i = sum_j attn_comb_ij Xa_j + attn_post_i y_attn, rounded to the hc
 * element type (the attention sublayer's own post / expand), then this
 * layer's steps 1-13 on X.  Written in the fused form: the expand and, in the
 * same pass over (s, h), the square sum and the mix products; the mix is then
 * scaled by rho as in the unfused mix (SGLang "[DeepSeek-V4] Add
 * mhc_fused_post_pre kernel", Modifications: the attention's hc_post fused
 * with the FFN's hc_pre inside one layer).  x_attn [R][S][H] and y_attn [R][H]
 * in hc_dtype, attn_post [R][S] and attn_comb [R][S][S] fp32.  x_out, when
 * not NULL, receives the materialised X [R][S][H] in hc_dtype. */
EXPORT int orc_layer_pending(const orc_cfg* c, const orc_weights* w, const void* x_attn, const float* attn_post,
                             const float* attn_comb, const void* y_attn, void* hc_out, void* x_out, orc_taps* t) {
  const int S = c->hc, H = c->hidden, M = 2 * c->hc + c->hc * c->hc;
  const int64_t SH = (int64_t)S * H;
  int rc = 0;
  double* Xa;
  double* X;
  double* y;
  double* out;
  row_state st;
  if (check_cfg(c) || S > 8) return -1;
  Xa = (double*)malloc(sizeof(double) * (size_t)SH);
  X = (double*)malloc(sizeof(double) * (size_t)SH);
  out = (double*)malloc(sizeof(double) * (size_t)SH);
  y = (double*)malloc(sizeof(double) * (size_t)H);
  state_alloc(c, &st);
  for (int r = 0; r < c->rows && !rc; ++r) {
    double pcomb[64], ppost[8], ss = 0.0, acc[64];
    for (int64_t i = 0; i < SH; ++i) Xa[i] = dec_act(x_attn, (int64_t)r * SH + i, c->hc_dtype);
    for (int h = 0; h < H; ++h) y[h] = dec_act(y_attn, (int64_t)r * H + h, c->hc_dtype);
    for (int i = 0; i < S * S; ++i) pcomb[i] = attn_comb[(int64_t)r * S * S + i];
    for (int i = 0; i < S; ++i) ppost[i] = attn_post[(int64_t)r * S + i];
    expand(c, Xa, pcomb, ppost, y, X);
    for (int64_t i = 0; i < SH; ++i) ss += X[i] * X[i];
    for (int col = 0; col < M; ++col) {
      acc[col] = 0.0;
      for (int64_t i = 0; i < SH; ++i) acc[col] += X[i] * (double)w->mix_w[i * M + col];
    }
    st.rho = 1.0 / sqrt(ss / (double)SH + c->rms_eps);
    for (int col = 0; col < M; ++col) st.mix[col] = st.rho * acc[col];
    for (int i = 0; i < S; ++i) {
      st.pre[i] = sigmoid(st.mix[i]) + c->pre_eps;
      st.post[i] = c->post_mult * sigmoid(st.mix[S + i]);
    }
    orc_sinkhorn(st.mix + 2 * S, S, c->sinkhorn_iters, st.comb);
    collapse_norm(c, w, X, &st);
    if (c->dense) {
      rc = dense_mlp(c, w, &st);
    } else {
      route(c, w, &st);
      rc = moe(c, w, &st);
    }
    taps_store(c, t, r, &st, !rc);
    if (rc) break;
    if (x_out)
      for (int64_t i = 0; i < SH; ++i) enc_act(x_out, (int64_t)r * SH + i, c->hc_dtype, X[i]);
    expand(c, X, st.comb, st.post, st.y, out);
    for (int64_t i = 0; i < SH; ++i) enc_act(hc_out, (int64_t)r * SH + i, c->hc_dtype, out[i]);
  }
  state_free(&st);
  free(Xa);
  free(X);
  free(out);
  free(y);
  return rc;
}

/* The expand alone, per row: x_out_i = sum_j comb_ij x_in_j + post_i y,
 * rounded to the hc element type (the op-by-op form of a sublayer's post). */
EXPORT int orc_expand(const orc_cfg* c, const void* x_in, const float* post, const float* comb, const void* y,
                      void* x_out) {
  const int S = c->hc, H = c->hidden;
  const int64_t SH = (int64_t)S * H;
  double* Xa;
  double* X;
  double* yy;
  if (check_cfg(c) || S > 8) return -1;
  Xa = (double*)malloc(sizeof(double) * (size_t)SH);
  X = (double*)malloc(sizeof(double) * (size_t)SH);
  yy = (double*)malloc(sizeof(double) * (size_t)H);
  for (int r = 0; r < c->rows; ++r) {
    double pc[64], pp[8];
    for (int64_t i = 0; i < SH; ++i) Xa[i] = dec_act(x_in, (int64_t)r * SH + i, c->hc_dtype);
    for (int h = 0; h < H; ++h) yy[h] = dec_act(y, (int64_t)r * H + h, c->hc_dtype);
    for (int i = 0; i < S * S; ++i) pc[i] = comb[(int64_t)r * S * S + i];
    for (int i = 0; i < S; ++i) pp[i] = post[(int64_t)r * S + i];
    expand(c, Xa, pc, pp, yy, X);
    for (int64_t i = 0; i < SH; ++i) enc_act(x_out, (int64_t)r * SH + i, c->hc_dtype, X[i]);
  }
  free(Xa);
  free(X);
  free(yy);
  return 0;
}
