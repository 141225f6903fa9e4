/*
 * moe_oracle.c -- plain CPU oracle of one sparse Mixture-of-Experts layer
 * forward over 4-bit block-quantised experts.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header, table or helper with
 * the CUDA library.
 *
 * Precision: values are stored as the checkpoint gives them (bf16 activations,
 * fp32 router, FP4 codes + block scales); every dot product and sum is
 * accumulated in fp64 and rounded to fp32 only at the step boundaries named
 * below, so the comparison tolerance budgets GPU error alone.  Built without
 * -ffast-math and with -ffp-contract=off.
 *
 * Sources (pages of the Strata reference set):
 *  - "ro99/strata" (C++20/CUDA engine), bullet "MXFP4 is read as MXFP4": two
 *    E2M1 codes per byte, one E8M0 exponent per group of 32;
 *  - same page, bullet "Scales are admitted, not clamped": E8M0 is placed in a
 *    BF16 exponent field, so codes 0 and 255 (+0 and +inf) fail admission;
 *  - same page, list of rules: precision, routing, expert count and top-k come
 *    from the checkpoint; exact mode completes or fails;
 *  - strata.amperor.ai (fit list legend): paged output is bit-identical to the
 *    resident model;
 *  - "Strata, Explained" section 2: shared experts are always on.
 * The pages never write the layer's formulas.  The readings used where they
 * are silent (softmax routing with renormalised top-k gates, SwiGLU
 * h = silu(gate) * up, low nibble = even element, groups along the input
 * dimension, E4M3 + fp32 per-tensor NVFP4 scales, A4 activation quantisation)
 * are the plainest ones and are listed with the design notes.
 *
 * Parity pins: every function here is checked by tests that do not re-use its
 * code (closed-form value tables, library routines, brute force on tiny
 * inputs, invariants).  The A4 activation quantisers are pinned by brute-force
 * nearest-code search and hand-built blocks.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_FMT_MXFP4 0
#define ORC_FMT_NVFP4 1
/* Other expert formats of at least four bits that checkpoints ship
 * ("ro99/strata", model table: "INT4 group-128, W4A16" and "FP8 E4M3
 * block-128 with F32 inverse scales"):
 *  INT4G128: codes [rows, K/2], two signed 4-bit integers per byte (even
 *            element in the low nibble, two's complement, -8..7), one bf16
 *            scale per row and group of 128 along K: scales [rows, K/128]
 *            (uint16 bf16 bits); w = q * scale;
 *  FP8B128:  codes [rows, K], one E4M3 byte per weight, one fp32 inverse
 *            scale per block of 128 rows x 128 columns: scales [rows/128,
 *            K/128] (fp32); w = e4m3(q) * scale. */
#define ORC_FMT_INT4G128 2
#define ORC_FMT_FP8B128 3
#define ORC_EXACT 0
#define ORC_A4 1
#define ORC_SOFTMAX 0
#define ORC_SIGMOID 1

/* Router variants (what a checkpoint may declare; "ro99/strata", rules list:
 * routing, expert count and top-k come from the checkpoint, and its model
 * table: "256 experts + 2 sinks", "256 experts + 1 shared").  The routing
 * targets are the E experts followed by n_sinks sink targets: a sink takes part
 * in scoring, top-k and renormalisation like an expert but has no FFN, so
 * choosing it contributes nothing to y.  scoring: softmax over all targets, or
 * an independent sigmoid per target; renorm: the k chosen scores divided by
 * their sum, or used as they are.  shared_gate_w (optional): the shared expert
 * is scaled by sigmoid(x . shared_gate_w) instead of weight 1. */
typedef struct {
  int H, I, E, k, Is;
  int fmt;                       /* ORC_FMT_* */
  int numerics;                  /* ORC_EXACT or ORC_A4 */
  const float *router_w;         /* [E + n_sinks, H] */
  const float *router_bias;      /* [E + n_sinks] or NULL */
  const uint8_t *codes[3];       /* [E, rows, K/2]: gate [I,H], up [I,H], down [H,I] */
  const uint8_t *scales[3];      /* [E, rows, K/G] */
  const float *global_scale;     /* [E, 3] (NVFP4) or NULL */
  const uint16_t *shared_w[3];   /* bf16: [Is,H], [Is,H], [H,Is]; NULL if Is == 0 */
  int scoring;                   /* ORC_SOFTMAX or ORC_SIGMOID */
  int renorm;                    /* 1: chosen scores renormalised to sum to 1 */
  int n_sinks;                   /* sink targets after the E experts */
  const float *shared_gate_w;    /* [H] or NULL */
} orc_layer_t;

/* ------------------------------------------------------------------------ */
/* O1: format decode                                                         */
/* ------------------------------------------------------------------------ */

/* E2M1: sign bit, 2 exponent bits (bias 1), 1 mantissa bit; exponent 0 is
 * subnormal (0 or 0.5).  Values {0, .5, 1, 1.5, 2, 3, 4, 6} and negatives. */
double orc_e2m1(unsigned code) {
  unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u, m = code & 1u;
  double mag = (e == 0) ? 0.5 * (double)m : ldexp(1.0 + 0.5 * (double)m, (int)e - 1);
  return s ? -mag : mag;
}

/* E8M0: a bare biased exponent, value 2^(code - 127).  Admission rejects 0 and
 * 255, which a BF16 exponent field would turn into +0 and +inf. */
double orc_e8m0(unsigned code) { return ldexp(1.0, (int)code - 127); }

/* E4M3 (finite variant): bias 7, 3 mantissa bits, exponent 0 subnormal,
 * S.1111.111 is NaN, no infinities. */
double orc_e4m3(unsigned code) {
  unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexp((double)m / 8.0, -6);
  else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
  return s ? -mag : mag;
}

double orc_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Admission: index of the first rejected scale code, or -1.
 * MXFP4: E8M0 codes 0 and 255 are rejected.  NVFP4: E4M3 NaN codes and codes
 * with the sign bit set are rejected (a block scale is a magnitude).  INT4G128
 * (bf16 scales, n = number of scales): NaN and infinite scales are rejected.
 * FP8B128 (fp32 scales): NaN, infinite, zero and negative scales. */
long orc_admit_scales(int fmt, const uint8_t *s, long n) {
  for (long i = 0; i < n; ++i) {
    if (fmt == ORC_FMT_INT4G128) {
      uint16_t b;
      memcpy(&b, s + 2 * i, 2);
      if ((b & 0x7F80u) == 0x7F80u) return i;
      continue;
    }
    if (fmt == ORC_FMT_FP8B128) {
      float f;
      memcpy(&f, s + 4 * i, 4);
      if (!(f > 0.0f) || isinf(f)) return i;
      continue;
    }
    unsigned c = s[i];
    if (fmt == ORC_FMT_MXFP4) {
      if (c == 0u || c == 255u) return i;
    } else {
      if ((c & 0x7Fu) == 0x7Fu || (c & 0x80u)) return i;
    }
  }
  return -1;
}

/* FP8B128 weights: E4M3 NaN codes (S.1111.111) are rejected; index or -1. */
long orc_admit_fp8_codes(const uint8_t *q, long n) {
  for (long i = 0; i < n; ++i)
    if ((q[i] & 0x7Fu) == 0x7Fu) return i;
  return -1;
}

static void mat_shape(const orc_layer_t *L, int m, int *rows, int *K) {
  if (m == 2) { *rows = L->H; *K = L->I; }
  else { *rows = L->I; *K = L->H; }
}

static int group_of(const orc_layer_t *L) { return L->fmt == ORC_FMT_MXFP4 ? 32 : 16; }

/* INT4: a nibble as a two's complement integer in -8..7. */
double orc_int4(unsigned nib) { return (double)((int)(nib & 15u) - ((nib & 8u) ? 16 : 0)); }

/* Decode row r of matrix m of expert e into out[K] (fp64, exact). */
void orc_dequant_row(const orc_layer_t *L, int m, int e, int r, double *out) {
  int rows, K;
  mat_shape(L, m, &rows, &K);
  if (L->fmt == ORC_FMT_INT4G128) {
    const uint8_t *codes = L->codes[m] + ((size_t)e * rows + r) * (size_t)(K / 2);
    const uint8_t *sc = L->scales[m] + ((size_t)e * rows + r) * (size_t)(K / 128) * 2;
    for (int c = 0; c < K; ++c) {
      uint8_t byte = codes[c / 2];
      unsigned nib = (c % 2 == 0) ? (byte & 15u) : (byte >> 4);
      uint16_t sb;
      memcpy(&sb, sc + 2 * (c / 128), 2);
      out[c] = orc_int4(nib) * orc_bf16(sb);
    }
    return;
  }
  if (L->fmt == ORC_FMT_FP8B128) {
    const uint8_t *codes = L->codes[m] + ((size_t)e * rows + r) * (size_t)K;
    const uint8_t *sc = L->scales[m] + ((size_t)e * (rows / 128) + r / 128) * (size_t)(K / 128) * 4;
    for (int c = 0; c < K; ++c) {
      float s;
      memcpy(&s, sc + 4 * (c / 128), 4);
      out[c] = orc_e4m3(codes[c]) * (double)s;
    }
    return;
  }
  const int G = group_of(L);
  const uint8_t *codes = L->codes[m] + ((size_t)e * rows + r) * (size_t)(K / 2);
  const uint8_t *sc = L->scales[m] + ((size_t)e * rows + r) * (size_t)(K / G);
  double gscale = (L->fmt == ORC_FMT_NVFP4) ? (double)L->global_scale[e * 3 + m] : 1.0;
  for (int c = 0; c < K; ++c) {
    uint8_t byte = codes[c / 2];
    unsigned code = (c % 2 == 0) ? (byte & 15u) : (byte >> 4);
    double s = (L->fmt == ORC_FMT_MXFP4) ? orc_e8m0(sc[c / G]) : orc_e4m3(sc[c / G]) * gscale;
    out[c] = orc_e2m1(code) * s;
  }
}

/* ------------------------------------------------------------------------ */
/* A4 activation quantisers (opt-in numerics mode)                           */
/* ------------------------------------------------------------------------ */

/* Round a float to the nearest E2M1 value, ties to the code with an even
 * mantissa bit, saturating at +-6.  Returns the 4-bit code. */
unsigned orc_rne_e2m1(float q) {
  static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  unsigned s = signbit(q) ? 8u : 0u;
  float a = fabsf(q);
  if (isnan(a) || a >= 6.0f) return s | 7u;     /* saturate */
  unsigned best = 0;
  for (unsigned c = 1; c < 8; ++c) {
    double db = fabs((double)a - (double)mag[best]), dc = fabs((double)a - (double)mag[c]);
    if (dc < db || (dc == db && (c & 1u) == 0u)) best = c;
  }
  return s | best;
}

/* Round a non-negative float to the nearest E4M3 value (ties to even mantissa),
 * saturating at 448.  Returns the 8-bit code. */
unsigned orc_rn_e4m3(float t) {
  if (!(t > 0.0f)) return 0u;
  double a = (double)t;
  unsigned best = 0;
  double bd = a;
  for (unsigned c = 1; c < 0x7F; ++c) {          /* all finite positive codes */
    double v = orc_e4m3(c);
    double d = fabs(a - v);
    if (d < bd || (d == bd && (c & 1u) == 0u)) { bd = d; best = c; }
  }
  return best;
}

/* OCP MX rule for one block of n values (n = 32): shared exponent
 * X = floor(log2(amax)) - 2 (2 = largest E2M1 exponent), stored as E8M0 code
 * clamp(X + 127, 1, 254) (1 when amax = 0); element code = RNE(v / 2^X). */
void orc_quant_mx_block(const float *v, int n, uint8_t *codes, uint8_t *scale) {
  float amax = 0.0f;
  for (int i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(v[i]));
  int code = 1;
  if (amax > 0.0f) {
    int ex;
    frexpf(amax, &ex);                /* amax = f * 2^ex, f in [0.5, 1) */
    code = (ex - 1) - 2 + 127;
    if (code < 1) code = 1;
    if (code > 254) code = 254;
  }
  *scale = (uint8_t)code;
  float inv = ldexpf(1.0f, 127 - code);    /* exact power of two */
  for (int i = 0; i < n; ++i) codes[i] = (uint8_t)orc_rne_e2m1(v[i] * inv);
}

/* NVFP4 activation rule for one row of K values (blocks of 16):
 *   G = 2^ceil(log2(amax_row / (6 * 448)))   (1 when amax_row = 0)
 *   block scale code  = RN_E4M3((amax_block / 6) / G)
 *   element code      = RNE_E2M1(v * (1 / (scale * G)))   (0 when scale = 0)
 * All steps in fp32, in this order, so that the same decisions are taken as
 * in the GPU kernel. */
void orc_quant_nv_row(const float *v, int K, uint8_t *codes, uint8_t *scales, float *G_out) {
  float amax = 0.0f;
  for (int i = 0; i < K; ++i) amax = fmaxf(amax, fabsf(v[i]));
  float G = 1.0f;
  if (amax > 0.0f) {
    double r = (double)amax / (6.0 * 448.0);
    int ex;
    double f = frexp(r, &ex);          /* r = f * 2^ex, f in [0.5,1) */
    int c = (f == 0.5) ? ex - 1 : ex;  /* ceil(log2(r)) */
    G = ldexpf(1.0f, c);
  }
  *G_out = G;
  for (int b = 0; b < K / 16; ++b) {
    float bmax = 0.0f;
    for (int i = 0; i < 16; ++i) bmax = fmaxf(bmax, fabsf(v[b * 16 + i]));
    float t = (bmax / 6.0f) / G;
    unsigned sc = orc_rn_e4m3(t);
    scales[b] = (uint8_t)sc;
    float denom = (float)orc_e4m3(sc) * G;
    for (int i = 0; i < 16; ++i) {
      if (sc == 0u) { codes[b * 16 + i] = 0; continue; }
      float inv = 1.0f / denom;
      codes[b * 16 + i] = (uint8_t)orc_rne_e2m1(v[b * 16 + i] * inv);
    }
  }
}

/* Quantise-dequantise one activation row per the A4 rule of the layer's format:
 * MXFP4 out[i] = e2m1(code_i) * 2^(scale_{i/32} - 127); NVFP4
 * out[i] = e2m1(code_i) * e4m3(scale_{i/16}) * G (per-row G, rule above). */
void orc_a4_qdq_row(int fmt, const float *v, int K, double *out) {
  uint8_t *codes = (uint8_t *)malloc((size_t)K);
  if (fmt == ORC_FMT_MXFP4) {
    uint8_t sc;
    for (int b = 0; b < K / 32; ++b) {
      orc_quant_mx_block(v + b * 32, 32, codes + b * 32, &sc);
      for (int i = 0; i < 32; ++i) out[b * 32 + i] = orc_e2m1(codes[b * 32 + i]) * orc_e8m0(sc);
    }
  } else {
    uint8_t *sc = (uint8_t *)malloc((size_t)(K / 16));
    float G;
    orc_quant_nv_row(v, K, codes, sc, &G);
    for (int i = 0; i < K; ++i) out[i] = orc_e2m1(codes[i]) * orc_e4m3(sc[i / 16]) * (double)G;
    free(sc);
  }
  free(codes);
}

/* ------------------------------------------------------------------------ */
/* O2: router logits   l[t,e] = fp32( sum_h x[t,h] * W_r[e,h] + b[e] )      */
/* ------------------------------------------------------------------------ */
/* The logits of all E + n_sinks routing targets (experts first, then sinks). */
void orc_router_logits_row(const orc_layer_t *L, const uint16_t *xt, float *lt) {
  for (int e = 0; e < L->E + L->n_sinks; ++e) {
    double acc = 0.0;
    const float *w = L->router_w + (size_t)e * L->H;
    for (int h = 0; h < L->H; ++h) acc += orc_bf16(xt[h]) * (double)w[h];
    if (L->router_bias) acc += (double)L->router_bias[e];
    lt[e] = (float)acc;
  }
}

/* Shared-expert gate logit fp32( sum_h x[t,h] * w_sg[h] ) (0 without a gate). */
float orc_shared_gate_logit(const orc_layer_t *L, const uint16_t *xt) {
  if (!L->shared_gate_w) return 0.0f;
  double acc = 0.0;
  for (int h = 0; h < L->H; ++h) acc += orc_bf16(xt[h]) * (double)L->shared_gate_w[h];
  return (float)acc;
}

/* ------------------------------------------------------------------------ */
/* O3: routing over n targets.  ids = the k targets of largest logit, in     */
/* descending order, the lower index first on ties (both scorings are        */
/* monotone in the logit, so the order is the logits' order).  Scores, fp64: */
/*   softmax: s_j = exp(l_j - l_max) / sum_{all n targets} exp(l_e - l_max)  */
/*   sigmoid: s_j = 1 / (1 + exp(-l_j))                                      */
/* gates = s_j / sum_{i in top-k} s_i when renormalised, else s_j; rounded   */
/* to fp32.  (Softmax renormalised equals exp(l_j - l_max) over the chosen   */
/* k's sum.)                                                                 */
/* ------------------------------------------------------------------------ */
void orc_route_row_v(const float *lt, int n, int k, int scoring, int renorm, int32_t *ids, float *gates) {
  char *taken = (char *)calloc((size_t)n, 1);
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < n; ++e)
      if (!taken[e] && (best < 0 || lt[e] > lt[best])) best = e;
    taken[best] = 1;
    ids[j] = best;
  }
  free(taken);
  double s[64];
  const double lmax = (double)lt[ids[0]];
  double all = 0.0;
  if (scoring == ORC_SOFTMAX && !renorm)
    for (int e = 0; e < n; ++e) all += exp((double)lt[e] - lmax);
  for (int j = 0; j < k; ++j) {
    const double l = (double)lt[ids[j]];
    if (scoring == ORC_SOFTMAX) s[j] = renorm ? exp(l - lmax) : exp(l - lmax) / all;
    else s[j] = 1.0 / (1.0 + exp(-l));
  }
  double den = 0.0;
  for (int j = 0; j < k; ++j) den += s[j];
  for (int j = 0; j < k; ++j) gates[j] = (float)(renorm ? s[j] / den : s[j]);
}

/* The default routing: softmax over all E renormalised to the chosen k,
 * i.e. exp(l_j - l_max) / sum_{i in top-k} exp(l_i - l_max). */
void orc_route_row(const float *lt, int E, int k, int32_t *ids, float *gates) {
  orc_route_row_v(lt, E, k, ORC_SOFTMAX, 1, ids, gates);
}

/* ------------------------------------------------------------------------ */
/* O4: permutation.  Pair index p = t*k + j; stable counting sort of p by    */
/* ids[p]: counts, exclusive offsets (E+1), perm (sorted position -> p) and  */
/* inv (p -> sorted position).                                               */
/* ------------------------------------------------------------------------ */
void orc_permute(const int32_t *ids, int n_pairs, int E, int32_t *counts, int32_t *offsets,
                 int32_t *perm, int32_t *inv) {
  memset(counts, 0, sizeof(int32_t) * (size_t)E);
  for (int p = 0; p < n_pairs; ++p) counts[ids[p]]++;
  offsets[0] = 0;
  for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
  int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
  memcpy(cursor, offsets, sizeof(int32_t) * (size_t)E);
  for (int p = 0; p < n_pairs; ++p) {
    int pos = cursor[ids[p]]++;
    perm[pos] = p;
    inv[p] = pos;
  }
  free(cursor);
}

/* ------------------------------------------------------------------------ */
/* O5: one routed expert on one token (SwiGLU).                               */
/*   a_i = fp32(sum_c Wg[i,c] x_c),  u_i = fp32(sum_c Wu[i,c] x_c)            */
/*   h_i = fp32(silu(a_i) * u_i),    silu(a) = a / (1 + exp(-a))              */
/*   o_r = sum_i Wd[r,i] h_i          (kept in fp64)                          */
/* A4 mode quantises x before gate/up and h before down (per-row rules).      */
/* ------------------------------------------------------------------------ */
static double silu(double a) { return a / (1.0 + exp(-a)); }

void orc_expert_token(const orc_layer_t *L, int e, const double *xt, double *o) {
  const int H = L->H, I = L->I;
  const int K = H > I ? H : I;
  double *row = (double *)malloc(sizeof(double) * (size_t)K);
  double *xin = (double *)malloc(sizeof(double) * (size_t)H);
  double *hin = (double *)malloc(sizeof(double) * (size_t)I);
  float *h = (float *)malloc(sizeof(float) * (size_t)I);
  if (L->numerics == ORC_A4) {
    float *xf = (float *)malloc(sizeof(float) * (size_t)H);
    for (int c = 0; c < H; ++c) xf[c] = (float)xt[c];
    orc_a4_qdq_row(L->fmt, xf, H, xin);
    free(xf);
  } else {
    memcpy(xin, xt, sizeof(double) * (size_t)H);
  }
  for (int i = 0; i < I; ++i) {
    double a = 0.0, u = 0.0;
    orc_dequant_row(L, 0, e, i, row);
    for (int c = 0; c < H; ++c) a += row[c] * xin[c];
    orc_dequant_row(L, 1, e, i, row);
    for (int c = 0; c < H; ++c) u += row[c] * xin[c];
    float af = (float)a, uf = (float)u;
    h[i] = (float)(silu((double)af) * (double)uf);
  }
  if (L->numerics == ORC_A4) orc_a4_qdq_row(L->fmt, h, I, hin);
  else for (int i = 0; i < I; ++i) hin[i] = (double)h[i];
  for (int r = 0; r < H; ++r) {
    double acc = 0.0;
    orc_dequant_row(L, 2, e, r, row);
    for (int i = 0; i < I; ++i) acc += row[i] * hin[i];
    o[r] = acc;
  }
  free(row); free(xin); free(hin); free(h);
}

/* Timing sample for the benchmark's CPU leg (EXACT mode only): the formula of
 * orc_expert_token restricted to intermediate rows [i0, i0+n): h_i for those
 * rows and their terms Wd[r,i] * h_i added, in i order, into o[H]. */
void orc_expert_rows(const orc_layer_t *L, int e, const double *xt, int i0, int n, double *o) {
  const int H = L->H, I = L->I;
  const int K = H > I ? H : I;
  double *row = (double *)malloc(sizeof(double) * (size_t)K);
  double *dcol = (double *)malloc(sizeof(double) * (size_t)I);
  float *h = (float *)malloc(sizeof(float) * (size_t)n);
  for (int i = i0; i < i0 + n; ++i) {
    double a = 0.0, u = 0.0;
    orc_dequant_row(L, 0, e, i, row);
    for (int c = 0; c < H; ++c) a += row[c] * xt[c];
    orc_dequant_row(L, 1, e, i, row);
    for (int c = 0; c < H; ++c) u += row[c] * xt[c];
    float af = (float)a, uf = (float)u;
    h[i - i0] = (float)(silu((double)af) * (double)uf);
  }
  for (int r = 0; r < H; ++r) {
    orc_dequant_row(L, 2, e, r, dcol);
    double acc = o[r];
    for (int i = i0; i < i0 + n; ++i) acc += dcol[i] * (double)h[i - i0];
    o[r] = acc;
  }
  free(row); free(dcol); free(h);
}

/* Shared expert on one token: the same SwiGLU with bf16 weights, weight 1. */
void orc_shared_token(const orc_layer_t *L, const double *xt, double *s) {
  const int H = L->H, Is = L->Is;
  float *h = (float *)malloc(sizeof(float) * (size_t)Is);
  for (int i = 0; i < Is; ++i) {
    double a = 0.0, u = 0.0;
    const uint16_t *wg = L->shared_w[0] + (size_t)i * H;
    const uint16_t *wu = L->shared_w[1] + (size_t)i * H;
    for (int c = 0; c < H; ++c) { a += orc_bf16(wg[c]) * xt[c]; u += orc_bf16(wu[c]) * xt[c]; }
    float af = (float)a, uf = (float)u;
    h[i] = (float)(silu((double)af) * (double)uf);
  }
  for (int r = 0; r < H; ++r) {
    double acc = 0.0;
    const uint16_t *wd = L->shared_w[2] + (size_t)r * Is;
    for (int i = 0; i < Is; ++i) acc += orc_bf16(wd[i]) * (double)h[i];
    s[r] = acc;
  }
  free(h);
}

/* ------------------------------------------------------------------------ */
/* O6: the layer.  For every listed token t:                                  */
/*   y[t] = fp32( sum_{j<k, ids_j < E} g_j * o_{ids_j}(x_t)  + gs * s(x_t) ) */
/* the routed terms added in j order (a chosen sink adds nothing), then the   */
/* shared expert, with gs = 1, or sigmoid(shared-gate logit) (fp64) when the  */
/* layer has a shared-expert gate.                                            */
/* rows: token indices to evaluate (NULL = all T); outputs are per listed row.*/
/* logits [n, E + n_sinks], ids [n,k], gates [n,k] may be NULL.               */
/* ------------------------------------------------------------------------ */
int orc_forward(const orc_layer_t *L, const uint16_t *x, int T, const int32_t *rows, int n_rows,
                float *y, float *logits, int32_t *ids, float *gates, int n_threads) {
  const int H = L->H, E = L->E + L->n_sinks, k = L->k;
  const int n = rows ? n_rows : T;
  if (L->Is > 0 && !L->shared_w[0]) return -1;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
  for (int r = 0; r < n; ++r) {
    int t = rows ? rows[r] : r;
    if (t < 0 || t >= T) { bad = 1; continue; }
    const uint16_t *xt16 = x + (size_t)t * H;
    float *lt = (float *)malloc(sizeof(float) * (size_t)E);
    int32_t *it = (int32_t *)malloc(sizeof(int32_t) * (size_t)k);
    float *gt = (float *)malloc(sizeof(float) * (size_t)k);
    double *xt = (double *)malloc(sizeof(double) * (size_t)H);
    double *o = (double *)malloc(sizeof(double) * (size_t)H);
    double *acc = (double *)calloc((size_t)H, sizeof(double));
    for (int c = 0; c < H; ++c) xt[c] = orc_bf16(xt16[c]);
    orc_router_logits_row(L, xt16, lt);
    orc_route_row_v(lt, E, k, L->scoring, L->renorm, it, gt);
    for (int j = 0; j < k; ++j) {
      if (it[j] >= L->E) continue;                 /* a sink: no FFN */
      orc_expert_token(L, it[j], xt, o);
      for (int c = 0; c < H; ++c) acc[c] += (double)gt[j] * o[c];
    }
    if (L->Is > 0) {
      const double gs = L->shared_gate_w ? 1.0 / (1.0 + exp(-(double)orc_shared_gate_logit(L, xt16))) : 1.0;
      orc_shared_token(L, xt, o);
      for (int c = 0; c < H; ++c) acc[c] += gs * o[c];
    }
    for (int c = 0; c < H; ++c) y[(size_t)r * H + c] = (float)acc[c];
    if (logits) memcpy(logits + (size_t)r * E, lt, sizeof(float) * (size_t)E);
    if (ids) memcpy(ids + (size_t)r * k, it, sizeof(int32_t) * (size_t)k);
    if (gates) memcpy(gates + (size_t)r * k, gt, sizeof(float) * (size_t)k);
    free(lt); free(it); free(gt); free(xt); free(o); free(acc);
  }
  return bad ? -2 : 0;
}

/* Router only (logits, ids, gates) for every token; cheap enough for full T. */
void orc_route_all(const orc_layer_t *L, const uint16_t *x, int T, float *logits, int32_t *ids,
                   float *gates, int n_threads) {
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#else
  (void)n_threads;
#endif
  const int n = L->E + L->n_sinks;
#pragma omp parallel for schedule(static)
  for (int t = 0; t < T; ++t) {
    orc_router_logits_row(L, x + (size_t)t * L->H, logits + (size_t)t * n);
    orc_route_row_v(logits + (size_t)t * n, n, L->k, L->scoring, L->renorm, ids + (size_t)t * L->k,
                    gates + (size_t)t * L->k);
  }
}

int orc_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
