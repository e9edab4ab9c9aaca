/*
 * CPU oracle for the Step-5 routed Mixture-of-Experts feed-forward layer.
 *
 * TEST INFRASTRUCTURE ONLY. The tests, the package's smoke check and the
 * benchmark's CPU-baseline leg may call this; the GPU product path never does.
 * It shares no code with the CUDA library.
 *
 * Plain, slow and obviously correct: one token at a time, no blocking, sums in
 * double precision in ascending index order. What the layer computes:
 *
 *   Layer geometry -- NeMo AutoModel "Step-5-Preview" page, "Model Architecture"
 *   table: hidden 4,096; 352 routed experts per MoE layer with top-8 routing and
 *   one shared expert; expert intermediate size 1,536 for routed and shared
 *   experts; the parameter count "includes the learned router".
 *
 *   Expert storage -- StepFun "Step-5 minimal inference" README, opening section
 *   and the expert-storage paragraph before "Install": experts are BF16, or FP8
 *   E4M3 with block scales ("block-scaled FP8 expert GEMM"). A third storage,
 *   NVFP4 (TensorFold PR page: E2M1 codes, an E4M3 scale per 16 inputs and an
 *   fp32 global scale, read by W4A16 linears), is a variant the pages describe
 *   for another model; it keeps the BF16 activations.
 *
 *   Accumulation -- same README, "Long-output stability": partial results are
 *   added in a fixed order with FP32 (here: at least FP32) accumulation.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   router: logits l = x . Wr^T (+ optional per-expert bias b); softmax over all
 *     experts; the k largest logits are chosen (ties to the lower expert index),
 *     ordered by descending logit; gates are the chosen softmax probabilities
 *     renormalised to sum 1; no extra scaling factor.
 *   experts: SwiGLU, h = silu(x W1^T) * (x W3^T), y = h W2^T; W1 = gate, W3 = up,
 *     W2 = down, all in nn.Linear [out, in] order.
 *   shared expert: weight 1, added after the k routed terms.
 *   BF16 storage: h is rounded to bf16 (through fp32) before the down projection.
 *   FP8 storage: weights carry one fp32 scale per 128x128 block; activations
 *     (x, and h before the down projection) are quantised per 1x128 row block
 *     with scale = blockmax/448 computed in fp32 and codes = E4M3(v / scale)
 *     (fp32 division, round to nearest even, saturating); an all-zero block has
 *     scale 1 and zero codes. Every E4M3 value is dequantised exactly.
 *   output: the fp64 sum rounded once to bf16 (nearest even).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- bf16 ---- */

static double bf16_val(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* Round a float to bf16, nearest even (the oracle's own rounding). */
static uint16_t float_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
  uint32_t upper = u >> 16, lower = u & 0xFFFFu;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
  return (uint16_t)upper;
}

/* Round a double to bf16 once, nearest even (8 significant bits). */
static uint16_t double_to_bf16(double d) {
  if (d != d || d == 0.0 || fabs(d) < 1.1754943508222875e-38 || fabs(d) >= 3.3895313892515355e38)
    return float_to_bf16((float)d); /* NaN, zero, subnormal or overflow range: not reached by the tests */
  int e;
  const double m = frexp(d, &e);                  /* d = m 2^e, 0.5 <= |m| < 1 */
  const double q = nearbyint(ldexp(m, 8));        /* 8 significant bits, ties to even */
  return float_to_bf16((float)ldexp(q, e - 8));   /* exact in float, so this only repacks */
}

/* ---------------------------------------------------------------- E4M3 ---- */
/*
 * OCP 8-bit floating point, E4M3 ("FN": 4 exponent bits with bias 7, 3 mantissa
 * bits, no infinities, S.1111.111 is NaN, largest finite 448). The oracle keeps
 * the 127 non-negative finite values in a table, ascending with the code, and
 * encodes by searching it: the nearest value wins, an exact tie goes to the even
 * code (even mantissa), and anything at or above 448 saturates to 448.
 */
static float E4M3_POS[127];
static int e4m3_ready = 0;

static void e4m3_init(void) {
  if (e4m3_ready) return;
  for (int c = 0; c < 127; ++c) {
    const int e = c >> 3, m = c & 7;
    E4M3_POS[c] = (e == 0) ? (float)m / 512.0f : ldexpf(1.0f + (float)m / 8.0f, e - 7);
  }
  e4m3_ready = 1;
}

/* Threads the OpenMP loops below run on (1 without OpenMP): reported with the
 * oracle's timings. */
int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

double orc_e4m3_value(uint8_t c) {
  e4m3_init();
  if ((c & 0x7F) == 0x7F) return NAN;
  const double v = (double)E4M3_POS[c & 0x7F];
  return (c & 0x80) ? -v : v;
}

uint8_t orc_e4m3_encode(float v) {
  e4m3_init();
  if (v != v) return 0x7F;
  const uint8_t sign = (v < 0.0f || (v == 0.0f && signbit(v))) ? 0x80 : 0x00;
  const float a = fabsf(v);
  if (a >= E4M3_POS[126]) return sign | 126;
  int lo = 0, hi = 126; /* invariant: E4M3_POS[lo] <= a < E4M3_POS[hi] */
  while (hi - lo > 1) {
    const int mid = (lo + hi) / 2;
    if (E4M3_POS[mid] <= a) lo = mid; else hi = mid;
  }
  const double dlo = (double)a - (double)E4M3_POS[lo], dhi = (double)E4M3_POS[hi] - (double)a;
  int c;
  if (dlo < dhi) c = lo;
  else if (dhi < dlo) c = hi;
  else c = (lo % 2 == 0) ? lo : hi;
  return sign | (uint8_t)c;
}

void orc_e4m3_encode_array(int64_t n, const float* in, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(in[i]);
}

void orc_e4m3_decode_array(int64_t n, const uint8_t* in, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_value(in[i]);
}

/* 1x128 activation block quantisation of n fp32 values (n a multiple of 128). */
static void quantize_blocks(int64_t n, const float* v, uint8_t* q, float* s) {
  for (int64_t b = 0; b < n / 128; ++b) {
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) {
      const float a = fabsf(v[b * 128 + i]);
      if (a > amax) amax = a;
    }
    if (amax == 0.0f) {
      s[b] = 1.0f;
      for (int i = 0; i < 128; ++i) q[b * 128 + i] = 0;
      continue;
    }
    const float sc = amax / 448.0f;
    s[b] = sc;
    for (int i = 0; i < 128; ++i) q[b * 128 + i] = orc_e4m3_encode(v[b * 128 + i] / sc);
  }
}

/* Activation quantisation of x [T, H] (bf16) -> codes [T, H], scales [T, H/128]. */
void orc_quantize_rows(int64_t T, int32_t H, const uint16_t* x, uint8_t* q, float* s) {
  e4m3_init();
#pragma omp parallel
  {
    float* row = (float*)malloc(sizeof(float) * (size_t)H);
#pragma omp for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
      for (int h = 0; h < H; ++h) row[h] = (float)bf16_val(x[t * H + h]);
      quantize_blocks(H, row, q + t * (int64_t)H, s + t * (int64_t)(H / 128));
    }
    free(row);
  }
}

/* -------------------------------------------------------------- routing ---- */
/*
 * Learned router with top-k selection (NeMo "Step-5-Preview" page, "Model
 * Architecture": 352 routed experts, top-8 routing, a learned router).
 * logits_out (optional) receives the double logits [T, E].
 */
void orc_route(int64_t T, int32_t H, int32_t E, int32_t k, const uint16_t* x, const uint16_t* wr,
               const float* bias, double* logits_out, int32_t* idx, float* gate) {
#pragma omp parallel
  {
    double* l = (double*)malloc(sizeof(double) * (size_t)E);
    double* p = (double*)malloc(sizeof(double) * (size_t)E);
    char* taken = (char*)malloc((size_t)E);
#pragma omp for schedule(dynamic, 8)
    for (int64_t t = 0; t < T; ++t) {
      for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int h = 0; h < H; ++h) acc += bf16_val(x[t * H + h]) * bf16_val(wr[(int64_t)e * H + h]);
        if (bias) acc += (double)bias[e];
        l[e] = acc;
        if (logits_out) logits_out[t * E + e] = acc;
      }
      /* softmax over every expert */
      double m = l[0];
      for (int e = 1; e < E; ++e) if (l[e] > m) m = l[e];
      double z = 0.0;
      for (int e = 0; e < E; ++e) { p[e] = exp(l[e] - m); z += p[e]; }
      for (int e = 0; e < E; ++e) p[e] /= z;
      /* top-k by logit, ties to the lower index, in descending order */
      memset(taken, 0, (size_t)E);
      double psum = 0.0;
      for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
          if (taken[e]) continue;
          if (best < 0 || l[e] > l[best]) best = e;
        }
        taken[best] = 1;
        idx[t * k + j] = best;
        psum += p[best];
      }
      for (int j = 0; j < k; ++j) gate[t * k + j] = (float)(p[idx[t * k + j]] / psum);
    }
    free(l); free(p); free(taken);
  }
}

/* ------------------------------------------------------ histogram/permute ---- */
/*
 * The token -> expert histogram, its exclusive scan and the gather indices (the
 * README's "critical MoE primitives"). Groups 0..E-1 are the routed experts;
 * group E is the shared expert (when n_shared == 1) and receives every token.
 *   counts[g]  = number of rows of group g                     [E + S]
 *   offsets[g] = sum of counts of groups before g              [E + S + 1]
 *   perm[r]    = token of row r; rows of a group ascend by token [(k + S) T]
 *   pos[t, j]  = row of (token t, slot j); slot k is the shared row [T, k + S]
 * Returns 0; 1 for a bad shape; 5 if an expert index is outside [0, E).
 */
int orc_permute(int64_t T, int32_t E, int32_t k, int32_t n_shared, const int32_t* idx,
                int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos) {
  const int G = E + n_shared, S = k + n_shared;
  if (E <= 0 || k <= 0 || n_shared < 0 || n_shared > 1 || T < 0) return 1;
  for (int g = 0; g < G; ++g) counts[g] = 0;
  for (int64_t t = 0; t < T; ++t)
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      if (e < 0 || e >= E) return 5;
      counts[e] += 1;
    }
  if (n_shared) counts[E] = (int32_t)T;
  offsets[0] = 0;
  for (int g = 0; g < G; ++g) offsets[g + 1] = offsets[g] + counts[g];
  int32_t* fill = (int32_t*)calloc((size_t)G, sizeof(int32_t));
  for (int64_t t = 0; t < T; ++t) {  /* ascending tokens: a stable counting sort */
    for (int j = 0; j < k; ++j) {
      const int e = idx[t * k + j];
      const int32_t r = offsets[e] + fill[e]++;
      perm[r] = (int32_t)t;
      pos[t * S + j] = r;
    }
    if (n_shared) {
      const int32_t r = offsets[E] + fill[E]++;
      perm[r] = (int32_t)t;
      pos[t * S + k] = r;
    }
  }
  free(fill);
  return 0;
}

/* ---------------------------------------------------------- expert MLPs ---- */

/* ---------------------------------------------------------------- NVFP4 ---- */
/*
 * NVFP4 expert storage, as the TensorFold PR page describes the format its
 * W4A16 linears read: E2M1 codes two to a byte (input 2j in the low nibble of
 * byte j), one E4M3 scale per 16 inputs, and an fp32 global scale that
 * multiplies; an element is e2m1 x e4m3 x global. E2M1 (OCP 4-bit float): one
 * sign bit, two exponent bits with bias 1 and one mantissa bit; exponent 0 is
 * subnormal (m x 0.5). Its magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4 and 6.
 */
double orc_e2m1_value(uint8_t code) {
  const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  const double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

/* ---------------------------------------------------------- expert MLPs ---- */

/* wdtype: 0 = BF16; 1 = FP8 E4M3 with 128x128 fp32 block scales (E4M3 1x128
 * activations); 2 = NVFP4 (bf16 activations and h, as for BF16). */
typedef struct {
  int64_t T;
  int32_t H, E, k, n_shared, I, wdtype;
} orc_shape;

typedef struct {
  const uint16_t* router_w;
  const float* router_bias;
  const void *w1, *w3, *w2;   /* [E, I, H], [E, I, H], [E, H, I]; NVFP4: codes [E, I, H/2], [E, I, H/2], [E, H, I/2] */
  const void *s1, *s3, *s2;   /* FP8: fp32 [E, I/128, H/128], .., [E, H/128, I/128]; NVFP4: E4M3 [E, I, H/16], .., [E, H, I/16] */
  const void *sw1, *sw3, *sw2; /* shared expert, same layouts with E = 1 */
  const void *ss1, *ss3, *ss2;
  const float *g1, *g3, *g2;    /* NVFP4 global scales [E] */
  const float *sg1, *sg3, *sg2; /* NVFP4 global scales of the shared expert [1] */
} orc_weights;

/* Weight element W[g][r][c] of a stacked [G, R, C] tensor, dequantised exactly. */
static double wval(const orc_shape* sh, const void* w, const void* s, const float* gs, int64_t g, int64_t R,
                   int64_t C, int64_t r, int64_t c) {
  const int64_t row = g * R + r;
  if (sh->wdtype == 0) return bf16_val(((const uint16_t*)w)[row * C + c]);
  if (sh->wdtype == 1) {
    const double sc = (double)((const float*)s)[(g * (R / 128) + r / 128) * (C / 128) + c / 128];
    return orc_e4m3_value(((const uint8_t*)w)[row * C + c]) * sc;
  }
  const uint8_t byte = ((const uint8_t*)w)[row * (C / 2) + c / 2];
  const uint8_t code = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15);
  const uint8_t scale = ((const uint8_t*)s)[row * (C / 16) + c / 16];
  return orc_e2m1_value(code) * orc_e4m3_value(scale) * (double)gs[g];
}

/*
 * One expert on one activation row a[H] (already the values the expert sees):
 * y[H] = (round_h(silu(a W1^T) * (a W3^T))) W2^T, sums in double.
 */
static void expert_row(const orc_shape* sh, const orc_weights* w, int shared, int64_t g, const double* a,
                       double* hbuf, float* hf, uint8_t* hq, float* hs, double* y) {
  const int64_t H = sh->H, I = sh->I;
  const void *w1 = shared ? w->sw1 : w->w1, *w3 = shared ? w->sw3 : w->w3, *w2 = shared ? w->sw2 : w->w2;
  const void *s1 = shared ? w->ss1 : w->s1, *s3 = shared ? w->ss3 : w->s3, *s2 = shared ? w->ss2 : w->s2;
  const float *g1 = shared ? w->sg1 : w->g1, *g3 = shared ? w->sg3 : w->g3, *g2 = shared ? w->sg2 : w->g2;
  for (int64_t i = 0; i < I; ++i) {
    double gt = 0.0, up = 0.0;
    for (int64_t h = 0; h < H; ++h) {
      gt += a[h] * wval(sh, w1, s1, g1, g, I, H, i, h);
      up += a[h] * wval(sh, w3, s3, g3, g, I, H, i, h);
    }
    hbuf[i] = gt / (1.0 + exp(-gt)) * up; /* silu(gate) * up */
  }
  if (sh->wdtype != 1) {
    for (int64_t i = 0; i < I; ++i) hbuf[i] = bf16_val(float_to_bf16((float)hbuf[i]));
  } else {
    for (int64_t i = 0; i < I; ++i) hf[i] = (float)hbuf[i];
    quantize_blocks(I, hf, hq, hs);
    for (int64_t i = 0; i < I; ++i) hbuf[i] = orc_e4m3_value(hq[i]) * (double)hs[i / 128];
  }
  for (int64_t c = 0; c < H; ++c) {
    double acc = 0.0;
    for (int64_t i = 0; i < I; ++i) acc += hbuf[i] * wval(sh, w2, s2, g2, g, H, I, c, i);
    y[c] = acc;
  }
}

/*
 * The layer output for n_tok listed tokens, given the routing (idx [T, k],
 * gate [T, k]):
 *   out[t] = sum_{j<k} gate[t,j] * y_{idx[t,j]}(t)  +  y_shared(t)
 * summed in double in slot order. out_f64 [n_tok, H]; out_bf16 [n_tok, H] (optional);
 * y_out [n_tok, k + S, H] (optional, the ungated expert outputs per slot).
 */
void orc_moe_tokens(const orc_shape* sh, const orc_weights* w, const uint16_t* x, const int32_t* idx,
                    const float* gate, int64_t n_tok, const int64_t* tokens, double* out_f64,
                    uint16_t* out_bf16, double* y_out) {
  e4m3_init();
  const int64_t H = sh->H, I = sh->I;
  const int k = sh->k, S = sh->k + sh->n_shared;
  double* ys = (double*)malloc(sizeof(double) * (size_t)(n_tok * S * H));
#pragma omp parallel
  {
    double* a = (double*)malloc(sizeof(double) * (size_t)H);
    double* hbuf = (double*)malloc(sizeof(double) * (size_t)I);
    float* hf = (float*)malloc(sizeof(float) * (size_t)I);
    uint8_t* hq = (uint8_t*)malloc((size_t)I);
    float* hs = (float*)malloc(sizeof(float) * (size_t)(I / 128));
    float* xf = (float*)malloc(sizeof(float) * (size_t)H);
    uint8_t* xq = (uint8_t*)malloc((size_t)H);
    float* xs = (float*)malloc(sizeof(float) * (size_t)(H / 128));
#pragma omp for schedule(dynamic, 1)
    for (int64_t pi = 0; pi < n_tok * S; ++pi) {
      const int64_t n = pi / S, j = pi % S, t = tokens[n];
      /* the activation row the experts see */
      if (sh->wdtype != 1) {
        for (int64_t h = 0; h < H; ++h) a[h] = bf16_val(x[t * H + h]);
      } else {
        for (int64_t h = 0; h < H; ++h) xf[h] = (float)bf16_val(x[t * H + h]);
        quantize_blocks(H, xf, xq, xs);
        for (int64_t h = 0; h < H; ++h) a[h] = orc_e4m3_value(xq[h]) * (double)xs[h / 128];
      }
      double* y = ys + pi * H;
      if (j < k) expert_row(sh, w, 0, idx[t * k + j], a, hbuf, hf, hq, hs, y);
      else expert_row(sh, w, 1, 0, a, hbuf, hf, hq, hs, y);
    }
    free(a); free(hbuf); free(hf); free(hq); free(hs); free(xf); free(xq); free(xs);
  }
  for (int64_t n = 0; n < n_tok; ++n) {
    const int64_t t = tokens[n];
    for (int64_t c = 0; c < H; ++c) {
      double acc = 0.0;
      for (int j = 0; j < k; ++j) acc += (double)gate[t * k + j] * ys[(n * S + j) * H + c];
      if (sh->n_shared) acc += ys[(n * S + k) * H + c];
      out_f64[n * H + c] = acc;
      if (out_bf16) out_bf16[n * H + c] = double_to_bf16(acc);
    }
  }
  if (y_out) memcpy(y_out, ys, sizeof(double) * (size_t)(n_tok * S * H));
  free(ys);
}

/*
 * Single expert rows: y_out[i] = the (ungated) output of group groups[i] on
 * token tokens[i]'s activation row, for i < n. Groups 0..E-1 are the routed
 * experts, group E the shared expert. The same per-row evaluation as
 * orc_moe_tokens, for checking chosen rows of a large batch one by one.
 */
void orc_expert_rows(const orc_shape* sh, const orc_weights* w, const uint16_t* x, int64_t n,
                     const int64_t* tokens, const int32_t* groups, double* y_out) {
  e4m3_init();
  const int64_t H = sh->H, I = sh->I;
#pragma omp parallel
  {
    double* a = (double*)malloc(sizeof(double) * (size_t)H);
    double* hbuf = (double*)malloc(sizeof(double) * (size_t)I);
    float* hf = (float*)malloc(sizeof(float) * (size_t)I);
    uint8_t* hq = (uint8_t*)malloc((size_t)I);
    float* hs = (float*)malloc(sizeof(float) * (size_t)(I / 128));
    float* xf = (float*)malloc(sizeof(float) * (size_t)H);
    uint8_t* xq = (uint8_t*)malloc((size_t)H);
    float* xs = (float*)malloc(sizeof(float) * (size_t)(H / 128));
#pragma omp for schedule(dynamic, 1)
    for (int64_t i = 0; i < n; ++i) {
      const int64_t t = tokens[i];
      const int g = groups[i];
      if (sh->wdtype != 1) {
        for (int64_t h = 0; h < H; ++h) a[h] = bf16_val(x[t * H + h]);
      } else {
        for (int64_t h = 0; h < H; ++h) xf[h] = (float)bf16_val(x[t * H + h]);
        quantize_blocks(H, xf, xq, xs);
        for (int64_t h = 0; h < H; ++h) a[h] = orc_e4m3_value(xq[h]) * (double)xs[h / 128];
      }
      if (g < sh->E) expert_row(sh, w, 0, g, a, hbuf, hf, hq, hs, y_out + i * H);
      else expert_row(sh, w, 1, 0, a, hbuf, hf, hq, hs, y_out + i * H);
    }
    free(a); free(hbuf); free(hf); free(hq); free(hs); free(xf); free(xq); free(xs);
  }
}
