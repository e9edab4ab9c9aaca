/*
 * Seeded synthetic inputs for the Step-5 routed-MoE layer.
 *
 * This module only makes inputs. It is shared by the CPU oracle's tests and by
 * the benchmark; it does none of the layer's forward arithmetic (routing,
 * activation quantisation, expert MLPs, combine).
 *
 * Generator: counter-based, so every element depends only on (seed, tensor id,
 * element index) and never on the thread count.
 *   key(seed, id)   = splitmix64(splitmix64(seed) ^ (id * 0xD1B54A32D192ED03))
 *   draw(key, n)    = splitmix64(key + n * 0x9E3779B97F4A7C15)
 * splitmix64 is Vigna's published SplitMix64 output function. Element pairs
 * (2p, 2p+1) take one Box-Muller pair computed in double from
 *   u1 = ((draw(key, 2p)   >> 11) + 0.5) * 2^-53      in (0, 1)
 *   u2 =  (draw(key, 2p+1) >> 11)        * 2^-53      in [0, 1)
 *   z0 = sqrt(-2 ln u1) cos(2 pi u2),  z1 = sqrt(-2 ln u1) sin(2 pi u2)
 * and a value v = z * std is stored as bf16 by rounding (float)v to nearest even.
 *
 * FP8 weights are the same bf16 draws, quantised offline per 128x128 block the
 * way a block-scaled FP8 checkpoint stores them: scale = blockmax / 448 (fp32),
 * code = E4M3(value / scale) rounded to nearest even, saturating at 448; an
 * all-zero block gets scale 1 and zero codes. This is checkpoint preparation,
 * not part of the layer; it has its own E4M3 encoder (below), written apart
 * from the oracle's and the kernels'. NVFP4 weights (E2M1 codes, an E4M3 scale
 * per 16 inputs, an fp32 global scale) are prepared the same way, with this
 * module's own E2M1 encoder.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ull

static inline uint64_t splitmix64(uint64_t z) {
  z += GOLDEN;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t tensor_key(uint64_t seed, uint64_t id) {
  return splitmix64(splitmix64(seed) ^ (id * 0xD1B54A32D192ED03ull));
}

/* The Box-Muller pair for elements (2p, 2p+1) of the stream `key`. */
static inline void normal_pair(uint64_t key, uint64_t p, double* z0, double* z1) {
  const uint64_t r1 = splitmix64(key + (2 * p) * GOLDEN);
  const uint64_t r2 = splitmix64(key + (2 * p + 1) * GOLDEN);
  const double u1 = ((double)(r1 >> 11) + 0.5) * (1.0 / 9007199254740992.0);
  const double u2 = (double)(r2 >> 11) * (1.0 / 9007199254740992.0);
  const double rad = sqrt(-2.0 * log(u1));
  const double ang = 6.283185307179586476925286766559 * u2;
  *z0 = rad * cos(ang);
  *z1 = rad * sin(ang);
}

/* Standard normal for element n of the stream `key`. */
static inline double normal_at(uint64_t key, uint64_t n) {
  double z0, z1;
  normal_pair(key, n >> 1, &z0, &z1);
  return (n & 1) ? z1 : z0;
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* x[i] = bf16(std * N(0,1)_i) for i in [0, n). */
void synth_normal_bf16(uint64_t seed, uint64_t id, int64_t n, double std, uint16_t* out) {
  const uint64_t key = tensor_key(seed, id);
  const int64_t npair = (n + 1) / 2;
#pragma omp parallel for schedule(static)
  for (int64_t p = 0; p < npair; ++p) {
    double z0, z1;
    normal_pair(key, (uint64_t)p, &z0, &z1);
    out[2 * p] = f32_to_bf16_rne((float)(z0 * std));
    if (2 * p + 1 < n) out[2 * p + 1] = f32_to_bf16_rne((float)(z1 * std));
  }
}

/* Same values as fp32 (for per-expert bias vectors and similar small inputs). */
void synth_normal_f32(uint64_t seed, uint64_t id, int64_t n, double std, float* out) {
  const uint64_t key = tensor_key(seed, id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(normal_at(key, (uint64_t)i) * std);
}

/* Uniform 64-bit draws (used for seeded permutations). */
void synth_u64(uint64_t seed, uint64_t id, int64_t n, uint64_t* out) {
  const uint64_t key = tensor_key(seed, id);
  for (int64_t i = 0; i < n; ++i) out[i] = splitmix64(key + (uint64_t)i * GOLDEN);
}

/* E4M3 (OCP "FN" variant: bias 7, no infinities, max finite 448) encoder with
 * round-to-nearest-even and saturation, built from the bit layout. */
static inline uint8_t e4m3_encode_prep(float v) {
  uint8_t sign = 0;
  if (v < 0.0f || (v == 0.0f && signbit(v))) { sign = 0x80; v = -v; }
  if (v != v) return 0x7F;
  if (v >= 448.0f) return sign | 0x7E;
  if (v < 0.015625f) {                       /* below 2^-6: subnormal grid of step 2^-9 */
    const float m = nearbyintf(v * 512.0f);   /* exact scaling; default rounding is RNE */
    return sign | (uint8_t)m;                 /* m == 8 is the smallest normal, code 0x08 */
  }
  int ex;
  const float fr = frexpf(v, &ex);            /* v = fr * 2^ex, fr in [0.5, 1) */
  int e = ex - 1;                             /* v = (2 fr) 2^e, 2 fr in [1, 2) */
  float q = nearbyintf((2.0f * fr - 1.0f) * 8.0f);
  if (q == 8.0f) { q = 0.0f; e += 1; }
  int code = ((e + 7) << 3) | (int)q;
  if (code > 0x7E) code = 0x7E;
  return sign | (uint8_t)code;
}

static inline float e4m3_decode_prep(uint8_t c) {
  const int e = (c >> 3) & 15, m = c & 7;
  float v;
  if ((c & 0x7F) == 0x7F) return NAN;
  if (e == 0) v = ldexpf((float)m, -9);
  else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return (c & 0x80) ? -v : v;
}

/*
 * Block-scaled FP8 weights for G stacked matrices of shape [rows, cols]
 * (nn.Linear order: [out, in], in contiguous). rows and cols are multiples of
 * 128. Values are the bf16 draws of synth_normal_bf16(seed, id, G*rows*cols, std).
 * codes: [G, rows, cols] uint8; scales: [G, rows/128, cols/128] fp32.
 */
void synth_fp8_blocks(uint64_t seed, uint64_t id, int64_t G, int64_t rows, int64_t cols, double std,
                      uint8_t* codes, float* scales) {
  const uint64_t key = tensor_key(seed, id);
  const int64_t br = rows / 128, bc = cols / 128;
  const int64_t nblk = G * br * bc;
#pragma omp parallel
  {
    float vals[128 * 128];
#pragma omp for schedule(dynamic, 4)
    for (int64_t b = 0; b < nblk; ++b) {
      const int64_t g = b / (br * bc), rb = (b / bc) % br, cb = b % bc;
      float amax = 0.0f;
      for (int r = 0; r < 128; ++r) {
        const int64_t row = rb * 128 + r;
        const int64_t base = (g * rows + row) * cols + cb * 128;
        for (int c = 0; c < 128; c += 2) {
          double z0, z1;
          normal_pair(key, (uint64_t)((base + c) >> 1), &z0, &z1);
          const float f0 = bf16_to_f32(f32_to_bf16_rne((float)(z0 * std)));
          const float f1 = bf16_to_f32(f32_to_bf16_rne((float)(z1 * std)));
          vals[r * 128 + c] = f0;
          vals[r * 128 + c + 1] = f1;
          if (fabsf(f0) > amax) amax = fabsf(f0);
          if (fabsf(f1) > amax) amax = fabsf(f1);
        }
      }
      const float s = (amax > 0.0f) ? amax / 448.0f : 1.0f;
      scales[b] = s;
      for (int r = 0; r < 128; ++r) {
        const int64_t row = rb * 128 + r;
        uint8_t* dst = codes + (g * rows + row) * cols + cb * 128;
        for (int c = 0; c < 128; ++c) dst[c] = (amax > 0.0f) ? e4m3_encode_prep(vals[r * 128 + c] / s) : 0;
      }
    }
  }
}

/* Decoded value of a code under this module's decoder (for input checks). */
float synth_e4m3_value(uint8_t c) { return e4m3_decode_prep(c); }

/* E2M1 (OCP 4-bit float: 1 sign, 2 exponent bits with bias 1, 1 mantissa bit;
 * magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) encoder: nearest magnitude, an exact
 * tie to the even code, saturation at 6. This module's own, for checkpoint
 * preparation. */
static const float E2M1_MAG[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

static inline uint8_t e2m1_encode_prep(float v) {
  const uint8_t sign = (v < 0.0f || (v == 0.0f && signbit(v))) ? 8 : 0;
  const float a = fabsf(v);
  if (a >= 6.0f) return sign | 7;
  int lo = 0;
  while (lo < 7 && E2M1_MAG[lo + 1] <= a) ++lo; /* E2M1_MAG[lo] <= a < E2M1_MAG[lo + 1] */
  const float dlo = a - E2M1_MAG[lo], dhi = E2M1_MAG[lo + 1] - a;
  int c = (dlo < dhi) ? lo : (dhi < dlo ? lo + 1 : ((lo & 1) ? lo + 1 : lo));
  return sign | (uint8_t)c;
}

float synth_e2m1_value(uint8_t c) { return (c & 8) ? -E2M1_MAG[c & 7] : E2M1_MAG[c & 7]; }

/*
 * NVFP4 weights for G stacked matrices of shape [rows, cols] (nn.Linear order,
 * cols a multiple of 16), the way an NVFP4 checkpoint stores them: per matrix a
 * global fp32 scale gs = amax / (6 * 448) (1 for an all-zero matrix); per 16
 * consecutive inputs of a row an E4M3 scale s = E4M3(blockmax / (6 gs)); codes
 * E2M1(v / (s gs)), two per byte with input 2j in the low nibble of byte j (all
 * zero where s decodes to 0). Values are the bf16 draws of
 * synth_normal_bf16(seed, id, G*rows*cols, std).
 * codes [G, rows, cols/2] uint8; scales [G, rows, cols/16] uint8; gscale [G] fp32.
 */
void synth_nvfp4(uint64_t seed, uint64_t id, int64_t G, int64_t rows, int64_t cols, double std, uint8_t* codes,
                 uint8_t* scales, float* gscale) {
  const uint64_t key = tensor_key(seed, id);
  const int64_t n = rows * cols;
#pragma omp parallel
  {
    float* vals = (float*)malloc(sizeof(float) * (size_t)n);
#pragma omp for schedule(dynamic, 1)
    for (int64_t g = 0; g < G; ++g) {
      float amax = 0.0f;
      for (int64_t i = 0; i < n; i += 2) {
        double z0, z1;
        normal_pair(key, (uint64_t)((g * n + i) >> 1), &z0, &z1);
        vals[i] = bf16_to_f32(f32_to_bf16_rne((float)(z0 * std)));
        vals[i + 1] = bf16_to_f32(f32_to_bf16_rne((float)(z1 * std)));
        if (fabsf(vals[i]) > amax) amax = fabsf(vals[i]);
        if (fabsf(vals[i + 1]) > amax) amax = fabsf(vals[i + 1]);
      }
      const float gs = amax > 0.0f ? amax / (6.0f * 448.0f) : 1.0f;
      gscale[g] = gs;
      for (int64_t b = 0; b < n / 16; ++b) {
        const float* v = vals + b * 16;
        float bmax = 0.0f;
        for (int i = 0; i < 16; ++i) if (fabsf(v[i]) > bmax) bmax = fabsf(v[i]);
        const uint8_t sc = e4m3_encode_prep(bmax / (6.0f * gs));
        const float s = e4m3_decode_prep(sc);
        scales[g * (n / 16) + b] = sc;
        uint8_t* dst = codes + g * (n / 2) + b * 8;
        for (int i = 0; i < 16; i += 2) {
          const uint8_t lo = s > 0.0f ? e2m1_encode_prep(v[i] / (s * gs)) : 0;
          const uint8_t hi = s > 0.0f ? e2m1_encode_prep(v[i + 1] / (s * gs)) : 0;
          dst[i / 2] = (uint8_t)(lo | (hi << 4));
        }
      }
    }
    free(vals);
  }
}
