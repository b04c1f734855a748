/*
 * TTQ oracle: a plain, slow, single-threaded CPU statement of what the TTQ
 * linear layer computes.  TEST INFRASTRUCTURE ONLY: it is loaded by the test
 * suite, by the package's smoke check and by the benchmark's CPU-baseline leg.
 * No product code path calls it, and it shares no code, header or constant
 * generator with the CUDA library.
 *
 * Sources (arXiv:2603.19296, "TTQ: Activation-Aware Test-Time Quantization to
 * Accelerate LLM Inference On The Fly", as summarised on three gist.science
 * pages, plus the blog.lo0.es "Test-time quantization" post):
 *   - gist.science/zh/paper/2603.19296, section 2.1 (online AWQ):
 *       D_ii = (||X_i,:||_p + lambda)^alpha ,  W_hat = Q[W D^{1/2}] D^{-1/2}
 *   - gist.science/zh/paper/2603.19296, section 2.2 (low-rank): W ~ W_q + B A
 *   - gist.science/zh/paper/2603.19296, section 2.3: projection costs O[d' d T]
 *   - blog.lo0.es (English post), "The maths that matter": affine quantiser
 *       with scale s and zero point z, error bounded by s/2.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *   - the L_p norm is the raw norm over the T tokens passed in (no 1/T);
 *   - groups are `group` consecutive input channels of one row of W;
 *   - the range is min/max extended to include 0; the scale is rounded to
 *     binary16 toward +infinity and floored at 2^-14; the zero point is an
 *     integer in [0, 2^b-1]; codes are q = clamp(rint(x * (1/s)) + z);
 *     rint is round-half-to-even of the exact product; reconstruction is
 *     s (q - z);
 *   - the W given to the forward is the residual W_q is formed from; B, A
 *     are static and B (A X) is added unscaled.
 *
 * Precision: statistics, dequantisation and products are fp64.  The
 * quantiser (activation-aware pre-scale, range, scale, zero, codes) is run
 * in IEEE binary32 in a fixed operation order, because its output is an
 * integer decision that the GPU must reproduce bit for bit.  Build with
 * -O2 -ffp-contract=off and without fast-math.
 *
 * Every entry point returns 0 on success, or a positive flag word
 * (1 = invalid argument, 4 = non-finite value met).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define TTQO_OK 0
#define TTQO_BAD_ARG 1
#define TTQO_NONFINITE 4

/* ------------------------------------------------------------------------ */
/* IEEE 754 binary16 conversions written from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits; subnormals are
 * n * 2^-24 for n < 1024; the largest finite value is 65504.               */

float ttqo_f16_to_f32(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int f = h & 0x3ff;
  double v;
  if (e == 0x1f) {
    v = f ? NAN : INFINITY;
  } else if (e == 0) {
    v = ldexp((double)f, -24);
  } else {
    v = ldexp(1024.0 + (double)f, e - 25);
  }
  return (float)(sign ? -v : v);
}

/* Round a binary32 value to binary16 toward +infinity: the result is the
 * smallest binary16 value that is >= x (for x < -65504 that is -65504; for
 * x > 65504 it is +infinity). */
uint16_t ttqo_f32_to_f16_ru(float xf) {
  double x = (double)xf;
  if (isnan(x)) return 0x7e00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  if (sign == 0 && a > 65504.0) return 0x7c00;
  if (sign != 0 && a >= 65504.0) return 0xfbff;
  /* quantum of the binade that holds a */
  double ulp;
  int e = 0; /* exponent with a in [2^e, 2^(e+1)) */
  if (a < ldexp(1.0, -14)) {
    ulp = ldexp(1.0, -24);
  } else {
    int E;
    (void)frexp(a, &E); /* a = f 2^E, f in [0.5, 1) */
    e = E - 1;
    ulp = ldexp(1.0, e - 10);
  }
  double m = a / ulp; /* exact: a has <= 24 significant bits, ulp is 2^k */
  /* toward +inf: magnitude rounds up for positive, down for negative */
  double n = sign ? floor(m) : ceil(m);
  if (a < ldexp(1.0, -14)) {
    /* subnormal: the bit pattern is n itself; n == 1024 is 2^-14 */
    return (uint16_t)(sign | (uint16_t)n);
  }
  /* normal: a = n 2^(e-10), n in [1024, 2048]; n == 2048 carries into the
   * exponent field, and 0x7c00 (infinity) if e + 1 == 16 */
  uint32_t bits = ((uint32_t)(e + 15) << 10) + (uint32_t)(n - 1024.0);
  return (uint16_t)(sign | bits);
}

/* Binary16 nearest-even from an integer-valued zero point (exact for
 * integers up to 2048). */
static uint16_t f16_from_small_int(int v) {
  if (v == 0) return 0;
  return ttqo_f32_to_f16_ru((float)v); /* exact, so rounding never acts */
}

/* ------------------------------------------------------------------------ */
/* Step 1: activation statistic (gist.science/zh, section 2.1):
 *   n_i  = ( sum_t |X[t][i]|^p )^(1/p)     (the L_p norm of channel i)
 *   D_i  = (n_i + lambda)^alpha
 *   Dr_i = D_i^(-1/2)
 * X is stored [T][d] (token-major), so channel i is column i.            */
int ttqo_act_norm(const double* X, int64_t T, int64_t d, double p,
                  double lambda, double alpha, double* D, double* Dr) {
  if (!X || !D || !Dr || T < 0 || d < 1 || !(p >= 1.0) || !(lambda >= 0.0) ||
      !(alpha >= 0.0))
    return TTQO_BAD_ARG;
  int flags = TTQO_OK;
  for (int64_t i = 0; i < d; ++i) {
    double acc = 0.0;
    for (int64_t t = 0; t < T; ++t) acc += pow(fabs(X[t * d + i]), p);
    double n = pow(acc, 1.0 / p);
    double Di = pow(n + lambda, alpha);
    D[i] = Di;
    Dr[i] = 1.0 / sqrt(Di);
    if (!isfinite(Di) || !(Di > 0.0) || !isfinite(Dr[i])) flags |= TTQO_NONFINITE;
  }
  return flags;
}

/* ------------------------------------------------------------------------ */
/* Packed codes: row j is a little-endian bit stream of uint32 words; code i
 * sits in bits [b*i, b*i + b).  Words per row = ceil(d*b/32).             */
int64_t ttqo_words_per_row(int64_t d, int bits) {
  return (d * bits + 31) / 32;
}

int ttqo_code_at(const uint32_t* row, int64_t i, int bits) {
  int64_t bit = i * bits;
  uint64_t lo = row[bit >> 5];
  uint64_t hi = ((bit & 31) + bits > 32) ? row[(bit >> 5) + 1] : 0;
  uint64_t v = (lo | (hi << 32)) >> (bit & 31);
  return (int)(v & ((1u << bits) - 1));
}

static void put_code(uint32_t* row, int64_t i, int bits, uint32_t q) {
  for (int k = 0; k < bits; ++k) {
    int64_t bit = i * bits + k;
    if ((q >> k) & 1u) row[bit >> 5] |= 1u << (bit & 31);
  }
}

/* Step 2: Q[W D^{1/2}] as group-wise asymmetric b-bit round-to-nearest
 * (gist.science/zh section 2.1 for the pre-scale; blog.lo0.es "The maths
 * that matter" for the affine quantiser).  Binary32, in this order:
 *   h_i  = sqrt(D_i)                     (1 when D is NULL: plain RTN)
 *   x    = W[j][i] * h_i
 *   m    = min(0, min_group x),  M = max(0, max_group x)
 *   s32  = (M - m) / (2^b - 1);  if !(s32 >= 2^-14) s32 = 2^-14
 *   s    = binary16(s32, toward +inf)   -> scales[j][k]
 *   inv  = 1 / s
 *   z    = clamp(rint(-m * inv), 0, 2^b - 1)   -> zeros[j][k] (binary16)
 *   q    = clamp(rint(x * inv) + z, 0, 2^b - 1) -> codes
 * The two products inside rint are exact (binary32 x binary32 fits in
 * binary64), so each code is rint of the true x * inv: one rounding, to the
 * integer, half to even.
 * W and D are binary32 arrays (bf16 inputs widen to binary32 exactly).    */
int ttqo_quantize(const float* W, int64_t dp, int64_t d, const float* D,
                  int bits, int group, uint32_t* codes, uint16_t* scales,
                  uint16_t* zeros) {
  if (!W || !codes || !scales || !zeros || dp < 0 || d < 1 || bits < 1 ||
      bits > 8 || group < 1 || d % group != 0)
    return TTQO_BAD_ARG;
  int flags = TTQO_OK;
  const int qmax = (1 << bits) - 1;
  const int64_t wpr = ttqo_words_per_row(d, bits);
  const int64_t ngroups = d / group;
  float* h = (float*)malloc(sizeof(float) * (size_t)d);
  float* x = (float*)malloc(sizeof(float) * (size_t)group);
  if (!h || !x) {
    free(h);
    free(x);
    return TTQO_BAD_ARG;
  }
  for (int64_t i = 0; i < d; ++i) {
    h[i] = D ? sqrtf(D[i]) : 1.0f;
    if (!isfinite(h[i])) flags |= TTQO_NONFINITE;
  }
  memset(codes, 0, sizeof(uint32_t) * (size_t)(dp * wpr));
  for (int64_t j = 0; j < dp; ++j) {
    uint32_t* crow = codes + j * wpr;
    for (int64_t k = 0; k < ngroups; ++k) {
      float m = 0.0f, M = 0.0f;
      for (int c = 0; c < group; ++c) {
        int64_t i = k * group + c;
        float w = W[j * d + i];
        if (!isfinite(w)) flags |= TTQO_NONFINITE;
        x[c] = w * h[i];
        if (x[c] < m) m = x[c];
        if (x[c] > M) M = x[c];
      }
      float range = M - m;
      float s32 = range / (float)qmax;
      if (!(s32 >= 0x1p-14f)) s32 = 0x1p-14f;
      uint16_t s16 = ttqo_f32_to_f16_ru(s32);
      if ((s16 & 0x7c00) == 0x7c00) flags |= TTQO_NONFINITE;
      float s = ttqo_f16_to_f32(s16);
      float inv = 1.0f / s;
      double zr = rint(-(double)m * (double)inv);
      int z = (int)(zr < 0.0 ? 0.0 : (zr > (double)qmax ? (double)qmax : zr));
      scales[j * ngroups + k] = s16;
      zeros[j * ngroups + k] = f16_from_small_int(z);
      for (int c = 0; c < group; ++c) {
        double r = rint((double)x[c] * (double)inv);
        long q = (long)r + z;
        if (q < 0) q = 0;
        if (q > qmax) q = qmax;
        put_code(crow, k * group + c, bits, (uint32_t)q);
      }
    }
  }
  free(h);
  free(x);
  return flags;
}

/* Step 2, symmetric variant (blog.lo0.es "Test-time quantization ...",
 * section "The maths that matter": a symmetric b-bit range has levels
 * +-(2^(b-1) - 1) and the scale that covers a group of largest magnitude M
 * is M / (2^(b-1) - 1); every element is then off by at most s/2).
 * Binary32, in this order:
 *   h_i  = sqrt(D_i)                     (1 when D is NULL)
 *   x    = W[j][i] * h_i
 *   M    = max_group |x|
 *   s32  = M / (2^(b-1) - 1);  if !(s32 >= 2^-14) s32 = 2^-14
 *   s    = binary16(s32, toward +inf)   -> scales[j][k]
 *   inv  = 1 / s
 *   l    = clamp(rint(x * inv), -(2^(b-1) - 1), 2^(b-1) - 1)  (exact product)
 *   code = l + 2^(b-1)  in [1, 2^b - 1];  zeros[j][k] = 2^(b-1)
 * so that the stored (code, scale, zero) reconstruct s (code - zero) = s l
 * exactly as the asymmetric format does.  Needs bits >= 2.                */
int ttqo_quantize_sym(const float* W, int64_t dp, int64_t d, const float* D,
                      int bits, int group, uint32_t* codes, uint16_t* scales,
                      uint16_t* zeros) {
  if (!W || !codes || !scales || !zeros || dp < 0 || d < 1 || bits < 2 ||
      bits > 8 || group < 1 || d % group != 0)
    return TTQO_BAD_ARG;
  int flags = TTQO_OK;
  const int lmax = (1 << (bits - 1)) - 1;
  const int zero = 1 << (bits - 1);
  const int64_t wpr = ttqo_words_per_row(d, bits);
  const int64_t ngroups = d / group;
  float* sq = (float*)malloc(sizeof(float) * (size_t)d);  /* sqrt(D_i) */
  float* v = (float*)malloc(sizeof(float) * (size_t)group);  /* prescaled group */
  if (!sq || !v) {
    free(sq);
    free(v);
    return TTQO_BAD_ARG;
  }
  for (int64_t i = 0; i < d; ++i) {
    sq[i] = D ? sqrtf(D[i]) : 1.0f;
    if (!isfinite(sq[i])) flags |= TTQO_NONFINITE;
  }
  memset(codes, 0, sizeof(uint32_t) * (size_t)(dp * wpr));
  for (int64_t j = 0; j < dp; ++j) {
    uint32_t* crow = codes + j * wpr;
    for (int64_t k = 0; k < ngroups; ++k) {
      float M = 0.0f;
      for (int c = 0; c < group; ++c) {
        int64_t i = k * group + c;
        float w = W[j * d + i];
        if (!isfinite(w)) flags |= TTQO_NONFINITE;
        v[c] = w * sq[i];
        float a = fabsf(v[c]);
        if (a > M) M = a;
      }
      float s32 = M / (float)lmax;
      if (!(s32 >= 0x1p-14f)) s32 = 0x1p-14f; /* binary16 normal range */
      uint16_t s16 = ttqo_f32_to_f16_ru(s32);
      if ((s16 & 0x7c00) == 0x7c00) flags |= TTQO_NONFINITE;
      float s = ttqo_f16_to_f32(s16);
      float inv = 1.0f / s;
      scales[j * ngroups + k] = s16;
      zeros[j * ngroups + k] = f16_from_small_int(zero);
      for (int c = 0; c < group; ++c) {
        long l = (long)rint((double)v[c] * (double)inv);
        if (l < -lmax) l = -lmax;
        if (l > lmax) l = lmax;
        put_code(crow, k * group + c, bits, (uint32_t)(l + zero));
      }
    }
  }
  free(sq);
  free(v);
  return flags;
}

/* ------------------------------------------------------------- FP8 codes
 * blog.lo0.es (English post), the comparison with FP8 end to end: TTQ
 * decides how s is obtained, not the format of the code, so "TTQ over FP8"
 * is the same activation-aware scale feeding an FP8 quantiser.  Readings:
 *   - the format is E4M3 as the OCP 8-bit floating point specification
 *     defines it: 1 sign bit, 4 exponent bits (bias 7), 3 fraction bits;
 *     exponent 0 is subnormal (m/8 * 2^-6); no infinities; S.1111.111 is NaN;
 *     the largest finite magnitude is 448 (S.1111.110);
 *   - the scale is symmetric per group: s = binary16 round-up of
 *     max|x| / 448 (floored at 2^-14), so |x| / s <= 448;
 *   - the code is the E4M3 value nearest to the binary32 product x * (1/s),
 *     ties to the even code, saturating at +-448 (the sign of a product that
 *     rounds to zero is kept);
 *   - the zero point is 0 (stored as binary16 +0) and the reconstruction is
 *     s * e4m3(code); the 8-bit codes are packed like any 8-bit code (4 per
 *     word, code i in bits 8 (i mod 4) .. of word i / 4).                  */
double ttqo_e4m3_value(uint32_t code) {
  const int sign = (code >> 7) & 1;
  const int e = (code >> 3) & 15;
  const int m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);             /* m/8 * 2^-6 */
  else v = ldexp(8.0 + (double)m, e - 10);           /* (1 + m/8) 2^(e-7) */
  return sign ? -v : v;
}

/* Nearest finite E4M3 magnitude by search over the 127 non-negative finite
 * codes, ties to the code whose last fraction bit is 0; beyond 448 the
 * result is 448; the sign of v is kept.  NaN maps to the NaN code 0x7F.  */
uint32_t ttqo_e4m3_from(double v) {
  if (isnan(v)) return 0x7Fu;
  const uint32_t sign = signbit(v) ? 0x80u : 0u;
  const double a = fabs(v);
  uint32_t best = 0;
  double bestd = INFINITY;
  for (uint32_t c = 0; c <= 0x7Eu; ++c) {
    const double dd = fabs(ttqo_e4m3_value(c) - a);
    if (dd < bestd || (dd == bestd && (c & 1u) == 0u)) {
      bestd = dd;
      best = c;
    }
  }
  return best | sign;
}

/* The FP8 (E4M3) quantiser with the activation-aware scale; codes are 8 bits
 * per weight, zeros are binary16 +0.                                      */
int ttqo_quantize_fp8(const float* W, int64_t dp, int64_t d, const float* D, int group,
                      uint32_t* codes, uint16_t* scales, uint16_t* zeros) {
  if (!W || !codes || !scales || !zeros || dp < 0 || d < 1 || group < 1 || d % group != 0)
    return TTQO_BAD_ARG;
  int flags = TTQO_OK;
  const int64_t wpr = ttqo_words_per_row(d, 8);
  const int64_t ngroups = d / group;
  float* sd = (float*)malloc(sizeof(float) * (size_t)d);
  float* xg = (float*)malloc(sizeof(float) * (size_t)group);
  if (!sd || !xg) {
    free(sd);
    free(xg);
    return TTQO_BAD_ARG;
  }
  for (int64_t i = 0; i < d; ++i) {
    sd[i] = D ? sqrtf(D[i]) : 1.0f;
    if (!isfinite(sd[i])) flags |= TTQO_NONFINITE;
  }
  memset(codes, 0, sizeof(uint32_t) * (size_t)(dp * wpr));
  for (int64_t j = 0; j < dp; ++j) {
    uint32_t* crow = codes + j * wpr;
    for (int64_t k = 0; k < ngroups; ++k) {
      float amax = 0.0f;
      for (int c = 0; c < group; ++c) {
        const int64_t i = k * group + c;
        const float w = W[j * d + i];
        if (!isfinite(w)) flags |= TTQO_NONFINITE;
        xg[c] = w * sd[i];
        if (fabsf(xg[c]) > amax) amax = fabsf(xg[c]);
      }
      float s32 = amax / 448.0f;
      if (!(s32 >= 0x1p-14f)) s32 = 0x1p-14f;
      const uint16_t s16 = ttqo_f32_to_f16_ru(s32);
      if ((s16 & 0x7c00) == 0x7c00) flags |= TTQO_NONFINITE;
      const float s = ttqo_f16_to_f32(s16);
      const float inv = 1.0f / s;
      scales[j * ngroups + k] = s16;
      zeros[j * ngroups + k] = 0;
      for (int c = 0; c < group; ++c) {
        const float prod = xg[c] * inv;               /* binary32 product */
        put_code(crow, k * group + c, 8, ttqo_e4m3_from((double)prod));
      }
    }
  }
  free(sd);
  free(xg);
  return flags;
}

/* FP8 reconstruction: w_hat[j][i] = s_jk e4m3(q_ji) Dr_i in fp64, for the
 * listed rows (rows == NULL: rows 0..nrows-1); Dr == NULL means D = I.     */
int ttqo_dequant_rows_fp8(const uint32_t* codes, const uint16_t* scales, const double* Dr,
                          int64_t dp, int64_t d, int group, const int64_t* rows, int64_t nrows,
                          double* What) {
  if (!codes || !scales || !What || d < 1 || group < 1 || d % group != 0 || nrows < 0)
    return TTQO_BAD_ARG;
  const int64_t wpr = ttqo_words_per_row(d, 8);
  const int64_t ngroups = d / group;
  for (int64_t rr = 0; rr < nrows; ++rr) {
    const int64_t j = rows ? rows[rr] : rr;
    if (j < 0 || j >= dp) return TTQO_BAD_ARG;
    for (int64_t i = 0; i < d; ++i) {
      const double sc = (double)ttqo_f16_to_f32(scales[j * ngroups + i / group]);
      const double val = ttqo_e4m3_value((uint32_t)ttqo_code_at(codes + j * wpr, i, 8));
      What[rr * d + i] = sc * val * (Dr ? Dr[i] : 1.0);
    }
  }
  return TTQO_OK;
}

/* Step 3: W_hat = Q[.] D^{-1/2}: w_hat[j][i] = s_jk (q_ji - z_jk) Dr_i, in
 * fp64, for the listed rows only (rows == NULL means rows 0..nrows-1).
 * Dr == NULL means D = I.                                                  */
int ttqo_dequant_rows(const uint32_t* codes, const uint16_t* scales,
                      const uint16_t* zeros, const double* Dr, int64_t dp,
                      int64_t d, int bits, int group, const int64_t* rows,
                      int64_t nrows, double* What) {
  if (!codes || !scales || !zeros || !What || d < 1 || group < 1 ||
      d % group != 0 || bits < 1 || bits > 8 || nrows < 0)
    return TTQO_BAD_ARG;
  const int64_t wpr = ttqo_words_per_row(d, bits);
  const int64_t ngroups = d / group;
  for (int64_t rr = 0; rr < nrows; ++rr) {
    int64_t j = rows ? rows[rr] : rr;
    if (j < 0 || j >= dp) return TTQO_BAD_ARG;
    for (int64_t i = 0; i < d; ++i) {
      int64_t k = i / group;
      double s = (double)ttqo_f16_to_f32(scales[j * ngroups + k]);
      double z = (double)ttqo_f16_to_f32(zeros[j * ngroups + k]);
      double q = (double)ttqo_code_at(codes + j * wpr, i, bits);
      double dr = Dr ? Dr[i] : 1.0;
      What[rr * d + i] = s * (q - z) * dr;
    }
  }
  return TTQO_OK;
}

/* Step 4: projection Y = W_hat X (gist.science/zh section 2.3), written
 * token-major: Y[t][r] = sum_i What[r][i] X[t][i].                         */
int ttqo_project(const double* What, int64_t nrows, const double* X,
                 int64_t T, int64_t d, double* Y) {
  if (!What || !X || !Y || nrows < 0 || T < 0 || d < 1) return TTQO_BAD_ARG;
  for (int64_t t = 0; t < T; ++t)
    for (int64_t r = 0; r < nrows; ++r) {
      double acc = 0.0;
      for (int64_t i = 0; i < d; ++i) acc += What[r * d + i] * X[t * d + i];
      Y[t * nrows + r] = acc;
    }
  return TTQO_OK;
}

/* Step 5: the static low-rank term (gist.science/zh section 2.2):
 *   AX[t][k] = sum_i A[k][i] X[t][i];  Y[t][r] += sum_k B[row r][k] AX[t][k]
 * Brows holds the B rows of the listed output rows, [nrows][rank].        */
int ttqo_lowrank_add(const double* A, const double* Brows, int64_t rank,
                     int64_t nrows, const double* X, int64_t T, int64_t d,
                     double* Y) {
  if (rank < 0 || nrows < 0 || T < 0 || d < 1 || !Y) return TTQO_BAD_ARG;
  if (rank == 0) return TTQO_OK;
  if (!A || !Brows || !X) return TTQO_BAD_ARG;
  double* ax = (double*)malloc(sizeof(double) * (size_t)(rank > 0 ? rank : 1));
  if (!ax) return TTQO_BAD_ARG;
  for (int64_t t = 0; t < T; ++t) {
    for (int64_t k = 0; k < rank; ++k) {
      double acc = 0.0;
      for (int64_t i = 0; i < d; ++i) acc += A[k * d + i] * X[t * d + i];
      ax[k] = acc;
    }
    for (int64_t r = 0; r < nrows; ++r) {
      double acc = 0.0;
      for (int64_t k = 0; k < rank; ++k) acc += Brows[r * rank + k] * ax[k];
      Y[t * nrows + r] += acc;
    }
  }
  free(ax);
  return TTQO_OK;
}

/* Unpacks rows of codes into one int32 per code, [dp][d] (test helper). */
int ttqo_unpack(const uint32_t* codes, int64_t dp, int64_t d, int bits,
                int32_t* out) {
  if (!codes || !out || dp < 0 || d < 1 || bits < 1 || bits > 8)
    return TTQO_BAD_ARG;
  const int64_t wpr = ttqo_words_per_row(d, bits);
  for (int64_t j = 0; j < dp; ++j)
    for (int64_t i = 0; i < d; ++i)
      out[j * d + i] = ttqo_code_at(codes + j * wpr, i, bits);
  return TTQO_OK;
}
