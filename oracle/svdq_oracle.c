/*
 * CPU oracle for the SVDQuant W4A4 linear layer (NVFP4 g16 and INT4 g64) and
 * the AWQ W4A16 linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do. It shares no code with the CUDA library.
 *
 * What it computes (the pages: Diffusers "Nunchaku Lite" page, table
 * "Supported quantization types"; blog "Introducing Nunchaku 4-bit inference
 * in Diffusers", section "Background: SVDQuant and Nunchaku"):
 *   SVDQuant moves activation outliers into the weights with a per-channel
 *   smoothing vector lambda, keeps a 16-bit low-rank branch L1 L2 and quantises
 *   the residual R to 4 bits:
 *       y = Q4(x_hat) . Q4(R) + (x_hat L1) L2 + b,
 *       x_hat = bf16(x * (1/lambda)),  R = diag(lambda) W - L1 L2.
 *   svdq_w4a4/nvfp4 uses E2M1 values with one E4M3 scale per 16 along K and one
 *   fp32 tensor scale; svdq_w4a4/int4 uses symmetric INT4 with one bf16 scale
 *   per 64 along K; awq_w4a16/int4 uses asymmetric INT4 weights with bf16
 *   scale and zero point per 64 along K and bf16 activations.
 *
 * Where the pages leave a step open, the plainest reading is taken; every
 * such reading is listed in the design notes of the repository. In brief:
 *   - scales are computed from the group absolute maximum; quantised values
 *     are value * (1/dequant_scale) rounded to the grid (ties to even,
 *     saturating);
 *   - NVFP4: block scale = e4m3(amax / (6 * t)), t = tensor scale; the weight
 *     tensor scale is amax(R) / (6 * 448); the activation tensor scale is a
 *     static argument (1.0 in every workload);
 *   - INT4: scale = bf16(amax / 7), codes clamp(rne(v/s), -8, 7);
 *   - AWQ: scale = bf16((max-min)/15) (1 if zero), zero = clamp(rne(-min/s),0,15),
 *     q = clamp(rne(w/s) + zero, 0, 15), dequantised as (q - zero) * s;
 *   - packed codes: element 2j in the low nibble of byte j; weights [N, K/2].
 *
 * Every floating-point step that feeds a quantisation decision is one fp32
 * operation with one rounding, written out below (this file is compiled with
 * -ffp-contract=off so no multiply-add is fused). Sums that only produce
 * floating outputs (P, y) are taken in double and rounded once.
 *
 * Format definitions (OCP Microscaling spec v1.0 for E2M1 and E4M3; bfloat16
 * as the top half of IEEE binary32):
 *   E2M1: 1 sign, 2 exponent (bias 1), 1 mantissa bit; magnitudes
 *         {0, 0.5, 1, 1.5, 2, 3, 4, 6}; no inf/NaN.
 *   E4M3 (fn): 1 sign, 4 exponent (bias 7), 3 mantissa bits, subnormals,
 *         max 448, S.1111.111 is NaN, no inf.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL -1

/* ------------------------------------------------------------------------- */
/* threads                                                                   */
/* ------------------------------------------------------------------------- */

void orc_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int orc_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------- */
/* number formats                                                            */
/* ------------------------------------------------------------------------- */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

float orc_bf16_to_f32(uint16_t b) { return f32_from_bits((uint32_t)b << 16); }

/* Round a real value (given exactly as a double) to the nearest bfloat16,
 * ties to the even significand; magnitudes at or beyond the overflow
 * threshold give infinity, as IEEE round-to-nearest does. */
uint16_t orc_bf16_rn_f64(double v) {
  if (isnan(v)) return (uint16_t)(signbit(v) ? 0xFFC0u : 0x7FC0u);
  int neg = signbit(v) != 0;
  double a = fabs(v);
  double r;
  if (a == 0.0) {
    r = 0.0;
  } else if (a < 0x1p-126) {
    /* subnormal range: spacing 2^-133 */
    r = ldexp(nearbyint(ldexp(a, 133)), -133);
  } else {
    int e;
    double m = frexp(a, &e);               /* a = m * 2^e, m in [0.5, 1) */
    double q = nearbyint(ldexp(m, 8));     /* 8 significant bits */
    r = ldexp(q, e - 8);
  }
  uint16_t out;
  if (isinf(r) || r > 0x1.FEp127) {
    out = 0x7F80u; /* +inf */
  } else {
    out = (uint16_t)(bits_from_f32((float)r) >> 16); /* r is exactly a bf16 */
  }
  return (uint16_t)(out | (neg ? 0x8000u : 0u));
}

uint16_t orc_bf16_rn(float v) { return orc_bf16_rn_f64((double)v); }

float orc_e4m3_to_f32(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  float v;
  if (e == 0xF && m == 7) return s ? -NAN : NAN;
  if (e == 0) v = (float)m * 0x1p-9f;                 /* subnormal: m/8 * 2^-6 */
  else v = ldexpf(1.0f + (float)m / 8.0f, e - 7);
  return s ? -v : v;
}

/* fp32 -> E4M3, round to nearest (ties to even), saturating to +-448.
 * NaN maps to the NaN code (0x7F with the sign bit). */
uint8_t orc_e4m3_rn_sat(float v) {
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  if (isnan(v)) return (uint8_t)(sign | 0x7F);
  double a = fabs((double)v);
  uint8_t code;
  if (a >= 448.0) {
    code = 0x7E;
  } else if (a < 0x1p-6) {
    /* subnormals and zero: spacing 2^-9; 8 * 2^-9 is the smallest normal, whose
     * code (exponent field 1, mantissa 0) is 8 as well */
    code = (uint8_t)nearbyint(ldexp(a, 9));
  } else {
    int e;
    double m = frexp(a, &e);                 /* a = m * 2^e, m in [0.5, 1) */
    int E = e - 1;                           /* a = (2m) * 2^E, 2m in [1, 2) */
    int q = (int)nearbyint((2.0 * m - 1.0) * 8.0);
    if (q == 8) { q = 0; E += 1; }
    int ef = E + 7;
    code = (uint8_t)((ef << 3) | q);
    if (code > 0x7E) code = 0x7E;
  }
  return (uint8_t)(sign | code);
}

float orc_e2m1_to_f32(uint8_t c) {
  static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
  float v = mag[c & 7];
  return (c & 8) ? -v : v;
}

/* fp32 -> E2M1 code (low nibble), round to nearest (ties to even), saturating
 * to +-6. The sign bit follows the sign of the input, so -0 and negative
 * values that round to zero give 0x8. NaN gives 0x7 with its sign. */
uint8_t orc_e2m1_rn_sat(float v) {
  uint8_t sign = signbit(v) ? 0x8 : 0x0;
  if (isnan(v)) return (uint8_t)(sign | 0x7);
  double a = fabs((double)v);
  uint8_t code;
  if (a >= 6.0) {
    code = 7;
  } else if (a < 1.0) {
    code = (uint8_t)nearbyint(a * 2.0);      /* 0, 0.5, 1.0 -> codes 0, 1, 2 */
  } else {
    int e;
    double m = frexp(a, &e);                 /* a = (2m) * 2^(e-1) */
    int E = e - 1;                           /* 0, 1 or 2 */
    int q = (int)nearbyint((2.0 * m - 1.0) * 2.0);
    if (q == 2) { q = 0; E += 1; }
    code = (uint8_t)(((E + 1) << 1) | q);
    if (code > 7) code = 7;
  }
  return (uint8_t)(sign | code);
}

/* Sweep helper: compare device conversions of the fp32 bit patterns
 * [start, start+count) with this file's. Any of the three device arrays may
 * be NULL. bad[0..2] receive the mismatch counts (e2m1, e4m3, bf16) and
 * first_bad[0..2] the first mismatching bit pattern (or 0xFFFFFFFF). NaN
 * inputs are compared for e4m3 and bf16 by class only (any NaN code) and are
 * skipped for e2m1, which has no NaN. */
void orc_check_cvt_range(uint64_t start, uint64_t count, const uint8_t* e2m1_dev,
                         const uint8_t* e4m3_dev, const uint16_t* bf16_dev,
                         int64_t* bad, uint32_t* first_bad) {
  int64_t b0 = 0, b1 = 0, b2 = 0;
  uint32_t f0 = 0xFFFFFFFFu, f1 = 0xFFFFFFFFu, f2 = 0xFFFFFFFFu;
#pragma omp parallel for schedule(static) reduction(+ : b0, b1, b2) reduction(min : f0, f1, f2)
  for (int64_t i = 0; i < (int64_t)count; ++i) {
    uint32_t bits = (uint32_t)(start + (uint64_t)i);
    float v = f32_from_bits(bits);
    int is_nan = isnan(v);
    if (e2m1_dev && !is_nan) {
      if ((e2m1_dev[i] & 0xF) != orc_e2m1_rn_sat(v)) { ++b0; if (bits < f0) f0 = bits; }
    }
    if (e4m3_dev) {
      uint8_t ref = orc_e4m3_rn_sat(v);
      int ok = is_nan ? ((e4m3_dev[i] & 0x7F) == 0x7F) : (e4m3_dev[i] == ref);
      if (!ok) { ++b1; if (bits < f1) f1 = bits; }
    }
    if (bf16_dev) {
      uint16_t ref = orc_bf16_rn(v);
      int ok = is_nan ? (((bf16_dev[i] & 0x7F80) == 0x7F80) && (bf16_dev[i] & 0x7F))
                      : (bf16_dev[i] == ref);
      if (!ok) { ++b2; if (bits < f2) f2 = bits; }
    }
  }
  bad[0] = b0; bad[1] = b1; bad[2] = b2;
  first_bad[0] = f0; first_bad[1] = f1; first_bad[2] = f2;
}

/* ------------------------------------------------------------------------- */
/* group quantisers                                                          */
/* ------------------------------------------------------------------------- */

/* NVFP4 group of 16 values with tensor scale t:
 *   amax = max |v|;  sf = e4m3(amax / (6 t));  d = float(sf) * t;
 *   code_i = e2m1(v_i * (1/d)), or 0 for every element when d == 0. */
void orc_nvfp4_group(const float* v, float t, uint8_t* codes, uint8_t* sf) {
  float amax = 0.0f;
  for (int i = 0; i < 16; ++i) { float a = fabsf(v[i]); if (a > amax) amax = a; }
  float six_t = 6.0f * t;
  float ratio = amax / six_t;
  uint8_t s = orc_e4m3_rn_sat(ratio);
  float d = orc_e4m3_to_f32(s) * t;
  *sf = s;
  if (d == 0.0f) {
    for (int i = 0; i < 16; ++i) codes[i] = 0;
    return;
  }
  float inv = 1.0f / d;
  for (int i = 0; i < 16; ++i) {
    float q = v[i] * inv;
    codes[i] = orc_e2m1_rn_sat(q);
  }
}

static int clamp_int(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

/* Symmetric INT4 group of 64 values:
 *   s = bf16(amax / 7); q_i = clamp(rne(v_i * (1/float(s))), -8, 7), or 0 when s == 0. */
void orc_int4_group(const float* v, int8_t* q, uint16_t* s_out) {
  float amax = 0.0f;
  for (int i = 0; i < 64; ++i) { float a = fabsf(v[i]); if (a > amax) amax = a; }
  float ratio = amax / 7.0f;
  uint16_t s = orc_bf16_rn(ratio);
  float sf = orc_bf16_to_f32(s);
  *s_out = s;
  if (sf == 0.0f) {
    for (int i = 0; i < 64; ++i) q[i] = 0;
    return;
  }
  float inv = 1.0f / sf;
  for (int i = 0; i < 64; ++i) {
    float p = v[i] * inv;
    q[i] = (int8_t)clamp_int((int)nearbyintf(p), -8, 7);
  }
}

static void put_nibble(uint8_t* row, int k, uint8_t code) {
  uint8_t c = code & 0xF;
  if (k & 1) row[k >> 1] = (uint8_t)((row[k >> 1] & 0x0F) | (c << 4));
  else row[k >> 1] = (uint8_t)((row[k >> 1] & 0xF0) | c);
}

static uint8_t get_nibble(const uint8_t* row, int k) {
  return (k & 1) ? (uint8_t)(row[k >> 1] >> 4) : (uint8_t)(row[k >> 1] & 0xF);
}

static int int4_value(uint8_t nib) { return (nib & 8) ? (int)nib - 16 : (int)nib; }

/* ------------------------------------------------------------------------- */
/* svdq_w4a4                                                                 */
/* ------------------------------------------------------------------------- */

enum { ORC_NVFP4 = 0, ORC_INT4 = 1 };

/* Offline pack of one layer.
 *   inv_lam[k] = 1 / lam[k]                              (fp32)
 *   What[k,n]  = lam[k] * W[k,n]                         (fp32)
 *   R[k,n]     = fp32( What[k,n] - sum_j L1[k,j] L2[j,n] ) (the sum in double,
 *                                                         j ascending)
 *   NVFP4: s_tw = amax|R| / (6*448) (1 if that is 0); per (n, 16-block) as in
 *          orc_nvfp4_group with t = s_tw.
 *   INT4:  per (n, 64-block) as in orc_int4_group; s_tw = 1.
 * Outputs: w_codes [N, K/2]; w_scales [N, K/16] e4m3 bytes or [N, K/64] bf16;
 * s_tw [1]; inv_lam [K]; R_out [K, N] (nullable). */
int orc_svdq_pack_weight(int prec, int K, int N, int r, const float* W, const float* lam,
                         const uint16_t* L1, const uint16_t* L2, uint8_t* w_codes,
                         void* w_scales, float* s_tw_out, float* inv_lam, float* R_out) {
  const int G = prec == ORC_NVFP4 ? 16 : 64;
  if ((prec != ORC_NVFP4 && prec != ORC_INT4) || K <= 0 || N <= 0 || r < 0 || K % G) return ORC_EINVAL;
  for (int k = 0; k < K; ++k) inv_lam[k] = 1.0f / lam[k];

  float* R = (float*)malloc(sizeof(float) * (size_t)K * (size_t)N);
  if (!R) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
  for (int k = 0; k < K; ++k) {
    for (int n = 0; n < N; ++n) {
      float what = lam[k] * W[(size_t)k * N + n];
      double lr = 0.0;
      for (int j = 0; j < r; ++j)
        lr += (double)orc_bf16_to_f32(L1[(size_t)k * r + j]) * (double)orc_bf16_to_f32(L2[(size_t)j * N + n]);
      R[(size_t)k * N + n] = (float)((double)what - lr);
    }
  }

  float s_tw = 1.0f;
  if (prec == ORC_NVFP4) {
    float amax = 0.0f;
    for (size_t i = 0; i < (size_t)K * N; ++i) { float a = fabsf(R[i]); if (a > amax) amax = a; }
    float t = amax / 2688.0f; /* 6 * 448 */
    s_tw = (t == 0.0f) ? 1.0f : t;
  }
  *s_tw_out = s_tw;

#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    uint8_t* crow = w_codes + (size_t)n * (K / 2);
    float v[64];
    uint8_t c[16];
    int8_t q[64];
    for (int b = 0; b < K / G; ++b) {
      for (int i = 0; i < G; ++i) v[i] = R[(size_t)(b * G + i) * N + n];
      if (prec == ORC_NVFP4) {
        uint8_t sf;
        orc_nvfp4_group(v, s_tw, c, &sf);
        ((uint8_t*)w_scales)[(size_t)n * (K / 16) + b] = sf;
        for (int i = 0; i < 16; ++i) put_nibble(crow, b * 16 + i, c[i]);
      } else {
        uint16_t s;
        orc_int4_group(v, q, &s);
        ((uint16_t*)w_scales)[(size_t)n * (K / 64) + b] = s;
        for (int i = 0; i < 64; ++i) put_nibble(crow, b * 64 + i, (uint8_t)(q[i] & 0xF));
      }
    }
  }
  if (R_out) memcpy(R_out, R, sizeof(float) * (size_t)K * N);
  free(R);
  return ORC_OK;
}

/* Activation side of the layer.
 *   x_hat[m,k] = bf16( float(x[m,k]) * inv_lam[k] )
 *   NVFP4: orc_nvfp4_group on each 16-block of x_hat with t = s_tx;
 *   INT4:  orc_int4_group on each 64-block;
 *   P[m,j] = bf16( sum_k x_hat[m,k] L1[k,j] )  (double sum, rounded once).
 * Outputs: x_codes [M, K/2]; x_scales [M, K/16] e4m3 or [M, K/64] bf16; P [M, r]. */
int orc_svdq_quantize_act(int prec, int M, int K, int r, const uint16_t* x, const float* inv_lam,
                          float s_tx, const uint16_t* L1, uint8_t* x_codes, void* x_scales,
                          uint16_t* P) {
  const int G = prec == ORC_NVFP4 ? 16 : 64;
  if ((prec != ORC_NVFP4 && prec != ORC_INT4) || M < 0 || K <= 0 || r < 0 || K % G) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
  for (int m = 0; m < M; ++m) {
    float* xh = (float*)malloc(sizeof(float) * (size_t)K);
    uint8_t* crow = x_codes + (size_t)m * (K / 2);
    for (int k = 0; k < K; ++k) {
      float prod = orc_bf16_to_f32(x[(size_t)m * K + k]) * inv_lam[k];
      xh[k] = orc_bf16_to_f32(orc_bf16_rn(prod));
    }
    uint8_t c[16];
    int8_t q[64];
    for (int b = 0; b < K / G; ++b) {
      if (prec == ORC_NVFP4) {
        uint8_t sf;
        orc_nvfp4_group(xh + b * 16, s_tx, c, &sf);
        ((uint8_t*)x_scales)[(size_t)m * (K / 16) + b] = sf;
        for (int i = 0; i < 16; ++i) put_nibble(crow, b * 16 + i, c[i]);
      } else {
        uint16_t s;
        orc_int4_group(xh + b * 64, q, &s);
        ((uint16_t*)x_scales)[(size_t)m * (K / 64) + b] = s;
        for (int i = 0; i < 64; ++i) put_nibble(crow, b * 64 + i, (uint8_t)(q[i] & 0xF));
      }
    }
    for (int j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += (double)xh[k] * (double)orc_bf16_to_f32(L1[(size_t)k * r + j]);
      P[(size_t)m * r + j] = orc_bf16_rn_f64(acc);
    }
    free(xh);
  }
  return ORC_OK;
}

/* Dequantised value of element k of a packed row. */
static double deq(int prec, const uint8_t* crow, const void* srow, int k) {
  uint8_t nib = get_nibble(crow, k);
  if (prec == ORC_NVFP4)
    return (double)orc_e4m3_to_f32(((const uint8_t*)srow)[k / 16]) * (double)orc_e2m1_to_f32(nib);
  return (double)orc_bf16_to_f32(((const uint16_t*)srow)[k / 64]) * (double)int4_value(nib);
}

/* The layer output before its final rounding, in double:
 *   y[m,n] = s_tx * s_tw * sum_k deq_x[m,k] deq_w[n,k] + sum_j P[m,j] L2[j,n] + b[n]
 * (INT4: s_tx = s_tw = 1 and deq uses the bf16 group scales). Every product of
 * dequantised values is exact in double. rows (nullable) selects n_rows rows
 * of x; y is [n_rows, N]. */
int orc_svdq_linear(int prec, int M, int K, int N, int r, const uint8_t* x_codes,
                    const void* x_scales, float s_tx, const uint16_t* P, const uint8_t* w_codes,
                    const void* w_scales, float s_tw, const uint16_t* L2, const uint16_t* bias,
                    int n_rows, const int* rows, double* y) {
  const int G = prec == ORC_NVFP4 ? 16 : 64;
  if ((prec != ORC_NVFP4 && prec != ORC_INT4) || M < 0 || K <= 0 || N <= 0 || r < 0 || K % G) return ORC_EINVAL;
  const size_t sx_row = prec == ORC_NVFP4 ? (size_t)(K / 16) : (size_t)(K / 64) * 2;
  const double alpha = prec == ORC_NVFP4 ? (double)s_tx * (double)s_tw : 1.0;

  /* dequantised weights, one row per output column n */
  double* wd = (double*)malloc(sizeof(double) * (size_t)N * K);
  if (!wd) return ORC_EINVAL;
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    const uint8_t* crow = w_codes + (size_t)n * (K / 2);
    const uint8_t* srow = (const uint8_t*)w_scales + (size_t)n * sx_row;
    for (int k = 0; k < K; ++k) wd[(size_t)n * K + k] = deq(prec, crow, srow, k);
  }

#pragma omp parallel for schedule(dynamic, 1)
  for (int i = 0; i < n_rows; ++i) {
    int m = rows ? rows[i] : i;
    double* xd = (double*)malloc(sizeof(double) * (size_t)K);
    const uint8_t* crow = x_codes + (size_t)m * (K / 2);
    const uint8_t* srow = (const uint8_t*)x_scales + (size_t)m * sx_row;
    for (int k = 0; k < K; ++k) xd[k] = deq(prec, crow, srow, k);
    for (int n = 0; n < N; ++n) {
      const double* w = wd + (size_t)n * K;
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += xd[k] * w[k];
      double lr = 0.0;
      for (int j = 0; j < r; ++j)
        lr += (double)orc_bf16_to_f32(P[(size_t)m * r + j]) * (double)orc_bf16_to_f32(L2[(size_t)j * N + n]);
      double b = bias ? (double)orc_bf16_to_f32(bias[n]) : 0.0;
      y[(size_t)i * N + n] = alpha * acc + lr + b;
    }
    free(xd);
  }
  free(wd);
  return ORC_OK;
}

/* INT4 per-group integer dot products: out[m, n, g] = sum_{k in group g} qx[m,k] qw[n,k]. */
int orc_int4_group_sums(int M, int K, int N, const uint8_t* x_codes, const uint8_t* w_codes,
                        int32_t* out) {
  if (M < 0 || K <= 0 || N <= 0 || K % 64) return ORC_EINVAL;
  const int NG = K / 64;
#pragma omp parallel for schedule(static)
  for (int m = 0; m < M; ++m) {
    const uint8_t* xr = x_codes + (size_t)m * (K / 2);
    for (int n = 0; n < N; ++n) {
      const uint8_t* wr = w_codes + (size_t)n * (K / 2);
      for (int g = 0; g < NG; ++g) {
        int32_t acc = 0;
        for (int k = g * 64; k < g * 64 + 64; ++k)
          acc += int4_value(get_nibble(xr, k)) * int4_value(get_nibble(wr, k));
        out[((size_t)m * N + n) * NG + g] = acc;
      }
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* awq_w4a16                                                                 */
/* ------------------------------------------------------------------------- */

/* Round-to-nearest asymmetric INT4 pack of W [K, N], one (scale, zero) per
 * output column n and 64-block of K. Outputs q [N, K/2] (unsigned nibbles),
 * s [N, K/64] bf16, z [N, K/64] bf16 (an integer 0..15). */
int orc_awq_pack_weight(int K, int N, const float* W, uint8_t* q, uint16_t* s, uint16_t* z) {
  if (K <= 0 || N <= 0 || K % 64) return ORC_EINVAL;
  const int NG = K / 64;
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    uint8_t* qrow = q + (size_t)n * (K / 2);
    for (int g = 0; g < NG; ++g) {
      float mn = W[(size_t)(g * 64) * N + n], mx = mn;
      for (int k = g * 64; k < g * 64 + 64; ++k) {
        float w = W[(size_t)k * N + n];
        if (w < mn) mn = w;
        if (w > mx) mx = w;
      }
      float range = mx - mn;
      float ratio = range / 15.0f;
      uint16_t sb = orc_bf16_rn(ratio);
      if (orc_bf16_to_f32(sb) == 0.0f) sb = 0x3F80; /* 1.0 */
      float sf = orc_bf16_to_f32(sb);
      float inv = 1.0f / sf;
      float negmin = -mn;
      float zt = negmin * inv;
      int zi = clamp_int((int)nearbyintf(zt), 0, 15);
      s[(size_t)n * NG + g] = sb;
      z[(size_t)n * NG + g] = orc_bf16_rn((float)zi);
      for (int k = g * 64; k < g * 64 + 64; ++k) {
        float p = W[(size_t)k * N + n] * inv;
        int qi = clamp_int((int)nearbyintf(p) + zi, 0, 15);
        put_nibble(qrow, k, (uint8_t)qi);
      }
    }
  }
  return ORC_OK;
}

/* y[m,n] = sum_g s[n,g] * sum_{k in g} x[m,k] * (q[n,k] - z[n,g]) + b[n], in
 * double, before the final bf16 rounding. */
int orc_awq_linear(int M, int K, int N, const uint16_t* x, const uint8_t* q, const uint16_t* s,
                   const uint16_t* z, const uint16_t* bias, double* y) {
  if (M < 0 || K <= 0 || N <= 0 || K % 64) return ORC_EINVAL;
  const int NG = K / 64;
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    const uint8_t* qrow = q + (size_t)n * (K / 2);
    for (int m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int g = 0; g < NG; ++g) {
        double sg = (double)orc_bf16_to_f32(s[(size_t)n * NG + g]);
        double zg = (double)orc_bf16_to_f32(z[(size_t)n * NG + g]);
        double part = 0.0;
        for (int k = g * 64; k < g * 64 + 64; ++k)
          part += (double)orc_bf16_to_f32(x[(size_t)m * K + k]) * ((double)get_nibble(qrow, k) - zg);
        acc += sg * part;
      }
      y[(size_t)m * N + n] = acc + (bias ? (double)orc_bf16_to_f32(bias[n]) : 0.0);
    }
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* fused QKV epilogue: per-head RMSNorm of Q and K, then rotary embedding     */
/* ------------------------------------------------------------------------- */
/* The grouped projection's output y [M, 3*H*D] holds Q, K and V concatenated
 * along the output dimension in that order, each as H heads of D columns
 * (Diffusers "Nunchaku Lite" page, section on fused kernels: Q/K/V projection
 * combined with RMSNorm and RoPE; the grouped to_qkv module). For every row m
 * and every head of Q (weight wq) and of K (weight wk):
 *   u[d]      = v[d] / sqrt(mean_d(v^2) + eps) * w[d]          (RMSNorm over D)
 *   out[2i]   = u[2i] cos[m,i] - u[2i+1] sin[m,i]               (rotary embedding,
 *   out[2i+1] = u[2i] sin[m,i] + u[2i+1] cos[m,i]                pairs (2i, 2i+1))
 * V is passed through. y is the unrounded layer output (the fusion reads the
 * GEMM accumulator); everything is in double and the caller rounds once.
 * wq, wk: bf16 [D]; cos, sin: fp32 [M, D/2]; out: [M, 3*H*D]. */
int orc_qkv_norm_rope(int M, int H, int D, const double* y, const uint16_t* wq, const uint16_t* wk,
                      double eps, const float* cos_t, const float* sin_t, double* out) {
  if (M < 0 || H <= 0 || D <= 0 || D % 2 || eps < 0.0) return ORC_EINVAL;
  const size_t N = (size_t)3 * H * D;
#pragma omp parallel for schedule(static)
  for (int m = 0; m < M; ++m) {
    const double* yr = y + (size_t)m * N;
    double* orow = out + (size_t)m * N;
    for (size_t n = 2 * (size_t)H * D; n < N; ++n) orow[n] = yr[n];  /* V */
    double* u = (double*)malloc(sizeof(double) * (size_t)D);
    for (int sec = 0; sec < 2; ++sec) {
      const uint16_t* w = sec == 0 ? wq : wk;
      for (int h = 0; h < H; ++h) {
        const size_t off = ((size_t)sec * H + h) * D;
        double ss = 0.0;
        for (int d = 0; d < D; ++d) ss += yr[off + d] * yr[off + d];
        const double inv = 1.0 / sqrt(ss / D + eps);
        for (int d = 0; d < D; ++d) u[d] = yr[off + d] * inv * (double)orc_bf16_to_f32(w[d]);
        for (int i = 0; i < D / 2; ++i) {
          const double c = (double)cos_t[(size_t)m * (D / 2) + i], sn = (double)sin_t[(size_t)m * (D / 2) + i];
          orow[off + 2 * i] = u[2 * i] * c - u[2 * i + 1] * sn;
          orow[off + 2 * i + 1] = u[2 * i] * sn + u[2 * i + 1] * c;
        }
      }
    }
    free(u);
  }
  return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* fused GELU-MLP epilogue                                                     */
/* ------------------------------------------------------------------------- */
/* The MLP's up-projection output y (unrounded, as the GEMM accumulator holds
 * it) through GELU, rounded once to the bf16 activation the down-projection's
 * activation pass reads (Diffusers "Nunchaku Lite" page, section on fused
 * kernels: the MLP uses a fused GELU kernel):
 *   h = bf16( y * (1 + erf(y / sqrt(2))) / 2 )
 * in double. The down-projection then takes h through orc_svdq_quantize_act. */
void orc_gelu_bf16(const double* y, int64_t n, uint16_t* h) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    const double v = y[i];
    h[i] = orc_bf16_rn_f64(0.5 * v * (1.0 + erf(v * 0.70710678118654752440)));
  }
}

/* ------------------------------------------------------------------------- */
/* array forms of the format conversions (for the tests)                     */
/* ------------------------------------------------------------------------- */

void orc_bf16_rn_f64_array(const double* v, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_bf16_rn_f64(v[i]);
}

void orc_e4m3_rn_array(const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_rn_sat(v[i]);
}

void orc_e2m1_rn_array(const float* v, int64_t n, uint8_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_rn_sat(v[i]);
}
