/*
 * Oracle for the SVDQuant W4A4 linear layer (svdq_w4a4): plain, slow, obviously
 * correct CPU code.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library.  It shares no
 * code, header, table or constant with the CUDA library, and must never be
 * reached from the product path.
 *
 * What the method computes comes from two web pages:
 *   [P5] "Hugging Face встроила Nunchaku в Diffusers: диффузия быстрее на 30%,
 *        видеопамяти нужно до 50% меньше" (iitog.ru), paragraph "Суть метода":
 *        W4A4 = 4-bit weights AND 4-bit activations; activation outliers are moved
 *        into the weights; the hardest part of each weight matrix goes to a 16-bit
 *        low-rank branch; the remainder is quantized to 4 bits.  Next paragraph:
 *        runtime layer svdq_w4a4 in INT4 and NVFP4 variants.
 *   [P4] "SVDQuant ускоряет Krea 2 вдвое даже на старых NVIDIA GPU"
 *        (ainews.so), section "Решение: INT8 и W4A4": no calibration dataset,
 *        low-rank branches compensate the quantization error.
 * The pages print no formula.  The numeric readings taken here (group sizes,
 * scale encodings, rounding rules, the power-of-two per-tensor NVFP4 scale) are
 * listed with their reasons in the design notes; each function below says which
 * reading it implements.
 *
 * Number formats are written from their public definitions:
 *   bf16   : IEEE-754-style binary with 8 significant bits, exponent range of binary32.
 *   fp16   : IEEE-754 binary16 (11 significant bits, emin = -14, max 65504).
 *   E4M3   : OCP 8-bit floating point "E4M3" (4 significant bits, emin = -6,
 *            max finite 448, no infinities, S.1111.111 is NaN).
 *   E2M1   : OCP MX 4-bit floating point (2 significant bits, emin = 0,
 *            values +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}).
 * Every encoder rounds to nearest, ties to even, through one generic routine.
 *
 * Build: gcc -O2 -ffp-contract=off -fno-fast-math -shared -fPIC (no fused
 * multiply-add may change a rounding step).
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* Generic round-to-nearest-even onto a binary floating-point grid.           */
/* ------------------------------------------------------------------------- */

/* Round x to the grid of a binary format with `p` significant bits whose
 * smallest normal binade starts at 2^emin.  In the binade [2^E, 2^(E+1)) the
 * spacing is 2^(E-p+1); below 2^emin (subnormals) the spacing is fixed at
 * 2^(emin-p+1).  Ties go to the even multiple of the spacing, which is the
 * grid point whose last significand bit is 0.  No overflow handling here. */
static double rne_to_grid(double x, int p, int emin) {
  if (x == 0.0 || isnan(x) || isinf(x)) return x;
  int e2;
  double m = frexp(fabs(x), &e2); /* |x| = m * 2^e2, m in [0.5, 1) */
  (void)m;
  int E = e2 - 1;                  /* |x| in [2^E, 2^(E+1)) */
  if (E < emin) E = emin;
  double quantum = ldexp(1.0, E - p + 1);
  double n = nearbyint(x / quantum); /* default mode: nearest, ties to even */
  return n * quantum;
}

/* ---------------------------------- bf16 --------------------------------- */

static uint16_t bits_of_f32_top(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

/* double -> bf16, one rounding (no detour through binary32). */
uint16_t orc_f64_to_bf16(double x) {
  if (isnan(x)) return 0x7FC0;
  double y = rne_to_grid(x, 8, -126);
  if (fabs(y) >= ldexp(1.0, 128)) return (uint16_t)(signbit(x) ? 0xFF80 : 0x7F80);
  /* y has at most 8 significant bits and a binary32 exponent: exact in float,
     and its low 16 float bits are zero. */
  return bits_of_f32_top((float)y);
}

uint16_t orc_f32_to_bf16(float x) { return orc_f64_to_bf16((double)x); }

float orc_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ---------------------------------- fp16 --------------------------------- */

uint16_t orc_f32_to_f16(float xf) {
  double x = (double)xf;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  if (isnan(x)) return 0x7E00;
  double y = fabs(rne_to_grid(x, 11, -14));
  if (y > 65504.0 || isinf(y)) return sign | 0x7C00;
  if (y == 0.0) return sign;
  if (y < ldexp(1.0, -14)) { /* subnormal: y = mant * 2^-24 */
    return sign | (uint16_t)(y / ldexp(1.0, -24));
  }
  int e2;
  frexp(y, &e2);
  int E = e2 - 1; /* y in [2^E, 2^(E+1)) */
  uint16_t mant = (uint16_t)((y / ldexp(1.0, E) - 1.0) * 1024.0);
  return sign | (uint16_t)((E + 15) << 10) | mant;
}

float orc_f16_to_f32(uint16_t h) {
  int s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  double v;
  if (e == 0) v = ldexp((double)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = ldexp(1.0 + m / 1024.0, e - 15);
  return (float)(s ? -v : v);
}

/* ---------------------------------- E4M3 --------------------------------- */

/* Saturating: finite values beyond +-448 (after rounding) become +-448. */
uint8_t orc_f32_to_e4m3_satfinite(float xf) {
  double x = (double)xf;
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0;
  double y = fabs(rne_to_grid(x, 4, -6));
  if (y > 448.0 || isinf(y)) y = 448.0;
  if (y == 0.0) return sign;
  if (y < ldexp(1.0, -6)) return sign | (uint8_t)(y / ldexp(1.0, -9));
  int e2;
  frexp(y, &e2);
  int E = e2 - 1;
  uint8_t mant = (uint8_t)((y / ldexp(1.0, E) - 1.0) * 8.0);
  return sign | (uint8_t)((E + 7) << 3) | mant;
}

float orc_e4m3_to_f32(uint8_t c) {
  int s = (c >> 7) & 1, e = (c >> 3) & 0xF, m = c & 7;
  double v;
  if (e == 15 && m == 7) v = NAN;
  else if (e == 0) v = ldexp((double)m, -9);
  else v = ldexp(1.0 + m / 8.0, e - 7);
  return (float)(s ? -v : v);
}

/* ---------------------------------- E2M1 --------------------------------- */

/* 4-bit code: bit 3 sign, bits 2..1 exponent (bias 1), bit 0 mantissa.
 * Saturating to +-6.  The sign bit follows the sign of the input, so an input
 * that rounds to zero from below encodes as 0x8 (negative zero). */
uint8_t orc_f32_to_e2m1_satfinite(float xf) {
  double x = (double)xf;
  if (isnan(x)) return 0x7; /* no NaN in E2M1; never reached by the method */
  uint8_t sign = signbit(x) ? 0x8 : 0;
  double y = fabs(rne_to_grid(x, 2, 0));
  if (y > 6.0 || isinf(y)) y = 6.0;
  if (y == 0.0) return sign;
  if (y < 1.0) return sign | 0x1; /* the single subnormal, 0.5 */
  int e2;
  frexp(y, &e2);
  int E = e2 - 1;
  uint8_t mant = (uint8_t)((y / ldexp(1.0, E) - 1.0) * 2.0);
  return sign | (uint8_t)((E + 1) << 1) | mant;
}

float orc_e2m1_to_f32(uint8_t c) {
  int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
  double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return (float)(s ? -v : v);
}

/* Vector forms, for exhaustive codec tests. */
void orc_vec_f64_to_bf16(int64_t n, const double* x, uint16_t* o) { for (int64_t i = 0; i < n; ++i) o[i] = orc_f64_to_bf16(x[i]); }
void orc_vec_f32_to_bf16(int64_t n, const float* x, uint16_t* o) { for (int64_t i = 0; i < n; ++i) o[i] = orc_f32_to_bf16(x[i]); }
void orc_vec_f32_to_f16(int64_t n, const float* x, uint16_t* o) { for (int64_t i = 0; i < n; ++i) o[i] = orc_f32_to_f16(x[i]); }
void orc_vec_f16_to_f32(int64_t n, const uint16_t* x, float* o) { for (int64_t i = 0; i < n; ++i) o[i] = orc_f16_to_f32(x[i]); }
void orc_vec_f32_to_e4m3(int64_t n, const float* x, uint8_t* o) { for (int64_t i = 0; i < n; ++i) o[i] = orc_f32_to_e4m3_satfinite(x[i]); }
void orc_vec_e4m3_to_f32(int64_t n, const uint8_t* x, float* o) { for (int64_t i = 0; i < n; ++i) o[i] = orc_e4m3_to_f32(x[i]); }
void orc_vec_f32_to_e2m1(int64_t n, const float* x, uint8_t* o) { for (int64_t i = 0; i < n; ++i) o[i] = orc_f32_to_e2m1_satfinite(x[i]); }
void orc_vec_e2m1_to_f32(int64_t n, const uint8_t* x, float* o) { for (int64_t i = 0; i < n; ++i) o[i] = orc_e2m1_to_f32(x[i]); }

/* ------------------------------------------------------------------------- */
/* Smoothing (outlier migration) -- [P5] "Суть метода": activation outliers   */
/* are moved into the weights.  Reading: per input channel j,                 */
/*   lambda_j = amax_x[j]^alpha / amax_w[j]^(1-alpha),                       */
/* lambda_j = 1 when either statistic is 0.  X^ = X / lambda, W^ = W * lambda. */
/* ------------------------------------------------------------------------- */
void orc_smooth_factors(int64_t K, const float* amax_x, const float* amax_w, double alpha,
                        double* lambda_d, float* lambda_f, float* inv_lambda_f) {
  for (int64_t j = 0; j < K; ++j) {
    double ax = amax_x[j], aw = amax_w[j];
    double lam = (ax > 0.0 && aw > 0.0) ? pow(ax, alpha) / pow(aw, 1.0 - alpha) : 1.0;
    lambda_d[j] = lam;
    lambda_f[j] = (float)lam;
    inv_lambda_f[j] = (float)(1.0 / lam);
  }
}

/* x^[m,k] = float(x[m,k]) * inv_lambda[k], one binary32 multiply. */
void orc_smooth_act(int64_t M, int64_t K, const uint16_t* X, const float* inv_lambda, float* xhat) {
  #pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      float x = orc_bf16_to_f32(X[m * K + k]);
      volatile float p = x * inv_lambda[k];
      xhat[m * K + k] = p;
    }
}

/* ------------------------------------------------------------------------- */
/* 4-bit group quantizers -- [P5] "Суть метода" (4-bit activations and       */
/* residual), next paragraph (INT4 and NVFP4 variants).                       */
/* Packing: two codes per byte, element 2i in bits 0..3, 2i+1 in bits 4..7.   */
/* ------------------------------------------------------------------------- */

/* INT4, groups of 64 along K.  Per group:
 *   s = fp16_rne(amax / 7)  (binary32 division), S = float(s)
 *   S == 0 -> all codes 0
 *   else inv = 1/S (binary32), q = clamp(rne_integer(v * inv), -8, 7)
 * Codes are two's-complement nibbles. */
void orc_quant_int4_rows(int64_t rows, int64_t K, const float* v, uint8_t* codes, uint16_t* scales) {
  const int64_t G = K / 64;
  #pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < rows; ++m) {
    for (int64_t g = 0; g < G; ++g) {
      const float* x = v + m * K + g * 64;
      float amax = 0.0f;
      for (int i = 0; i < 64; ++i) { float a = fabsf(x[i]); if (a > amax) amax = a; }
      volatile float q7 = amax / 7.0f;
      uint16_t s = orc_f32_to_f16(q7);
      scales[m * G + g] = s;
      float S = orc_f16_to_f32(s);
      for (int i = 0; i < 64; i += 2) {
        int q[2] = {0, 0};
        if (S != 0.0f) {
          volatile float inv = 1.0f / S;
          for (int h = 0; h < 2; ++h) {
            volatile float p = x[i + h] * inv;
            double r = nearbyint((double)p);
            if (r < -8.0) r = -8.0;
            if (r > 7.0) r = 7.0;
            q[h] = (int)r;
          }
        }
        codes[m * (K / 2) + (g * 64 + i) / 2] = (uint8_t)((q[0] & 0xF) | ((q[1] & 0xF) << 4));
      }
    }
  }
}

/* NVFP4, blocks of 16 along K, per-tensor binary32 scale g.  Per block:
 *   sb = e4m3_rne_satfinite(amax / (6 g))   (6 g formed once in binary32)
 *   d  = float(sb) * g                      (binary32)
 *   sb == 0 -> all codes +0
 *   else inv = 1/d (binary32), code = e2m1_rne_satfinite(v * inv)
 */
void orc_quant_nvfp4_rows(int64_t rows, int64_t K, const float* v, float g, uint8_t* codes, uint8_t* scales) {
  const int64_t B = K / 16;
  const float den = 6.0f * g;
  #pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < rows; ++m) {
    for (int64_t b = 0; b < B; ++b) {
      const float* x = v + m * K + b * 16;
      float amax = 0.0f;
      for (int i = 0; i < 16; ++i) { float a = fabsf(x[i]); if (a > amax) amax = a; }
      volatile float ratio = amax / den;
      uint8_t sb = orc_f32_to_e4m3_satfinite(ratio);
      scales[m * B + b] = sb;
      volatile float d = orc_e4m3_to_f32(sb) * g;
      for (int i = 0; i < 16; i += 2) {
        uint8_t c[2] = {0, 0};
        if (sb != 0) {
          volatile float inv = 1.0f / d;
          for (int h = 0; h < 2; ++h) {
            volatile float p = x[i + h] * inv;
            c[h] = orc_f32_to_e2m1_satfinite(p);
          }
        }
        codes[m * (K / 2) + (b * 16 + i) / 2] = (uint8_t)(c[0] | (c[1] << 4));
      }
    }
  }
}

static int nib_int4(uint8_t byte, int hi) {
  int v = hi ? (byte >> 4) : (byte & 0xF);
  return v >= 8 ? v - 16 : v;
}
static double nib_e2m1(uint8_t byte, int hi) {
  return (double)orc_e2m1_to_f32(hi ? (byte >> 4) : (byte & 0xF));
}

/* Decode packed codes + scales back to values (double), row-major [rows, K]. */
void orc_dequant_int4_rows(int64_t rows, int64_t K, const uint8_t* codes, const uint16_t* scales, double* out) {
  const int64_t G = K / 64;
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t k = 0; k < K; ++k) {
      double S = (double)orc_f16_to_f32(scales[m * G + k / 64]);
      out[m * K + k] = S * nib_int4(codes[m * (K / 2) + k / 2], (int)(k & 1));
    }
}

void orc_dequant_nvfp4_rows(int64_t rows, int64_t K, const uint8_t* codes, const uint8_t* scales, float g, double* out) {
  const int64_t B = K / 16;
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t k = 0; k < K; ++k) {
      double d = (double)orc_e4m3_to_f32(scales[m * B + k / 16]) * (double)g;
      out[m * K + k] = d * nib_e2m1(codes[m * (K / 2) + k / 2], (int)(k & 1));
    }
}

/* ------------------------------------------------------------------------- */
/* Low-rank down-projection -- [P5] "Суть метода": 16-bit low-rank branch.    */
/*   t[m,j] = bf16_rne( sum_k bf16(x^[m,k]) * L1[k,j] ), sum in double.      */
/* ------------------------------------------------------------------------- */
void orc_lowrank_down(int64_t M, int64_t K, int64_t r, const float* xhat, const uint16_t* L1, uint16_t* t) {
  if (r > 512) return; /* ranks above 512 are not part of the method's use here */
  #pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m) {
    double acc[512];
    for (int64_t j = 0; j < r; ++j) acc[j] = 0.0;
    for (int64_t k = 0; k < K; ++k) {
      double xb = (double)orc_bf16_to_f32(orc_f32_to_bf16(xhat[m * K + k]));
      for (int64_t j = 0; j < r; ++j) acc[j] += xb * (double)orc_bf16_to_f32(L1[k * r + j]);
    }
    for (int64_t j = 0; j < r; ++j) t[m * r + j] = orc_f64_to_bf16(acc[j]);
  }
}

/* ------------------------------------------------------------------------- */
/* Main W4A4 product and output -- [P5] "Суть метода".                        */
/* ------------------------------------------------------------------------- */

/* INT4: acc_g[m,n] = sum over the 64 k of group g of qx * qw (exact integers). */
void orc_int4_group_acc(int64_t M, int64_t N, int64_t K, const uint8_t* xcodes, const uint8_t* wcodes, int32_t* acc /*[K/64, M, N]*/) {
  const int64_t G = K / 64;
  for (int64_t g = 0; g < G; ++g)
    for (int64_t m = 0; m < M; ++m)
      for (int64_t n = 0; n < N; ++n) {
        int64_t s = 0;
        for (int64_t k = g * 64; k < g * 64 + 64; ++k)
          s += (int64_t)nib_int4(xcodes[m * (K / 2) + k / 2], (int)(k & 1)) *
               (int64_t)nib_int4(wcodes[n * (K / 2) + k / 2], (int)(k & 1));
        acc[(g * M + m) * N + n] = (int32_t)s;
      }
}

/* Code value of one nibble as a small integer: INT4 -> q, E2M1 -> 2*value
 * (E2M1 values are multiples of 0.5, so 2*value is an integer in [-12, 12]). */
static void decode_codes_int(int64_t rows, int64_t K, const uint8_t* codes, int fmt, int8_t* out) {
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = codes[m * (K / 2) + k / 2];
      int hi = (int)(k & 1);
      out[m * K + k] = (int8_t)(fmt == 1 ? nib_int4(byte, hi) : (int)(2.0 * nib_e2m1(byte, hi)));
    }
}

/* y[m,n] = main[m,n] + sum_j t[m,j] L2[j,n] + bias[n], in double, then bf16_rne.
 *   INT4 : main = sum_g float(sx[m,g]) float(sw[n,g]) acc_g[m,n]
 *   NVFP4: main = g_x g_w sum_b float(sbx[m,b]) float(sbw[n,b]) sum_{k in b} e2m1(qx) e2m1(qw)
 * Every group / block sum is an exact integer (E2M1 handled as 2*value), so the
 * only roundings are the double accumulation across groups and the final bf16.
 * Writes y_f64 (optional) and y_bf16.  Rows are independent (OpenMP over m). */
void orc_forward_out(int64_t M, int64_t N, int64_t K, int64_t r, int fmt /*1 = INT4, 2 = NVFP4*/,
                     const uint8_t* xcodes, const void* xscales, const uint8_t* wcodes, const void* wscales,
                     float g_x, float g_w, const uint16_t* t, const uint16_t* L2, const uint16_t* bias,
                     double* y_f64, uint16_t* y_bf16) {
  int8_t* qx = (int8_t*)malloc((size_t)(M * K > 0 ? M * K : 1));
  int8_t* qw = (int8_t*)malloc((size_t)(N * K > 0 ? N * K : 1));
  decode_codes_int(M, K, xcodes, fmt, qx);
  decode_codes_int(N, K, wcodes, fmt, qw);
  const int64_t gs = (fmt == 1) ? 64 : 16;
  const int64_t G = K / gs;
  double* sxd = (double*)malloc(sizeof(double) * (size_t)(M * G > 0 ? M * G : 1));
  double* swd = (double*)malloc(sizeof(double) * (size_t)(N * G > 0 ? N * G : 1));
  for (int64_t i = 0; i < M * G; ++i)
    sxd[i] = fmt == 1 ? (double)orc_f16_to_f32(((const uint16_t*)xscales)[i]) : (double)orc_e4m3_to_f32(((const uint8_t*)xscales)[i]);
  for (int64_t i = 0; i < N * G; ++i)
    swd[i] = fmt == 1 ? (double)orc_f16_to_f32(((const uint16_t*)wscales)[i]) : (double)orc_e4m3_to_f32(((const uint8_t*)wscales)[i]);
  #pragma omp parallel for schedule(dynamic, 1)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      double main_ = 0.0;
      for (int64_t g = 0; g < G; ++g) {
        int64_t s = 0;
        const int8_t* a = qx + m * K + g * gs;
        const int8_t* b = qw + n * K + g * gs;
        for (int64_t i = 0; i < gs; ++i) s += (int64_t)a[i] * (int64_t)b[i];
        double blk = (fmt == 1) ? (double)s : (double)s * 0.25; /* undo the two factors of 2 */
        main_ += sxd[m * G + g] * swd[n * G + g] * blk;
      }
      if (fmt != 1) main_ = (double)g_x * (double)g_w * main_;
      double lr = 0.0;
      for (int64_t j = 0; j < r; ++j)
        lr += (double)orc_bf16_to_f32(t[m * r + j]) * (double)orc_bf16_to_f32(L2[j * N + n]);
      double y = main_ + lr + (bias ? (double)orc_bf16_to_f32(bias[n]) : 0.0);
      if (y_f64) y_f64[m * N + n] = y;
      y_bf16[m * N + n] = orc_f64_to_bf16(y);
    }
  }
  free(qx); free(qw); free(sxd); free(swd);
}

int orc_num_threads(void) {
#ifdef _OPENMP
  extern int omp_get_max_threads(void);
  return omp_get_max_threads();
#else
  return 1;
#endif
}
