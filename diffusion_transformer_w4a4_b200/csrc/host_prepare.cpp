// Host half of libsvdq: offline preparation of one svdq_w4a4 layer and the
// re-layout of the prepared weights into the blob the kernels read.
//
// Method ("Hugging Face встроила Nunchaku в Diffusers ...", paragraph
// "Суть метода"): move activation outliers into the weights with per-channel
// smoothing factors, keep the hardest part of the smoothed weight in a 16-bit
// rank-r branch, quantize the residual to 4 bits (INT4 or NVFP4 variant, next
// paragraph).  The truncated SVD is a randomized subspace iteration
// (Halko, Martinsson & Tropp 2011, "Finding structure with randomness",
// algorithm 4.4) followed by a one-sided Jacobi SVD (Hestenes) of the small
// projected matrix, all in binary64.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <random>
#include <thread>
#include <vector>

#include "svdq_internal.h"

namespace svdq {
namespace host {

// ------------------------------------------------------------------ codecs
// All conversions round to nearest, ties to even, implemented on the bit
// patterns of binary32.

uint16_t f32_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return 0x7FC0;  // NaN
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// binary64 -> bf16 with a single rounding: split off the bits below the bf16
// significand of the binary64 value.
uint16_t f64_to_bf16(double x) {
  if (std::isnan(x)) return 0x7FC0;
  uint64_t u;
  std::memcpy(&u, &x, 8);
  const uint64_t sign = u >> 63;
  const int bexp = (int)((u >> 52) & 0x7FF);
  if (bexp == 0x7FF) return (uint16_t)((sign << 15) | 0x7F80);
  const int e = bexp - 1023;  // unbiased exponent (binary64 subnormals are far below bf16 range)
  if (bexp == 0 || e < -134) return (uint16_t)(sign << 15);
  // significand with hidden bit: 53 bits
  uint64_t sig = (u & ((1ull << 52) - 1)) | (1ull << 52);
  // target spacing exponent: bf16 normal -> e - 7, subnormal -> -133
  int q = (e >= -126) ? e - 7 : -133;
  int shift = (52 + q) - e;  // number of low bits of sig below the target spacing
  // e >= -134 here, so 45 <= shift <= 53
  uint64_t keep = sig >> shift;
  uint64_t rem = sig & ((1ull << shift) - 1);
  uint64_t half = 1ull << (shift - 1);
  if (rem > half || (rem == half && (keep & 1))) keep += 1;
  // value = keep * 2^q
  double v = std::ldexp((double)keep, q);
  if (v >= std::ldexp(1.0, 128)) return (uint16_t)((sign << 15) | 0x7F80);
  float vf = (float)v;  // exact
  uint16_t h = f32_to_bf16(vf);
  return (uint16_t)(h | (sign << 15));
}

uint16_t f32_to_f16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint32_t sign = (u >> 16) & 0x8000u;
  const uint32_t absu = u & 0x7FFFFFFFu;
  if (absu > 0x7F800000u) return (uint16_t)(sign | 0x7E00u);
  if (absu >= 0x477FF000u) return (uint16_t)(sign | 0x7C00u);  // >= 65520: rounds to inf
  if (absu < 0x33000000u) return (uint16_t)sign;                // < 2^-25: rounds to 0 (tie -> even 0)
  int e = (int)(absu >> 23) - 127;
  uint32_t sig = (absu & 0x7FFFFFu) | 0x800000u;
  int shift = (e >= -14) ? 13 : 13 + (-14 - e);  // bits dropped below fp16 spacing
  uint32_t keep = sig >> shift;
  uint32_t rem = sig & ((1u << shift) - 1);
  uint32_t half = 1u << (shift - 1);
  if (rem > half || (rem == half && (keep & 1))) keep += 1;
  if (e >= -14) {
    // keep has 11 or 12 bits (carry); exponent field = e + 15, add carries naturally
    uint32_t bits = ((uint32_t)(e + 15) << 10) + (keep - 0x400u);
    return (uint16_t)(sign | bits);
  }
  return (uint16_t)(sign | keep);  // subnormal (a carry into 0x400 is the min normal)
}

float f16_to_f32(uint16_t h) {
  uint32_t s = (h >> 15) & 1, e = (h >> 10) & 0x1F, m = h & 0x3FF;
  float v;
  if (e == 0) v = std::ldexp((float)m, -24);
  else if (e == 31) v = m ? NAN : INFINITY;
  else v = std::ldexp((float)(m | 0x400), (int)e - 25);
  return s ? -v : v;
}

// The E4M3 byte of a small integer (exact for |v| <= 16).
uint8_t int_to_e4m3(int v) { return f32_to_e4m3_sat((float)v); }

// E4M3 (OCP FP8), saturating to +-448.
uint8_t f32_to_e4m3_sat(float f) {
  if (std::isnan(f)) return 0x7F;
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint8_t sign = (uint8_t)((u >> 24) & 0x80);
  float a = std::fabs(f);
  if (a >= 464.0f) return (uint8_t)(sign | 0x7E);  // 464 ties to 448 (even), above saturates
  uint32_t au;
  std::memcpy(&au, &a, 4);
  if (au < 0x3A000000u) return sign;  // < 2^-11 ... handled generally below too
  int e = (int)(au >> 23) - 127;
  uint32_t sig = (au & 0x7FFFFFu) | 0x800000u;
  int shift = (e >= -6) ? 20 : 20 + (-6 - e);
  if (shift > 31) return sign;
  uint32_t keep = sig >> shift;
  uint32_t rem = sig & ((1u << shift) - 1);
  uint32_t half = 1u << (shift - 1);
  if (rem > half || (rem == half && (keep & 1))) keep += 1;
  if (e >= -6) {
    uint32_t bits = ((uint32_t)(e + 7) << 3) + (keep - 8u);
    if (bits > 0x7E) bits = 0x7E;
    return (uint8_t)(sign | bits);
  }
  return (uint8_t)(sign | keep);
}

float e4m3_to_f32(uint8_t c) {
  int s = (c >> 7) & 1, e = (c >> 3) & 0xF, m = c & 7;
  float v;
  if (e == 15 && m == 7) v = NAN;
  else if (e == 0) v = std::ldexp((float)m, -9);
  else v = std::ldexp((float)(8 + m), e - 10);
  return s ? -v : v;
}

// E2M1 (OCP MX FP4), saturating to +-6, sign of zero follows the input.
uint8_t f32_to_e2m1_sat(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  const uint8_t sign = (uint8_t)((u >> 28) & 0x8);
  float a = std::fabs(f);
  // decision thresholds between neighbours {0,.5,1,1.5,2,3,4,6}; ties to even code
  uint8_t c;
  if (a <= 0.25f) c = 0;
  else if (a < 0.75f) c = 1;
  else if (a <= 1.25f) c = 2;
  else if (a < 1.75f) c = 3;
  else if (a <= 2.5f) c = 4;
  else if (a < 3.5f) c = 5;
  else if (a <= 5.0f) c = 6;
  else c = 7;
  return (uint8_t)(sign | c);
}

// ------------------------------------------------------------------ quantizers
// Same definitions as the GPU activation quantizer (binary32 arithmetic).
void quant_int4_rows(int64_t rows, int64_t K, const float* v, uint8_t* codes, uint16_t* scales) {
  const int64_t G = K / 64;
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t g = 0; g < G; ++g) {
      const float* x = v + m * K + g * 64;
      float amax = 0.f;
      for (int i = 0; i < 64; ++i) amax = std::max(amax, std::fabs(x[i]));
      uint16_t s = f32_to_f16(amax / 7.0f);
      scales[m * G + g] = s;
      float S = f16_to_f32(s);
      float inv = (S != 0.f) ? 1.0f / S : 0.f;
      for (int i = 0; i < 64; i += 2) {
        int q0 = 0, q1 = 0;
        if (S != 0.f) {
          q0 = (int)std::nearbyint(std::min(7.f, std::max(-8.f, x[i] * inv)));
          q1 = (int)std::nearbyint(std::min(7.f, std::max(-8.f, x[i + 1] * inv)));
        }
        codes[m * (K / 2) + (g * 64 + i) / 2] = (uint8_t)((q0 & 0xF) | ((q1 & 0xF) << 4));
      }
    }
}

void quant_nvfp4_rows(int64_t rows, int64_t K, const float* v, float g, uint8_t* codes, uint8_t* scales) {
  const int64_t B = K / 16;
  const float den = 6.0f * g;
  for (int64_t m = 0; m < rows; ++m)
    for (int64_t b = 0; b < B; ++b) {
      const float* x = v + m * K + b * 16;
      float amax = 0.f;
      for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(x[i]));
      uint8_t sb = f32_to_e4m3_sat(amax / den);
      scales[m * B + b] = sb;
      float d = e4m3_to_f32(sb) * g;
      float inv = (sb != 0) ? 1.0f / d : 0.f;
      for (int i = 0; i < 16; i += 2) {
        uint8_t c0 = 0, c1 = 0;
        if (sb != 0) {
          c0 = f32_to_e2m1_sat(x[i] * inv);
          c1 = f32_to_e2m1_sat(x[i + 1] * inv);
        }
        codes[m * (K / 2) + (b * 16 + i) / 2] = (uint8_t)(c0 | (c1 << 4));
      }
    }
}

// Smallest power of two >= amax / (6 * 448): the per-tensor NVFP4 scale that
// keeps every block scale amax_b / (6 g) within E4M3's 448.
float nvfp4_tensor_scale(float amax) {
  double a = (double)amax / 2688.0;
  if (!(a > 0.0)) return 1.0f;
  int e;
  double m = std::frexp(a, &e);  // a = m 2^e, m in [0.5,1)
  return (float)std::ldexp(1.0, (m == 0.5) ? e - 1 : e);
}

// ------------------------------------------------------------------ dense helpers
static int host_threads() {
  unsigned n = std::thread::hardware_concurrency();
  return (int)std::max(1u, std::min(n, 64u));
}

template <class F>
static void parallel_for(int64_t n, F f) {
  int T = host_threads();
  if (n < 2 * T) T = 1;
  std::vector<std::thread> th;
  for (int t = 0; t < T; ++t)
    th.emplace_back([=] {
      int64_t lo = n * t / T, hi = n * (t + 1) / T;
      for (int64_t i = lo; i < hi; ++i) f(i);
    });
  for (auto& x : th) x.join();
}

// Y[N,l] = A[N,K] X[K,l]
static void mm_A_X(const double* A, int64_t N, int64_t K, const double* X, int l, double* Y) {
  parallel_for(N, [&](int64_t n) {
    double* y = Y + n * l;
    for (int j = 0; j < l; ++j) y[j] = 0.0;
    const double* a = A + n * K;
    for (int64_t k = 0; k < K; ++k) {
      const double av = a[k];
      const double* x = X + k * l;
      for (int j = 0; j < l; ++j) y[j] += av * x[j];
    }
  });
}

// Z[K,l] = A[N,K]^T Q[N,l]
static void mm_At_Q(const double* A, int64_t N, int64_t K, const double* Q, int l, double* Z) {
  const int64_t KB = 64;
  const int64_t nblk = (K + KB - 1) / KB;
  parallel_for(nblk, [&](int64_t b) {
    int64_t k0 = b * KB, k1 = std::min(K, k0 + KB);
    for (int64_t k = k0; k < k1; ++k)
      for (int j = 0; j < l; ++j) Z[k * l + j] = 0.0;
    for (int64_t n = 0; n < N; ++n) {
      const double* q = Q + n * l;
      const double* a = A + n * K;
      for (int64_t k = k0; k < k1; ++k) {
        const double av = a[k];
        double* z = Z + k * l;
        for (int j = 0; j < l; ++j) z[j] += av * q[j];
      }
    }
  });
}

// Orthonormalize the l columns of Y [rows, l] in place (Gram-Schmidt, two passes).
static void orthonormalize(double* Y, int64_t rows, int l) {
  for (int j = 0; j < l; ++j) {
    for (int pass = 0; pass < 2; ++pass)
      for (int i = 0; i < j; ++i) {
        double d = 0.0;
        for (int64_t r = 0; r < rows; ++r) d += Y[r * l + i] * Y[r * l + j];
        for (int64_t r = 0; r < rows; ++r) Y[r * l + j] -= d * Y[r * l + i];
      }
    double nrm = 0.0;
    for (int64_t r = 0; r < rows; ++r) nrm += Y[r * l + j] * Y[r * l + j];
    nrm = std::sqrt(nrm);
    double inv = nrm > 0 ? 1.0 / nrm : 0.0;
    for (int64_t r = 0; r < rows; ++r) Y[r * l + j] *= inv;
  }
}

// One-sided Jacobi on the columns of A [rows, l] (in place): on return the
// columns are mutually orthogonal and V [l,l] holds the accumulated rotations,
// so A_in = A_out V^T.
static void one_sided_jacobi(double* A, int64_t rows, int l, double* V) {
  for (int i = 0; i < l * l; ++i) V[i] = 0.0;
  for (int i = 0; i < l; ++i) V[i * l + i] = 1.0;
  for (int sweep = 0; sweep < 60; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < l - 1; ++p)
      for (int q = p + 1; q < l; ++q) {
        double alpha = 0, beta = 0, gamma = 0;
        for (int64_t r = 0; r < rows; ++r) {
          double ap = A[r * l + p], aq = A[r * l + q];
          alpha += ap * ap;
          beta += aq * aq;
          gamma += ap * aq;
        }
        if (gamma == 0.0) continue;
        double rel = std::fabs(gamma) / std::sqrt(alpha * beta);
        off = std::max(off, rel);
        if (rel < 1e-15) continue;
        double zeta = (beta - alpha) / (2.0 * gamma);
        double t = (zeta >= 0 ? 1.0 : -1.0) / (std::fabs(zeta) + std::sqrt(1.0 + zeta * zeta));
        double c = 1.0 / std::sqrt(1.0 + t * t), s = c * t;
        for (int64_t r = 0; r < rows; ++r) {
          double ap = A[r * l + p], aq = A[r * l + q];
          A[r * l + p] = c * ap - s * aq;
          A[r * l + q] = s * ap + c * aq;
        }
        for (int r = 0; r < l; ++r) {
          double vp = V[r * l + p], vq = V[r * l + q];
          V[r * l + p] = c * vp - s * vq;
          V[r * l + q] = s * vp + c * vq;
        }
      }
    if (off < 1e-15) break;
  }
}

// Rank-r factors of What [N,K] (binary64): L1 [K,r] = V_r S^(1/2), L2 [r,N] = S^(1/2) U_r^T.
static void truncated_svd(const double* What, int64_t N, int64_t K, int r, double* L1, double* L2) {
  const int l = std::min<int64_t>(std::min(N, K), r + std::max(16, r / 2));
  const int q_iters = 8;
  std::vector<double> Om((size_t)K * l), Y((size_t)N * l), Z((size_t)K * l);
  std::mt19937_64 gen(0x5eed);
  std::normal_distribution<double> nd(0.0, 1.0);
  for (auto& x : Om) x = nd(gen);
  mm_A_X(What, N, K, Om.data(), l, Y.data());
  orthonormalize(Y.data(), N, l);
  for (int it = 0; it < q_iters; ++it) {
    mm_At_Q(What, N, K, Y.data(), l, Z.data());
    orthonormalize(Z.data(), K, l);
    mm_A_X(What, N, K, Z.data(), l, Y.data());
    orthonormalize(Y.data(), N, l);
  }
  // B^T = What^T Q  [K, l]; B = Q^T What.  One-sided Jacobi: B^T = W' Vj^T with
  // orthogonal columns W' (norms = singular values), so B = Vj W'^T.
  mm_At_Q(What, N, K, Y.data(), l, Z.data());
  std::vector<double> Vj((size_t)l * l);
  one_sided_jacobi(Z.data(), K, l, Vj.data());
  std::vector<double> sig(l);
  for (int j = 0; j < l; ++j) {
    double s = 0;
    for (int64_t k = 0; k < K; ++k) s += Z[k * l + j] * Z[k * l + j];
    sig[j] = std::sqrt(s);
  }
  std::vector<int> order(l);
  for (int j = 0; j < l; ++j) order[j] = j;
  std::sort(order.begin(), order.end(), [&](int a, int b) { return sig[a] > sig[b]; });
  for (int jj = 0; jj < r; ++jj) {
    const int j = order[jj];
    const double s = sig[j];
    // u = Q Vj[:, j]  (left vector), v = Z[:, j] / s (right vector)
    std::vector<double> u(N);
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0;
      for (int i = 0; i < l; ++i) acc += Y[n * l + i] * Vj[i * l + j];
      u[n] = acc;
    }
    int64_t imax = 0;
    for (int64_t n = 1; n < N; ++n)
      if (std::fabs(u[n]) > std::fabs(u[imax])) imax = n;
    const double sgn = u[imax] < 0 ? -1.0 : 1.0;
    const double rs = std::sqrt(s);
    for (int64_t n = 0; n < N; ++n) L2[(int64_t)jj * N + n] = sgn * rs * u[n];
    for (int64_t k = 0; k < K; ++k) L1[k * r + jj] = (s > 0 ? sgn * Z[k * l + j] / s * rs : 0.0);
  }
}

int prepare(const uint16_t* W, const uint16_t* bias, const float* act_absmax, float alpha, svdq_canonical* c) {
  const int64_t N = c->N, K = c->K;
  const int r = c->rank;
  const int fmt = c->fmt;
  for (int64_t j = 0; j < K; ++j)
    if (!std::isfinite(act_absmax[j]) || act_absmax[j] < 0) return SVDQ_ERR_NUMERIC;
  std::vector<float> amax_w(K, 0.f);
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) {
      float w = bf16_to_f32(W[n * K + k]);
      if (!std::isfinite(w)) return SVDQ_ERR_NUMERIC;
      amax_w[k] = std::max(amax_w[k], std::fabs(w));
    }
  for (int64_t k = 0; k < K; ++k) {
    double ax = act_absmax[k], aw = amax_w[k];
    double lam = (ax > 0 && aw > 0) ? std::pow(ax, (double)alpha) / std::pow(aw, 1.0 - (double)alpha) : 1.0;
    c->lambda[k] = (float)lam;
    c->inv_lambda[k] = (float)(1.0 / lam);
  }
  std::vector<double> What;
  try {
    What.resize((size_t)N * K);
  } catch (const std::bad_alloc&) {
    return SVDQ_ERR_OOM;
  }
  parallel_for(N, [&](int64_t n) {
    for (int64_t k = 0; k < K; ++k) What[n * K + k] = (double)bf16_to_f32(W[n * K + k]) * (double)c->lambda[k];
  });
  std::vector<float> R((size_t)N * K);
  if (r > 0) {
    std::vector<double> L1d((size_t)K * r), L2d((size_t)r * N);
    truncated_svd(What.data(), N, K, r, L1d.data(), L2d.data());
    for (size_t i = 0; i < L1d.size(); ++i) c->L1[i] = f64_to_bf16(L1d[i]);
    for (size_t i = 0; i < L2d.size(); ++i) c->L2[i] = f64_to_bf16(L2d[i]);
    std::vector<double> L1r((size_t)K * r);
    for (size_t i = 0; i < L1r.size(); ++i) L1r[i] = bf16_to_f32(c->L1[i]);
    std::vector<double> L2r((size_t)r * N);
    for (size_t i = 0; i < L2r.size(); ++i) L2r[i] = bf16_to_f32(c->L2[i]);
    parallel_for(N, [&](int64_t n) {
      for (int64_t k = 0; k < K; ++k) {
        double lr = 0;
        for (int j = 0; j < r; ++j) lr += L1r[k * r + j] * L2r[(int64_t)j * N + n];
        R[n * K + k] = (float)(What[n * K + k] - lr);
      }
    });
  } else {
    for (size_t i = 0; i < R.size(); ++i) R[i] = (float)What[i];
  }
  if (fmt == SVDQ_INT4_G64) {
    quant_int4_rows(N, K, R.data(), c->wcodes, (uint16_t*)c->wscales);
    c->g_w = 1.0f;
    c->g_x = 1.0f;
  } else {
    float amax = 0.f;
    for (float x : R) amax = std::max(amax, std::fabs(x));
    c->g_w = nvfp4_tensor_scale(amax);
    quant_nvfp4_rows(N, K, R.data(), c->g_w, c->wcodes, (uint8_t*)c->wscales);
    float xmax = 0.f;
    for (int64_t k = 0; k < K; ++k) xmax = std::max(xmax, act_absmax[k] * c->inv_lambda[k]);
    c->g_x = nvfp4_tensor_scale(xmax);
  }
  c->alpha = alpha;
  for (int64_t n = 0; n < N; ++n) c->bias[n] = bias ? bias[n] : (uint16_t)0;
  return SVDQ_OK;
}

// ------------------------------------------------------------------ awq_w4a16
// Activation-aware preparation of the 4-bit-weight / 16-bit-activation layer:
// s_j = mean|x_j|^alpha (1 where the mean is 0) for alpha = 0, 0.05, ..., 1;
// W diag(s) rounded to binary32 and quantized with the INT4 group-64
// quantizer above; the grid point with the smallest squared output error
// sum_mn ((f32(x) * inv_s) . deq^T - x . W^T)^2 on the calibration input (the
// first one on a tie) is kept.  Errors are summed per output row, then over rows
// in order, so the choice does not depend on the thread count.
int awq_prepare(const uint16_t* W, const uint16_t* bias, const uint16_t* X, int64_t Mc, svdq_awq_canonical* c) {
  const int64_t N = c->N, K = c->K, G = K / 64;
  for (int64_t i = 0; i < N * K; ++i)
    if (!std::isfinite(bf16_to_f32(W[i]))) return SVDQ_ERR_NUMERIC;
  for (int64_t i = 0; i < Mc * K; ++i)
    if (!std::isfinite(bf16_to_f32(X[i]))) return SVDQ_ERR_NUMERIC;
  std::vector<double> mabs(K, 0.0);
  for (int64_t m = 0; m < Mc; ++m)
    for (int64_t k = 0; k < K; ++k) mabs[k] += std::fabs((double)bf16_to_f32(X[m * K + k]));
  for (int64_t k = 0; k < K; ++k) mabs[k] /= (double)Mc;
  std::vector<float> xf(Mc * K);
  for (int64_t i = 0; i < Mc * K; ++i) xf[i] = bf16_to_f32(X[i]);
  std::vector<double> ref(Mc * N);
  parallel_for(N, [&](int64_t n) {
    for (int64_t m = 0; m < Mc; ++m) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += (double)xf[m * K + k] * (double)bf16_to_f32(W[n * K + k]);
      ref[m * N + n] = acc;
    }
  });
  auto scales_for = [&](double alpha, std::vector<float>& s_f, std::vector<float>& inv) {
    for (int64_t k = 0; k < K; ++k) {
      const double sd = mabs[k] > 0.0 ? std::pow(mabs[k], alpha) : 1.0;
      s_f[k] = (float)sd;
      inv[k] = (float)(1.0 / (double)s_f[k]);
    }
  };
  auto quant_row = [&](int64_t n, const std::vector<float>& s_f, std::vector<float>& ws, uint8_t* codes,
                       uint16_t* sc) {
    for (int64_t k = 0; k < K; ++k) ws[k] = (float)((double)bf16_to_f32(W[n * K + k]) * (double)s_f[k]);
    quant_int4_rows(1, K, ws.data(), codes, sc);
  };
  std::vector<float> s_f(K), inv(K);
  double best_err = INFINITY;
  int best = 0;
  std::vector<double> err_row(N);
  for (int i = 0; i <= 20; ++i) {
    const double alpha = i / 20.0;
    scales_for(alpha, s_f, inv);
    std::vector<float> xh(Mc * K);
    for (int64_t m = 0; m < Mc; ++m)
      for (int64_t k = 0; k < K; ++k) xh[m * K + k] = xf[m * K + k] * inv[k];  // binary32 product
    parallel_for(N, [&](int64_t n) {
      std::vector<float> ws(K);
      std::vector<uint8_t> codes(K / 2);
      std::vector<uint16_t> sc(G);
      quant_row(n, s_f, ws, codes.data(), sc.data());
      double e = 0.0;
      for (int64_t m = 0; m < Mc; ++m) {
        double acc = 0.0;
        for (int64_t k = 0; k < K; ++k) {
          const uint8_t b = codes[k / 2];
          int q = (k & 1) ? (b >> 4) : (b & 15);
          if (q >= 8) q -= 16;
          acc += (double)xh[m * K + k] * ((double)q * (double)f16_to_f32(sc[k / 64]));
        }
        const double d = acc - ref[m * N + n];
        e += d * d;
      }
      err_row[n] = e;
    });
    double err = 0.0;
    for (int64_t n = 0; n < N; ++n) err += err_row[n];
    if (err < best_err) {
      best_err = err;
      best = i;
    }
  }
  const double alpha = best / 20.0;
  c->alpha = (float)alpha;
  scales_for(alpha, s_f, inv);
  std::memcpy(c->s, s_f.data(), K * 4);
  std::memcpy(c->inv_s, inv.data(), K * 4);
  parallel_for(N, [&](int64_t n) {
    std::vector<float> ws(K);
    quant_row(n, s_f, ws, c->wcodes + n * (K / 2), c->wscales + n * G);
  });
  for (int64_t n = 0; n < N; ++n) c->bias[n] = bias ? bias[n] : 0;
  return SVDQ_OK;
}

}  // namespace host
}  // namespace svdq
