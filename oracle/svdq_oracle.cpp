// SVDQuant W4A4 linear -- CPU ORACLE.  TEST INFRASTRUCTURE ONLY.
//
// This file is the plain, slow, obviously-correct statement of what the
// SVDQuant 4-bit linear layer computes.  Only the tests, the smoke check and
// the benchmark's CPU-baseline leg may load it; the product path never does.
// It shares no code, header, table or constant with the CUDA library.
//
// Method (SVDQuant, "Absorbing outliers by low-rank components for 4-bit
// diffusion models", abstract as translated on ai-digest.ru; the principles
// section of chattools.cn article 584):
//   * smoothing moves activation outliers into the weights:
//       lambda_j = max_i |X_ij|^0.5 / max_n |W_jn|^0.5,  Xh = X diag(lambda)^-1,
//       Wh = diag(lambda) W;
//   * a rank-r SVD of Wh gives a 16-bit low-rank branch L1 (K x r) = U_r S_r,
//     L2 (r x N) = V_r^T, and the residual R = Wh - L1 L2 (Eckart-Young-Mirsky:
//     removing the top r singular values leaves the smallest residual);
//   * the residual and the smoothed activation are quantised to 4 bits
//     (NVFP4: E2M1 values, one unsigned E4M3 scale per 16 consecutive
//     elements along K, scale = amax / 6);
//   * Y = Xh L1 L2 + Q(Xh) Q(R) (+ bias).
// Where the pages are silent (rounding order, layouts, zero groups) the
// reading taken is stated beside each function below.
//
// Arithmetic: fp64 everywhere except where a rounding step is part of the
// encoding contract (fp32 products/quotients of the quantiser, the bf16 and
// fp8/fp4 roundings), which are written out explicitly.
//
// Build: g++ -O2 -std=c++17 -fopenmp -ffp-contract=off -fPIC -shared

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

// ---------------------------------------------------------------- bf16 ----

float bf16_to_f32(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round a double once, to nearest-even, onto the bf16 grid (8 significant
// bits, fp32 exponent range).  Exact integer arithmetic on the scaled value.
uint16_t bf16_from_f64(double x) {
  if (x == 0.0) return std::signbit(x) ? 0x8000 : 0x0000;
  if (std::isnan(x)) return 0x7FC0;
  const bool neg = std::signbit(x);
  double a = std::fabs(x);
  int e = std::ilogb(a);            // a in [2^e, 2^(e+1))
  if (e < -126) e = -126;           // bf16 subnormal quantum 2^-133
  const double q = std::ldexp(1.0, e - 7);
  double n = std::nearbyint(a / q); // a/q exact (power-of-two scaling), RNE
  double v = n * q;
  float f = static_cast<float>(v);  // exact: v has <= 9 significant bits
  if (std::isinf(f) || v > 3.3895313892515355e38) f = INFINITY;
  uint32_t u;
  std::memcpy(&u, &f, 4);
  uint16_t b = static_cast<uint16_t>(u >> 16);
  return neg ? static_cast<uint16_t>(b | 0x8000) : b;
}

// ----------------------------------------------------------------- E4M3 ----
// OCP FP8 E4M3 ("FN"): 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no
// infinities, S.1111.111 = NaN, largest finite 448, subnormal step 2^-9.

double e4m3_decode(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = m * std::ldexp(1.0, -9);
  else v = (1.0 + m / 8.0) * std::ldexp(1.0, e - 7);
  return s ? -v : v;
}

// Round to nearest-even onto the E4M3 grid, saturating finite values to 448.
uint8_t e4m3_encode(float x) {
  if (std::isnan(x)) return 0x7F;
  const uint8_t sign = std::signbit(x) ? 0x80 : 0x00;
  double a = std::fabs(static_cast<double>(x));
  if (a >= 448.0) return sign | 0x7E;
  double q;  // spacing of the grid around a
  if (a < std::ldexp(1.0, -6)) q = std::ldexp(1.0, -9);
  else q = std::ldexp(1.0, std::ilogb(a) - 3);
  double n = std::nearbyint(a / q);
  double v = n * q;  // <= 448 because a < 448 and 448 is on the grid
  if (v < std::ldexp(1.0, -6)) return sign | static_cast<uint8_t>(n);  // n in [0, 8]
  int e = std::ilogb(v);
  int m = static_cast<int>(v / std::ldexp(1.0, e) * 8.0) - 8;
  return sign | static_cast<uint8_t>(((e + 7) << 3) | m);
}

// ----------------------------------------------------------------- E2M1 ----
// FP4 E2M1: magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} for codes 0..7, bit 3 sign.

const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double e2m1_decode(uint8_t c) {
  double v = kE2M1[c & 7];
  return (c & 8) ? -v : v;
}

// Round to nearest-even onto the E2M1 grid, saturating to 6; the sign of the
// input is kept, also when the magnitude rounds to zero.
uint8_t e2m1_encode(float x) {
  const uint8_t sign = std::signbit(x) ? 0x8 : 0x0;
  double a = std::fabs(static_cast<double>(x));
  if (std::isnan(x)) return 0x7;  // never produced by finite inputs
  if (a >= 6.0) return sign | 7;
  double q = a < 2.0 ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
  double v = std::nearbyint(a / q) * q;  // ties to even grid index = even code
  uint8_t code = 0;
  for (uint8_t i = 0; i < 8; ++i)
    if (kE2M1[i] == v) code = i;
  return sign | code;
}

// ------------------------------------------------- NVFP4 group quantiser ----
// One group of 16 values v (fp32):
//   amax = max |v_i|                      (exact)
//   s_f  = RN_f32(amax / 6)               (IEEE single division)
//   s    = E4M3_RNE_satfinite(s_f),  s_d = decode(s)
//   rcp  = 0 if s_d == 0 else RN_f32(1 / s_d)
//   q_i  = E2M1_RNE_satfinite(RN_f32(v_i * rcp))
void quantize_group(const float* v, int64_t stride, uint8_t* codes, uint8_t* scale) {
  float amax = 0.0f;
  for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(v[i * stride]));
  float sf = amax / 6.0f;
  uint8_t s = e4m3_encode(sf);
  double sd = e4m3_decode(s);
  float rcp = (sd == 0.0) ? 0.0f : 1.0f / static_cast<float>(sd);
  for (int i = 0; i < 16; ++i) {
    float p = v[i * stride] * rcp;
    codes[i] = e2m1_encode(p);
  }
  *scale = s;
}

// ------------------------------------------------------------------ GELU ----
// GELU(x) = x Phi(x) = 0.5 x (1 + erf(x / sqrt 2)), with erf from the purely
// rational approximation of Abramowitz and Stegun, Handbook of Mathematical
// Functions, formula 7.1.28 (|error| <= 3e-7 for x >= 0; erf is odd):
//   erf(z) ~ 1 - 1 / (1 + a1 z + a2 z^2 + a3 z^3 + a4 z^4 + a5 z^5 + a6 z^6)^16.
// Every step is one fp32 operation rounded to nearest (no fused multiply-add;
// this file is built with -ffp-contract=off), in this order:
//   z = |x| * RN(1/sqrt 2);  p = 1 + z(a1 + z(a2 + z(a3 + z(a4 + z(a5 + z a6)))))
//   (Horner, a multiply then an add per step);  p16 = (((p^2)^2)^2)^2;
//   e = 1 - 1/p16;  erf = e with the sign of x;  GELU = (0.5 x) (1 + erf).
constexpr float kAsA1 = 0.0705230784f, kAsA2 = 0.0422820123f, kAsA3 = 0.0092705272f;
constexpr float kAsA4 = 0.0001520143f, kAsA5 = 0.0002765672f, kAsA6 = 0.0000430638f;
constexpr float kRsqrt2 = 0.70710678118654752f;

float gelu_as(float x) {
  const float z = std::fabs(x) * kRsqrt2;
  float p = kAsA6;
  p = p * z;
  p = p + kAsA5;
  p = p * z;
  p = p + kAsA4;
  p = p * z;
  p = p + kAsA3;
  p = p * z;
  p = p + kAsA2;
  p = p * z;
  p = p + kAsA1;
  p = p * z;
  p = p + 1.0f;
  p = p * p;
  p = p * p;
  p = p * p;
  p = p * p;
  const float e = 1.0f - 1.0f / p;
  const float erf = std::signbit(x) ? -e : e;
  return (0.5f * x) * (1.0f + erf);
}

// ---------------------------------- NVFP4 with a per-tensor global scale ----
// Two-level scaling: the tensor carries one fp32 scale g > 0 on top of the
// per-16 E4M3 scales, and an element dequantises to q * decode(s) * g.  One
// group of 16 values v (fp32):
//   amax = max |v_i|
//   s_f  = RN_f32(amax / 6)
//   s    = E4M3_RNE_satfinite(RN_f32(s_f * RN_f32(1 / g)))
//   d    = RN_f32(decode(s) * g)                 (the group's whole scale)
//   rcp  = 0 if d == 0 else RN_f32(1 / d)
//   q_i  = E2M1_RNE_satfinite(RN_f32(v_i * rcp))
// With g = 1 this is quantize_group above.
void quantize_group_gs(const float* v, int64_t stride, float g, uint8_t* codes, uint8_t* scale) {
  float amax = 0.0f;
  for (int i = 0; i < 16; ++i) amax = std::max(amax, std::fabs(v[i * stride]));
  const float sf = amax / 6.0f;
  const float inv_g = 1.0f / g;
  const uint8_t s = e4m3_encode(sf * inv_g);
  const float d = static_cast<float>(e4m3_decode(s)) * g;
  const float rcp = (d == 0.0f) ? 0.0f : 1.0f / d;
  for (int i = 0; i < 16; ++i) codes[i] = e2m1_encode(v[i * stride] * rcp);
  *scale = s;
}

// ------------------------------------------------------------- layouts ----
// Codes: row-major [rows][K/2]; element k of a row sits in byte k/2, in the
// low nibble when k is even and in the high nibble when k is odd.
// Scales: the block-scaled MMA's 128 x 4 tile layout.  Rows are padded to a
// multiple of 128; tile (row/128, g/4) is 512 contiguous bytes, tiles of one
// 128-row band are consecutive along K; inside a tile the byte of (row, g) is
// (row % 32) * 16 + ((row % 128) / 32) * 4 + (g % 4).
int64_t scale_offset(int64_t row, int64_t g, int64_t K) {
  const int64_t tiles_k = K / 64;
  return ((row / 128) * tiles_k + g / 4) * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + (g % 4);
}

int64_t scale_bytes(int64_t rows, int64_t K) { return ((rows + 127) / 128) * 128 * (K / 16); }

uint8_t code_at(const uint8_t* codes, int64_t row, int64_t k, int64_t K) {
  uint8_t b = codes[row * (K / 2) + k / 2];
  return (k & 1) ? static_cast<uint8_t>(b >> 4) : static_cast<uint8_t>(b & 15);
}

// Quantise `rows` vectors of length K, element (i, k) at V[i*row_stride + k*k_stride],
// into packed codes and tiled scales; `gs` > 0 selects the two-level
// quantiser with that global scale, 0 the plain one.
void quantize_rows(const float* V, int64_t rows, int64_t K, int64_t row_stride, int64_t k_stride,
                   uint8_t* codes, uint8_t* scales, float gs = 0.0f) {
  std::memset(scales, 0, static_cast<size_t>(scale_bytes(rows, K)));
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; ++i) {
    uint8_t q[16];
    for (int64_t g = 0; g < K / 16; ++g) {
      uint8_t s;
      if (gs > 0.0f)
        quantize_group_gs(V + i * row_stride + g * 16 * k_stride, k_stride, gs, q, &s);
      else
        quantize_group(V + i * row_stride + g * 16 * k_stride, k_stride, q, &s);
      scales[scale_offset(i, g, K)] = s;
      for (int j = 0; j < 16; j += 2)
        codes[i * (K / 2) + g * 8 + j / 2] = static_cast<uint8_t>(q[j] | (q[j + 1] << 4));
    }
  }
}

// ------------------------------------------------ symmetric eigensolver ----
// Top eigenpairs of a symmetric n x n matrix (Golub & Van Loan, Matrix
// Computations, ch. 8): Householder tridiagonalisation, Sturm-sequence
// bisection for the wanted eigenvalues, inverse iteration on the tridiagonal
// matrix for their eigenvectors, then back-transformation.

struct Tridiag {
  int64_t n;
  std::vector<double> d, e;     // diagonal, sub-diagonal
  std::vector<double> hv;       // Householder vectors (row k holds v_k on k+1..n-1)
  std::vector<double> beta;
};

void tridiagonalize(std::vector<double>& A, int64_t n, Tridiag& t) {
  t.n = n;
  t.d.assign(n, 0.0);
  t.e.assign(n > 1 ? n - 1 : 0, 0.0);
  t.beta.assign(n, 0.0);
  std::vector<double> v(n), p(n), w(n);
  for (int64_t k = 0; k + 2 < n; ++k) {
    const int64_t m = n - k - 1;  // trailing size
    double* x = &A[k * n + k + 1];
    double nrm2 = 0.0;
    for (int64_t i = 0; i < m; ++i) nrm2 += x[i] * x[i];
    double nrm = std::sqrt(nrm2);
    t.d[k] = A[k * n + k];
    if (nrm == 0.0) {
      t.e[k] = 0.0;
      t.beta[k] = 0.0;
      for (int64_t i = 0; i < m; ++i) x[i] = 0.0;
      continue;
    }
    double alpha = x[0] > 0 ? -nrm : nrm;  // H x = alpha e_1
    for (int64_t i = 0; i < m; ++i) v[i] = x[i];
    v[0] -= alpha;
    double vtv = nrm2 - x[0] * x[0] + v[0] * v[0];
    double beta = 2.0 / vtv;
    // p = beta * B v over the trailing block B = A[k+1.., k+1..]
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < m; ++i) {
      const double* row = &A[(k + 1 + i) * n + k + 1];
      double s = 0.0;
      for (int64_t j = 0; j < m; ++j) s += row[j] * v[j];
      p[i] = beta * s;
    }
    double ptv = 0.0;
    for (int64_t i = 0; i < m; ++i) ptv += p[i] * v[i];
    const double kk = 0.5 * beta * ptv;
    for (int64_t i = 0; i < m; ++i) w[i] = p[i] - kk * v[i];
    // B <- B - v w^T - w v^T
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < m; ++i) {
      double* row = &A[(k + 1 + i) * n + k + 1];
      const double vi = v[i], wi = w[i];
      for (int64_t j = 0; j < m; ++j) row[j] -= vi * w[j] + wi * v[j];
    }
    t.e[k] = alpha;
    t.beta[k] = beta;
    for (int64_t i = 0; i < m; ++i) x[i] = v[i];  // store v_k in row k
  }
  if (n >= 2) {
    t.d[n - 2] = A[(n - 2) * n + n - 2];
    t.d[n - 1] = A[(n - 1) * n + n - 1];
    t.e[n - 2] = A[(n - 2) * n + n - 1];
  } else if (n == 1) {
    t.d[0] = A[0];
  }
  t.hv.swap(A);
}

// Number of eigenvalues of the tridiagonal matrix strictly below x.
int64_t sturm_count(const Tridiag& t, double x, double pivmin) {
  int64_t c = 0;
  double q = t.d[0] - x;
  if (std::fabs(q) < pivmin) q = -pivmin;
  if (q < 0) ++c;
  for (int64_t i = 1; i < t.n; ++i) {
    q = t.d[i] - x - t.e[i - 1] * t.e[i - 1] / q;
    if (std::fabs(q) < pivmin) q = -pivmin;
    if (q < 0) ++c;
  }
  return c;
}

// Inverse iteration for eigenvalue mu of the tridiagonal matrix, kept
// orthogonal to the vectors already found (rows of prev, length n each).
void inverse_iteration(const Tridiag& t, double mu, double tnorm, const std::vector<double>& prev,
                       int64_t nprev, uint64_t seed, double* y) {
  const int64_t n = t.n;
  const double tiny = 1e-300 + tnorm * 1e-15;
  std::vector<double> dl(n), d(n), du(n), du2(n), L(n);
  std::vector<char> piv(n, 0);
  for (int64_t i = 0; i < n; ++i) d[i] = t.d[i] - mu;
  for (int64_t i = 0; i + 1 < n; ++i) { dl[i] = t.e[i]; du[i] = t.e[i]; du2[i] = 0.0; }
  // LU with partial pivoting of T - mu I (two super-diagonals after swaps).
  for (int64_t i = 0; i + 1 < n; ++i) {
    if (std::fabs(d[i]) >= std::fabs(dl[i])) {
      if (d[i] == 0.0) d[i] = tiny;
      L[i] = dl[i] / d[i];
      d[i + 1] -= L[i] * du[i];
      du2[i] = 0.0;
      piv[i] = 0;
    } else {
      const double l = d[i] / dl[i];
      const double d1 = d[i + 1], u0 = du[i], u1 = (i + 2 < n) ? du[i + 1] : 0.0;
      L[i] = l;
      d[i] = dl[i];
      du[i] = d1;
      du2[i] = u1;
      d[i + 1] = u0 - l * d1;
      if (i + 2 < n) du[i + 1] = -l * u1;
      piv[i] = 1;
    }
  }
  if (d[n - 1] == 0.0) d[n - 1] = tiny;
  for (int64_t i = 0; i < n; ++i) {
    if (std::fabs(d[i]) < tiny) d[i] = d[i] < 0 ? -tiny : tiny;
  }
  // deterministic start vector (SplitMix64 uniforms in [-1, 1))
  uint64_t s = seed;
  for (int64_t i = 0; i < n; ++i) {
    uint64_t z = (s += 0x9E3779B97F4A7C15ULL);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    z ^= z >> 31;
    y[i] = 2.0 * static_cast<double>(z >> 11) / 9007199254740992.0 - 1.0;
  }
  std::vector<double> b(n);
  for (int it = 0; it < 5; ++it) {
    // orthogonalise, normalise
    for (int pass = 0; pass < 2; ++pass)
      for (int64_t j = 0; j < nprev; ++j) {
        const double* q = &prev[j * n];
        double dot = 0.0;
        for (int64_t i = 0; i < n; ++i) dot += q[i] * y[i];
        for (int64_t i = 0; i < n; ++i) y[i] -= dot * q[i];
      }
    double nrm = 0.0;
    for (int64_t i = 0; i < n; ++i) nrm += y[i] * y[i];
    nrm = std::sqrt(nrm);
    for (int64_t i = 0; i < n; ++i) y[i] /= nrm;
    if (it == 4) break;
    // solve (T - mu I) z = y
    for (int64_t i = 0; i < n; ++i) b[i] = y[i];
    for (int64_t i = 0; i + 1 < n; ++i) {
      if (piv[i]) std::swap(b[i], b[i + 1]);
      b[i + 1] -= L[i] * b[i];
    }
    y[n - 1] = b[n - 1] / d[n - 1];
    if (n >= 2) y[n - 2] = (b[n - 2] - du[n - 2] * y[n - 1]) / d[n - 2];
    for (int64_t i = n - 3; i >= 0; --i) y[i] = (b[i] - du[i] * y[i + 1] - du2[i] * y[i + 2]) / d[i];
    double mx = 0.0;
    for (int64_t i = 0; i < n; ++i) mx = std::max(mx, std::fabs(y[i]));
    if (mx > 0) for (int64_t i = 0; i < n; ++i) y[i] /= mx;  // keep in range
  }
}

// Top `k` eigenpairs of symmetric A (n x n, row-major, destroyed), largest
// first.  vals[k], vecs[n][k] (column j is the eigenvector of vals[j]).
void sym_eig_top(std::vector<double>& A, int64_t n, int64_t k, double* vals, double* vecs) {
  Tridiag t;
  tridiagonalize(A, n, t);
  double lo = 1e300, hi = -1e300, tnorm = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    double r = (i > 0 ? std::fabs(t.e[i - 1]) : 0.0) + (i + 1 < n ? std::fabs(t.e[i]) : 0.0);
    lo = std::min(lo, t.d[i] - r);
    hi = std::max(hi, t.d[i] + r);
    tnorm = std::max(tnorm, std::fabs(t.d[i]) + r);
  }
  const double pivmin = std::max(1e-300, tnorm * 1e-300);
  lo -= 1e-12 * tnorm + 1e-300;
  hi += 1e-12 * tnorm + 1e-300;
  std::vector<double> tv(static_cast<size_t>(k) * n, 0.0);  // eigenvectors of T (rows)
  for (int64_t j = 0; j < k; ++j) {
    const int64_t idx = n - 1 - j;  // ascending index of the j-th largest
    double a = lo, b = hi;
    for (int it = 0; it < 200 && b - a > 2.2e-16 * std::max(std::fabs(a), std::fabs(b)) + pivmin; ++it) {
      double mid = 0.5 * (a + b);
      if (mid == a || mid == b) break;
      if (sturm_count(t, mid, pivmin) <= idx) a = mid;  // lambda_idx >= mid
      else b = mid;
    }
    vals[j] = 0.5 * (a + b);
    inverse_iteration(t, vals[j], tnorm, tv, j, 0x5EEDULL + 7919ULL * j, &tv[j * n]);
  }
  // back-transform: x = H_0 H_1 ... H_{n-3} y
#pragma omp parallel for schedule(dynamic)
  for (int64_t j = 0; j < k; ++j) {
    double* y = &tv[j * n];
    for (int64_t kk = n - 3; kk >= 0; --kk) {
      const double beta = t.beta[kk];
      if (beta == 0.0) continue;
      const double* v = &t.hv[kk * n + kk + 1];
      double s = 0.0;
      for (int64_t i = 0; i < n - kk - 1; ++i) s += v[i] * y[kk + 1 + i];
      s *= beta;
      for (int64_t i = 0; i < n - kk - 1; ++i) y[kk + 1 + i] -= s * v[i];
    }
  }
  for (int64_t j = 0; j < k; ++j)
    for (int64_t i = 0; i < n; ++i) vecs[i * k + j] = tv[j * n + i];
}

}  // namespace

// =========================================================== C interface ===

extern "C" {

// -- scalar codecs (pins) --
float oracle_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }
uint16_t oracle_bf16_from_f64(double x) { return bf16_from_f64(x); }
double oracle_e4m3_decode(uint8_t c) { return e4m3_decode(c); }
uint8_t oracle_e4m3_encode(float x) { return e4m3_encode(x); }
double oracle_e2m1_decode(uint8_t c) { return e2m1_decode(c); }
uint8_t oracle_e2m1_encode(float x) { return e2m1_encode(x); }

// One NVFP4 group: 16 floats -> 16 codes (one per byte, 4 bits used) + scale.
void oracle_nvfp4_quantize_group(const float* v, uint8_t* codes16, uint8_t* scale) {
  quantize_group(v, 1, codes16, scale);
}

int64_t oracle_scale_offset(int64_t row, int64_t g, int64_t K) { return scale_offset(row, g, K); }
int64_t oracle_scale_bytes(int64_t rows, int64_t K) { return scale_bytes(rows, K); }

// Rows of fp32 values [rows][K] -> packed codes [rows][K/2] + tiled scales.
int oracle_quantize_rows(const float* V, int64_t rows, int64_t K, uint8_t* codes, uint8_t* scales) {
  if (K % 64 != 0 || rows < 0) return 1;
  quantize_rows(V, rows, K, K, 1, codes, scales);
  return 0;
}

float oracle_gelu(float x) { return gelu_as(x); }

// One group of 16 with the two-level quantiser (global scale g > 0).
int oracle_quantize_group_gs(const float* v, float g, uint8_t* codes, uint8_t* scale) {
  if (!(g > 0.0f)) return 1;
  quantize_group_gs(v, 1, g, codes, scale);
  return 0;
}

int oracle_quantize_rows_gs(const float* V, int64_t rows, int64_t K, float g, uint8_t* codes, uint8_t* scales) {
  if (K % 64 != 0 || rows < 0 || !(g > 0.0f)) return 1;
  quantize_rows(V, rows, K, K, 1, codes, scales, g);
  return 0;
}

// Residual packer (step "pack R"): R fp32 [K][N] row-major; group of 16 along
// K for every output column n -> r_codes [N][K/2], r_scales tiled (N rows).
int oracle_pack_residual(const float* R, int64_t K, int64_t N, uint8_t* r_codes, uint8_t* r_scales) {
  if (K % 64 != 0 || N <= 0) return 1;
  quantize_rows(R, N, K, 1, N, r_codes, r_scales);
  return 0;
}

// The same with a global scale g_w > 0 for R (two-level NVFP4).
int oracle_pack_residual_gs(const float* R, int64_t K, int64_t N, float gw, uint8_t* r_codes, uint8_t* r_scales) {
  if (K % 64 != 0 || N <= 0 || !(gw > 0.0f)) return 1;
  quantize_rows(R, N, K, 1, N, r_codes, r_scales, gw);
  return 0;
}

// Smoothing factors (alpha = 0.5): a_j = max_i |Xcal_ij|, b_j = max_n |W_jn|,
// lambda_j = RN_f32(sqrt(a_j) / sqrt(b_j)) (1 when a_j or b_j is 0),
// inv_lambda_j = RN_f32(1 / lambda_j).
int oracle_smooth(const uint16_t* Xcal, int64_t Mc, const uint16_t* W, int64_t K, int64_t N,
                  float* lambda, float* inv_lambda) {
  std::vector<double> a(K, 0.0), b(K, 0.0);
  for (int64_t i = 0; i < Mc; ++i)
    for (int64_t j = 0; j < K; ++j) a[j] = std::max(a[j], std::fabs((double)bf16_to_f32(Xcal[i * K + j])));
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < K; ++j) {
    double m = 0.0;
    for (int64_t n = 0; n < N; ++n) m = std::max(m, std::fabs((double)bf16_to_f32(W[j * N + n])));
    b[j] = m;
  }
  for (int64_t j = 0; j < K; ++j) {
    float l = (a[j] == 0.0 || b[j] == 0.0) ? 1.0f : static_cast<float>(std::sqrt(a[j]) / std::sqrt(b[j]));
    lambda[j] = l;
    inv_lambda[j] = 1.0f / l;
  }
  return 0;
}

// Top-k eigenpairs of a symmetric matrix (copied), largest first.
int oracle_sym_eig_top(const double* A, int64_t n, int64_t k, double* vals, double* vecs) {
  if (k < 0 || k > n) return 1;
  std::vector<double> B(A, A + n * n);
  sym_eig_top(B, n, k, vals, vecs);
  return 0;
}

// Rank-r truncated SVD of a K x N matrix A (fp64): A ~ U diag(s) V^T.
// sigma receives r+1 values (sigma_{r+1} for the Eckart-Young-Mirsky check).
int oracle_svd_top(const double* A, int64_t K, int64_t N, int64_t r, double* U, double* sigma,
                   double* V) {
  const bool left = K <= N;  // eigen-solve the smaller Gram matrix
  const int64_t n = left ? K : N;
  const int64_t kk = std::min<int64_t>(r + 1, n);
  std::vector<double> G(static_cast<size_t>(n) * n, 0.0);
  if (left) {
#pragma omp parallel for schedule(dynamic)
    for (int64_t i = 0; i < K; ++i)
      for (int64_t j = i; j < K; ++j) {
        const double* a = A + i * N;
        const double* b = A + j * N;
        double s0 = 0, s1 = 0, s2 = 0, s3 = 0;
        int64_t q = 0;
        for (; q + 4 <= N; q += 4) {
          s0 += a[q] * b[q]; s1 += a[q + 1] * b[q + 1]; s2 += a[q + 2] * b[q + 2]; s3 += a[q + 3] * b[q + 3];
        }
        for (; q < N; ++q) s0 += a[q] * b[q];
        G[i * n + j] = G[j * n + i] = (s0 + s1) + (s2 + s3);
      }
  } else {
    std::vector<double> At(static_cast<size_t>(N) * K);
    for (int64_t i = 0; i < K; ++i)
      for (int64_t j = 0; j < N; ++j) At[j * K + i] = A[i * N + j];
#pragma omp parallel for schedule(dynamic)
    for (int64_t i = 0; i < N; ++i)
      for (int64_t j = i; j < N; ++j) {
        const double* a = &At[i * K];
        const double* b = &At[j * K];
        double s0 = 0, s1 = 0, s2 = 0, s3 = 0;
        int64_t q = 0;
        for (; q + 4 <= K; q += 4) {
          s0 += a[q] * b[q]; s1 += a[q + 1] * b[q + 1]; s2 += a[q + 2] * b[q + 2]; s3 += a[q + 3] * b[q + 3];
        }
        for (; q < K; ++q) s0 += a[q] * b[q];
        G[i * n + j] = G[j * n + i] = (s0 + s1) + (s2 + s3);
      }
  }
  std::vector<double> vals(kk), vecs(static_cast<size_t>(n) * kk);
  sym_eig_top(G, n, kk, vals.data(), vecs.data());
  for (int64_t j = 0; j < r + 1; ++j) sigma[j] = j < kk ? std::sqrt(std::max(0.0, vals[j])) : 0.0;
  // the other side's singular vectors: A^T u / s  (or A v / s)
  for (int64_t j = 0; j < r; ++j) {
    const double s = sigma[j];
    if (j >= kk) {  // rank beyond min(K, N): zero factors
      for (int64_t i = 0; i < K; ++i) U[i * r + j] = 0.0;
      for (int64_t c = 0; c < N; ++c) V[c * r + j] = 0.0;
      continue;
    }
    if (left) {
      for (int64_t i = 0; i < K; ++i) U[i * r + j] = vecs[i * kk + j];
#pragma omp parallel for schedule(static)
      for (int64_t c = 0; c < N; ++c) {
        double acc = 0.0;
        for (int64_t i = 0; i < K; ++i) acc += A[i * N + c] * vecs[i * kk + j];
        V[c * r + j] = s > 0 ? acc / s : 0.0;
      }
    } else {
      for (int64_t c = 0; c < N; ++c) V[c * r + j] = vecs[c * kk + j];
#pragma omp parallel for schedule(static)
      for (int64_t i = 0; i < K; ++i) {
        double acc = 0.0;
        for (int64_t c = 0; c < N; ++c) acc += A[i * N + c] * vecs[c * kk + j];
        U[i * r + j] = s > 0 ? acc / s : 0.0;
      }
    }
  }
  return 0;
}

// Offline preparation of one layer (step "prep"):
//   Wh = diag(lambda) W (fp64), rank-r SVD Wh ~ U S V^T,
//   L1 = bf16(U S) [K][r], L2 = bf16(V^T) [r][N],
//   R  = RN_f32(Wh - L1 L2) [K][N] with the bf16-rounded factors, fp64 sum.
// sigma receives r+1 singular values of Wh.
int oracle_lowrank(const uint16_t* W, const float* lambda, int64_t K, int64_t N, int64_t r,
                   uint16_t* L1, uint16_t* L2, float* R, double* sigma) {
  std::vector<double> Wh(static_cast<size_t>(K) * N);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < K; ++j)
    for (int64_t n = 0; n < N; ++n) Wh[j * N + n] = (double)lambda[j] * (double)bf16_to_f32(W[j * N + n]);
  std::vector<double> L1d(static_cast<size_t>(K) * r), L2d(static_cast<size_t>(r) * N);
  if (r > 0) {
    std::vector<double> U(static_cast<size_t>(K) * r), V(static_cast<size_t>(N) * r);
    oracle_svd_top(Wh.data(), K, N, r, U.data(), sigma, V.data());
    for (int64_t k = 0; k < K; ++k)
      for (int64_t j = 0; j < r; ++j) {
        L1[k * r + j] = bf16_from_f64(U[k * r + j] * sigma[j]);
        L1d[k * r + j] = bf16_to_f32(L1[k * r + j]);
      }
    for (int64_t j = 0; j < r; ++j)
      for (int64_t n = 0; n < N; ++n) {
        L2[j * N + n] = bf16_from_f64(V[n * r + j]);
        L2d[j * N + n] = bf16_to_f32(L2[j * N + n]);
      }
  } else if (sigma) {
    sigma[0] = 0.0;
  }
#pragma omp parallel for schedule(static)
  for (int64_t k = 0; k < K; ++k)
    for (int64_t n = 0; n < N; ++n) {
      double s = Wh[k * N + n];
      for (int64_t j = 0; j < r; ++j) s -= L1d[k * r + j] * L2d[j * N + n];
      R[k * N + n] = static_cast<float>(s);
    }
  return 0;
}

// LoRA adapter joined to the low-rank branch without re-quantising the
// residual (chattools.cn "SVDQuant的主要功能", item LoRA集成; the abstract: an
// adapter needs no re-quantisation).  With Xh = X diag(lambda)^-1,
//   Xh [L1 | diag(lambda) A] [L2 ; B] = Xh L1 L2 + X A B,
// so L1' = [L1 | bf16(RN_f32(lambda_k a_kj))], L2' = [L2 ; B] and R stays.
//   L1 [K][r], A [K][ra], L2 [r][N], B [ra][N] bf16 bits -> L1o [K][r+ra],
//   L2o [r+ra][N].
int oracle_attach_lora(const uint16_t* L1, const uint16_t* L2, const float* lambda, const uint16_t* A,
                       const uint16_t* B, int64_t K, int64_t N, int64_t r, int64_t ra, uint16_t* L1o,
                       uint16_t* L2o) {
  if (K <= 0 || N <= 0 || r < 0 || ra <= 0) return 1;
  const int64_t ro = r + ra;
  for (int64_t k = 0; k < K; ++k) {
    for (int64_t j = 0; j < r; ++j) L1o[k * ro + j] = L1[k * r + j];
    for (int64_t j = 0; j < ra; ++j) {
      const float prod = lambda[k] * bf16_to_f32(A[k * ra + j]);  // one fp32 rounding
      L1o[k * ro + r + j] = bf16_from_f64(static_cast<double>(prod));
    }
  }
  for (int64_t j = 0; j < r; ++j)
    for (int64_t n = 0; n < N; ++n) L2o[j * N + n] = L2[j * N + n];
  for (int64_t j = 0; j < ra; ++j)
    for (int64_t n = 0; n < N; ++n) L2o[(r + j) * N + n] = B[j * N + n];
  return 0;
}

// Activation step (quantise + low-rank down-projection), rows of X:
//   Xh  = RN_f32(X * inv_lambda)             per element
//   (x_codes, x_scales) = NVFP4(Xh) by groups of 16 along K
//   T   = bf16(sum_k bf16(Xh)_k L1[k][:])    fp64 sum, one rounding
int oracle_quantize_act_ex(const uint16_t* X, const float* inv_lambda, const uint16_t* L1, int64_t M,
                           int64_t K, int64_t r, int act, float gx, uint8_t* x_codes, uint8_t* x_scales,
                           uint16_t* T);

int oracle_quantize_act(const uint16_t* X, const float* inv_lambda, const uint16_t* L1, int64_t M,
                        int64_t K, int64_t r, uint8_t* x_codes, uint8_t* x_scales, uint16_t* T) {
  return oracle_quantize_act_ex(X, inv_lambda, L1, M, K, r, 0, 0.0f, x_codes, x_scales, T);
}

// The activation step with a global scale g_x for Xh (g_x = 0: the plain
// quantiser); T is of Xh itself, unaffected by the global scale.
int oracle_quantize_act_gs(const uint16_t* X, const float* inv_lambda, const uint16_t* L1, int64_t M,
                           int64_t K, int64_t r, float gx, uint8_t* x_codes, uint8_t* x_scales, uint16_t* T) {
  return oracle_quantize_act_ex(X, inv_lambda, L1, M, K, r, 0, gx, x_codes, x_scales, T);
}

// The general form: act = 1 applies GELU (gelu_as, in fp32, no bf16 rounding
// between) to the input before smoothing, Xh = RN_f32(GELU(x) * inv_lambda);
// act = 0 is the layer's own activation step.
int oracle_quantize_act_ex(const uint16_t* X, const float* inv_lambda, const uint16_t* L1, int64_t M,
                           int64_t K, int64_t r, int act, float gx, uint8_t* x_codes, uint8_t* x_scales,
                           uint16_t* T) {
  if (K % 64 != 0 || M < 0 || gx < 0.0f || act < 0 || act > 1) return 1;
  std::vector<float> Xh(static_cast<size_t>(M) * K);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < M; ++i)
    for (int64_t k = 0; k < K; ++k) {
      const float x = bf16_to_f32(X[i * K + k]);
      Xh[i * K + k] = (act == 1 ? gelu_as(x) : x) * inv_lambda[k];
    }
  quantize_rows(Xh.data(), M, K, K, 1, x_codes, x_scales, gx);
  if (r > 0) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < M; ++i) {
      std::vector<double> acc(r, 0.0);
      for (int64_t k = 0; k < K; ++k) {
        const double xb = bf16_to_f32(bf16_from_f64(Xh[i * K + k]));
        for (int64_t j = 0; j < r; ++j) acc[j] += xb * (double)bf16_to_f32(L1[k * r + j]);
      }
      for (int64_t j = 0; j < r; ++j) T[i * r + j] = bf16_from_f64(acc[j]);
    }
  }
  return 0;
}

// Dequantised 4-bit residual as fp32 [N][K] (exact: at most 6 significant bits).
int oracle_dequant(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t K, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < rows; ++i)
    for (int64_t k = 0; k < K; ++k)
      out[i * K + k] = static_cast<float>(e2m1_decode(code_at(codes, i, k, K)) *
                                          e4m3_decode(scales[scale_offset(i, k / 16, K)]));
  return 0;
}

// Output rows of the linear layer, in fp64:
//   Y[m][n] = sum_k deq(x)[m][k] deq(R)[n][k] + sum_j T[m][j] L2[j][n] + bias[n]
// for the listed rows only (rows[i] in [0, M)).  bias may be NULL.
int oracle_linear_rows_gs(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* T,
                          const uint8_t* r_codes, const uint8_t* r_scales, const uint16_t* L2,
                          const uint16_t* bias, int64_t M, int64_t K, int64_t N, int64_t r, double gx,
                          double gw, const int64_t* rows, int64_t nrows, double* Y);

int oracle_linear_rows(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* T,
                       const uint8_t* r_codes, const uint8_t* r_scales, const uint16_t* L2,
                       const uint16_t* bias, int64_t M, int64_t K, int64_t N, int64_t r,
                       const int64_t* rows, int64_t nrows, double* Y) {
  return oracle_linear_rows_gs(x_codes, x_scales, T, r_codes, r_scales, L2, bias, M, K, N, r, 1.0, 1.0, rows,
                               nrows, Y);
}

// With global scales: deq(x) and deq(R) carry their tensors' global scales,
//   Y[m][n] = g_x g_w sum_k q_x s_x q_R s_R + sum_j T[m][j] L2[j][n] + bias[n].
int oracle_linear_rows_gs(const uint8_t* x_codes, const uint8_t* x_scales, const uint16_t* T,
                          const uint8_t* r_codes, const uint8_t* r_scales, const uint16_t* L2,
                          const uint16_t* bias, int64_t M, int64_t K, int64_t N, int64_t r, double gx,
                          double gw, const int64_t* rows, int64_t nrows, double* Y) {
  if (K % 64 != 0 || !(gx > 0.0) || !(gw > 0.0)) return 1;
  std::vector<float> Rd(static_cast<size_t>(N) * K);
  oracle_dequant(r_codes, r_scales, N, K, Rd.data());
  for (int64_t t = 0; t < nrows; ++t) {
    const int64_t m = rows[t];
    if (m < 0 || m >= M) return 1;
    std::vector<double> xd(K);
    for (int64_t k = 0; k < K; ++k)
      xd[k] = e2m1_decode(code_at(x_codes, m, k, K)) * e4m3_decode(x_scales[scale_offset(m, k / 16, K)]);
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
      const float* rd = &Rd[n * K];
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += xd[k] * (double)rd[k];
      double lr = 0.0;
      for (int64_t j = 0; j < r; ++j) lr += (double)bf16_to_f32(T[m * r + j]) * (double)bf16_to_f32(L2[j * N + n]);
      Y[t * N + n] = gx * gw * acc + lr + (bias ? (double)bf16_to_f32(bias[n]) : 0.0);
    }
  }
  return 0;
}

int oracle_num_threads() {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

}  // extern "C"
