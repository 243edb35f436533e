// Plain CPU oracle for the NVFP4 (W4A4) and FP8-rowwise quantized linear layer.
//
// TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check and the
// benchmark's CPU-baseline leg may load this library. It shares no code with the
// CUDA path: no headers, tables, helpers or generated constants.
//
// What is computed, and where it is stated:
//   * "BFL (fp8r / nvfp4)" (Diffusers docs), scheme list:
//       - fp8r: an E4M3 `weight` with one fp32 `weight_scale` per row; activations
//         are quantized per row to E4M3 at run time.
//       - nvfp4 (ModelOpt layout): packed E2M1 `weight` (two values per byte), one
//         E4M3 block scale per 16 elements (`weight_scale`), one global fp32
//         `weight_scale_2`, and a calibrated fp32 activation scale `input_scale`.
//   * "BFL (fp8r / nvfp4)", section "Kernels", table: the nvfp4 forward quantizes
//     the activations at run time (nvfp4_quantize) and runs a block-scaled FP4
//     GEMM (mm_fp4); fp8r runs a GEMM with row-wise scales (_scaled_mm).
//   * "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers": the SVDQuant-style
//     layer (smoothing, 16-bit low-rank branch, 4-bit residual), the W4A16 family
//     (4-bit weights, bf16 activations) and the INT4 variant of the 4-bit layer;
//     their readings are stated at each function below.
//   The pages name the element formats but print no bit layout. This file takes the
//   public OCP definitions of the two formats: E4M3 "FN" (bias 7, no infinity,
//   S.1111.111 is NaN, largest finite 448) and E2M1 (bias 1, magnitudes
//   0, 0.5, 1, 1.5, 2, 3, 4, 6).
//
// Every fp32 step is a single IEEE round-to-nearest-even operation (the file is
// compiled with -ffp-contract=off on an SSE target). Contractions are in fp64.
//
// Pinned by tests/test_oracle_*.py (format grids, all 256 E4M3 codes against a
// library cast, round trips and ties, quantize invariants, exact integer brute
// force on tiny shapes, closed forms). No worked numeric example exists on the
// pages, so end-to-end values beyond those invariants are not pinned further.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>
#ifdef _OPENMP
#include <omp.h>
#endif

extern "C" {

// ---------------------------------------------------------------------------
// Threads
// ---------------------------------------------------------------------------
void oracle_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oracle_get_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

// ---------------------------------------------------------------------------
// Element formats (OCP definitions; the BFL page names them only).
// ---------------------------------------------------------------------------

// E4M3 "FN": sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.
// exponent 0 is subnormal (m * 2^-9); exponent 15 with mantissa 7 is NaN.
double oracle_e4m3_decode(uint8_t code) {
  int s = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = std::ldexp((double)m, -9);
  else mag = std::ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

// E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.
// exponent 0 is subnormal (m * 0.5).
double oracle_e2m1_decode(uint8_t nibble) {
  int s = (nibble >> 3) & 1;
  int e = (nibble >> 1) & 0x3;
  int m = nibble & 0x1;
  double mag = (e == 0) ? 0.5 * m : std::ldexp(1.0 + m / 2.0, e - 1);
  return s ? -mag : mag;
}

// Round a finite magnitude `a` (>= 0) to the nearest entry of the ascending table
// `vals` (indexed by magnitude code). Values at or beyond the last entry saturate
// to it. Exact ties go to the even code. The midpoint of two neighbours is exact
// in double and `a` is an fp32 value, so the comparison is exact.
static int nearest_code(double a, const double* vals, int n) {
  if (a >= vals[n - 1]) return n - 1;
  // first entry >= a; vals[hi-1] < a <= vals[hi], or hi == 0 when a == 0
  int hi = (int)(std::lower_bound(vals, vals + n, a) - vals);
  if (hi == 0) return 0;
  int lo = hi - 1;
  if (a <= vals[lo]) return lo;         // only when a == vals[0] == 0
  double mid = 0.5 * (vals[lo] + vals[hi]);
  if (a < mid) return lo;
  if (a > mid) return hi;
  return (lo % 2 == 0) ? lo : hi;
}

static const double* e4m3_magnitudes() {
  // codes 0x00..0x7E, ascending; 0x7F is NaN
  static double t[127];
  static bool init = false;
  if (!init) {
    for (int c = 0; c < 127; ++c) t[c] = oracle_e4m3_decode((uint8_t)c);
    init = true;
  }
  return t;
}

static const double* e2m1_magnitudes() {
  static double t[8];
  static bool init = false;
  if (!init) {
    for (int c = 0; c < 8; ++c) t[c] = oracle_e2m1_decode((uint8_t)c);
    init = true;
  }
  return t;
}

// fp32 -> E4M3 code: round to nearest, ties to even, saturating to +-448.
// The sign is kept, so values that round to zero keep their sign (-tiny -> 0x80).
// NaN -> 0x7F.
uint8_t oracle_e4m3_encode(float v) {
  if (std::isnan(v)) return 0x7F;
  uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  double a = std::fabs((double)v);
  int code = nearest_code(a, e4m3_magnitudes(), 127);
  return (uint8_t)(sign | code);
}

// fp32 -> E2M1 code (nibble): round to nearest, ties to even, saturating to +-6.
// The sign is kept (-tiny -> 0x8). NaN is not representable; it maps to 0x7
// (documented as outside the tested domain).
uint8_t oracle_e2m1_encode(float v) {
  if (std::isnan(v)) return 0x7;
  uint8_t sign = std::signbit(v) ? 0x8 : 0x0;
  double a = std::fabs((double)v);
  int code = nearest_code(a, e2m1_magnitudes(), 8);
  return (uint8_t)(sign | code);
}

void oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* out) {
  (void)e4m3_magnitudes();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(v[i]);
}

void oracle_e2m1_encode_array(const float* v, int64_t n, uint8_t* out) {
  (void)e2m1_magnitudes();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(v[i]);
}

// Encode every fp32 whose bit pattern lies in [first, first + count) (patterns are
// taken as uint32). Used by the exhaustive conversion test.
void oracle_e4m3_encode_bits_range(uint32_t first, int64_t count, uint8_t* out) {
  (void)e4m3_magnitudes();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) {
    uint32_t b = first + (uint32_t)i;
    float f;
    std::memcpy(&f, &b, 4);
    out[i] = oracle_e4m3_encode(f);
  }
}

void oracle_e2m1_encode_bits_range(uint32_t first, int64_t count, uint8_t* out) {
  (void)e2m1_magnitudes();
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) {
    uint32_t b = first + (uint32_t)i;
    float f;
    std::memcpy(&f, &b, 4);
    out[i] = oracle_e2m1_encode(f);
  }
}

// ---------------------------------------------------------------------------
// bf16 (IEEE bfloat16: fp32 with the low 16 bits dropped).
// ---------------------------------------------------------------------------
static inline float bf16_to_float(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// One rounding, nearest-even, from an fp64 value to bf16 (8 significant bits,
// exponent range of fp32, subnormal quantum 2^-133, overflow to infinity).
uint16_t oracle_bf16_from_double(double v) {
  if (std::isnan(v)) return 0x7FC0;
  uint16_t sign = std::signbit(v) ? 0x8000 : 0x0000;
  double a = std::fabs(v);
  if (std::isinf(a)) return sign | 0x7F80;
  double q;                                    // spacing of bf16 values near a
  if (a < std::ldexp(1.0, -126)) {
    q = std::ldexp(1.0, -133);
  } else {
    int e;
    std::frexp(a, &e);                         // a = f * 2^e, f in [0.5, 1)
    q = std::ldexp(1.0, (e - 1) - 7);
  }
  double r = std::nearbyint(a / q) * q;        // default rounding mode: nearest-even
  if (r >= std::ldexp(1.0, 128)) return sign | 0x7F80;
  float rf = (float)r;                         // exact: r has <= 8 significant bits
  uint32_t u;
  std::memcpy(&u, &rf, 4);
  return (uint16_t)(sign | (uint16_t)(u >> 16));
}

void oracle_bf16_from_double_array(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_from_double(v[i]);
}

// ---------------------------------------------------------------------------
// GELU of a bf16 tensor, back to bf16: the activation between the MLP's two
// linear layers, which the fused up-projection epilogue quantizes for the down
// projection. The pages name "fused GELU/MLP" kernels only (Nunchaku section);
// this file takes the exact (erf) GELU, GELU(v) = v * Phi(v), Phi the standard
// normal CDF, written with erfc so that it stays accurate for large negative v:
//   Phi(v) = erfc(-v / sqrt(2)) / 2,   h = bf16( v * Phi(v) ), in fp64.
// A GPU that evaluates GELU in fp32 can round to the other bf16 neighbour only
// when the exact value lies within its error of the midpoint of two bf16 values;
// `ambiguous[i]` = 1 marks those elements: the fp64 value within
// (tol_const + tol_sq * v^2) * |value| of such a midpoint. (The v^2 term: an fp32
// rounding of v / sqrt(2) moves erfc by its logarithmic derivative, about
// 2 |v / sqrt(2)|, times |v / sqrt(2)| relative ulps.)
// ---------------------------------------------------------------------------
double oracle_gelu(double v) { return 0.5 * v * std::erfc(-v / std::sqrt(2.0)); }

void oracle_gelu_bf16(const uint16_t* y, int64_t n, double tol_const, double tol_sq, uint16_t* h,
                      uint8_t* ambiguous) {
  for (int64_t i = 0; i < n; ++i) {
    const double v = static_cast<double>(bf16_to_float(y[i]));
    const double g = oracle_gelu(v);
    const double rel_tol = tol_const + tol_sq * v * v;
    const uint16_t b = oracle_bf16_from_double(g);
    h[i] = b;
    if (ambiguous) {
      // the bf16 neighbours of g: b and the next value away from b on g's side
      const double vb = static_cast<double>(bf16_to_float(b));
      uint16_t other = b;
      if (g > vb) other = (b & 0x8000) ? (b == 0x8000 ? 0x0001 : b - 1) : b + 1;
      else if (g < vb) other = (b & 0x8000) ? b + 1 : (b == 0x0000 ? 0x8001 : b - 1);
      const double vo = static_cast<double>(bf16_to_float(other));
      const double mid = 0.5 * (vb + vo);
      ambiguous[i] = (g != vb && std::fabs(g - mid) <= rel_tol * std::fabs(g)) ? 1 : 0;
    }
  }
}

// ---------------------------------------------------------------------------
// SVDQuant-style NVFP4 linear with a 16-bit low-rank branch ("Bringing Nunchaku
// 4-bit Diffusion Inference to Diffusers", sections "Background: SVDQuant and
// Nunchaku" and "Introducing Nunchaku Lite", svdq_w4a4): activation outliers are
// moved into the weights by a per-channel smoothing, the hardest part of the
// weight is a rank-r 16-bit branch, and the residual is quantized to 4 bits.
// The pages give no formulas; the plainest reading is taken:
//   xs[m,k] = bf16( RN32(x[m,k] * smooth[k]) )          smoothed activations
//   D[m,j]  = sum_k xs[m,k] * down[j,k]                  low-rank down, j < r
//   Y[m,n]  = bf16( input_scale * weight_scale_2 * sum_k NVFP4(xs) NVFP4(R)
//                   + sum_j D[m,j] * up[n,j] + bias[n] )
// down [r, K] and up [N, r] are bf16 (nn.Linear weight layouts, 16-bit as the
// pages say); NVFP4(xs) uses input_scale; R is the 4-bit residual weight. The
// contractions are exact (fp64). T_lr[m,n] = sum_j |D[m,j] * up[n,j]| bounds the
// low-rank term, for the tolerance of a 16-bit evaluation of that branch.
// ---------------------------------------------------------------------------
void oracle_smooth_bf16(const uint16_t* x, int64_t M, int64_t K, const float* smooth,
                        uint16_t* out) {
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) {
      const float p = bf16_to_float(x[m * K + k]) * smooth[k];  // one fp32 RN multiply
      out[m * K + k] = oracle_bf16_from_double(static_cast<double>(p));
    }
}

void oracle_lowrank_down(const uint16_t* xs, int64_t M, int64_t K, const uint16_t* down,
                         int64_t r, double* D) {
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k)
        acc += static_cast<double>(bf16_to_float(xs[m * K + k])) *
               static_cast<double>(bf16_to_float(down[j * K + k]));
      D[m * r + j] = acc;
    }
}

int oracle_nvfp4_linear(const uint8_t* xq, const uint8_t* xs, int64_t M, int64_t K,
                        const uint8_t* wq, const uint8_t* ws, int64_t N,
                        float input_scale, float weight_scale_2, const float* bias,
                        uint16_t* y, double* y64, double* T);  // below

int oracle_svdq_nvfp4_linear(const uint8_t* xq, const uint8_t* xsc, int64_t M, int64_t K,
                             const uint8_t* wq, const uint8_t* ws, int64_t N, float input_scale,
                             float weight_scale_2, const double* D, const uint16_t* up, int64_t r,
                             const float* bias, uint16_t* y, double* y64, double* T,
                             double* T_lr) {
  if (M < 0 || N < 0 || K <= 0 || K % 16 != 0 || r < 0) return -1;
  std::vector<double> main64((size_t)M * N), mainT((size_t)M * N);
  int rc = oracle_nvfp4_linear(xq, xsc, M, K, wq, ws, N, input_scale, weight_scale_2, nullptr,
                               nullptr, main64.data(), mainT.data());
  if (rc != 0) return rc;
#pragma omp parallel for schedule(static)
  for (int64_t m = 0; m < M; ++m)
    for (int64_t n = 0; n < N; ++n) {
      double lr = 0.0, lr_abs = 0.0;
      for (int64_t j = 0; j < r; ++j) {
        const double t = D[m * r + j] * static_cast<double>(bf16_to_float(up[n * r + j]));
        lr += t;
        lr_abs += std::fabs(t);
      }
      const double v = main64[m * N + n] + lr + (bias ? static_cast<double>(bias[n]) : 0.0);
      if (y) y[m * N + n] = oracle_bf16_from_double(v);
      if (y64) y64[m * N + n] = v;
      if (T) T[m * N + n] = mainT[m * N + n];
      if (T_lr) T_lr[m * N + n] = lr_abs;
    }
  return 0;
}

// ---------------------------------------------------------------------------
// Calibration rule of the workloads: global scale = amax / (6 * 448), i.e. the
// largest magnitude maps onto the largest E2M1 value times the largest E4M3
// scale. fp32 division, one rounding. The pages only say "calibrated".
// ---------------------------------------------------------------------------
float oracle_nvfp4_global_scale(const uint16_t* x, int64_t n) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    float a = std::fabs(bf16_to_float(x[i]));
    if (a > amax) amax = a;
  }
  return amax / 2688.0f;
}

// ---------------------------------------------------------------------------
// NVFP4 quantization of a bf16 matrix [R, K] (K % 16 == 0) with global scale g.
// Used with g = input_scale for activations and g = weight_scale_2 for weights.
//   per 16-element block along K:
//     amax = max |x|                      (exact)
//     s    = E4M3(amax * c), c = 1/(6g)   (c: two fp32 roundings, once per tensor)
//     d    = decode(s) * g                (fp32)
//     d == 0  -> all 16 codes 0
//     else    -> code_i = E2M1(x_i * (1/d))   (fp32 reciprocal, fp32 multiply)
//   packing: element 2j in bits 3..0 of byte j, element 2j+1 in bits 7..4.
// Outputs: q [R, K/2] bytes, s [R, K/16] E4M3 codes, both row-major.
// Returns 0, or -1 on a bad shape.
// ---------------------------------------------------------------------------
int oracle_nvfp4_quantize(const uint16_t* x, int64_t R, int64_t K, float g,
                          uint8_t* q, uint8_t* s) {
  if (R < 0 || K <= 0 || K % 16 != 0) return -1;
  (void)e4m3_magnitudes();
  (void)e2m1_magnitudes();
  const float c = 1.0f / (6.0f * g);
  const int64_t nb = K / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t b = 0; b < nb; ++b) {
      const uint16_t* xb = x + r * K + b * 16;
      float v[16];
      float amax = 0.0f;
      for (int i = 0; i < 16; ++i) {
        v[i] = bf16_to_float(xb[i]);
        float a = std::fabs(v[i]);
        if (a > amax) amax = a;
      }
      float sf = amax * c;
      uint8_t sc = oracle_e4m3_encode(sf);
      s[r * nb + b] = sc;
      float d = (float)oracle_e4m3_decode(sc) * g;
      uint8_t codes[16];
      if (d == 0.0f) {
        for (int i = 0; i < 16; ++i) codes[i] = 0;
      } else {
        float inv = 1.0f / d;
        for (int i = 0; i < 16; ++i) codes[i] = oracle_e2m1_encode(v[i] * inv);
      }
      uint8_t* qb = q + r * (K / 2) + b * 8;
      for (int j = 0; j < 8; ++j)
        qb[j] = (uint8_t)((codes[2 * j] & 0xF) | ((codes[2 * j + 1] & 0xF) << 4));
    }
  }
  return 0;
}

// Decode packed NVFP4 rows to fp64: out[r, k] = E2M1(q) * E4M3(s[r, k/16]).
// The global scale is not applied.
int oracle_nvfp4_dequantize(const uint8_t* q, const uint8_t* s, int64_t R, int64_t K,
                            double* out) {
  if (R < 0 || K <= 0 || K % 16 != 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      uint8_t byte = q[r * (K / 2) + k / 2];
      uint8_t nib = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      out[r * K + k] = oracle_e2m1_decode(nib) * oracle_e4m3_decode(s[r * (K / 16) + k / 16]);
    }
  }
  return 0;
}

// Plain fp64 contraction: Y[m, n] = alpha_m[m] * alpha_n[n] * sum_k A[m,k] B[n,k]
// + bias[n], summed in increasing k, with the tolerance scale
// T[m, n] = |alpha_m[m] * alpha_n[n]| * sum_k |A[m,k] B[n,k]|.
static void contract(const double* A, const double* B, int64_t M, int64_t K, int64_t N,
                     const double* alpha_m, const double* alpha_n, const float* bias,
                     uint16_t* y, double* y64, double* T) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t m = 0; m < M; ++m) {
    const double* a = A + m * K;
    for (int64_t n = 0; n < N; ++n) {
      const double* b = B + n * K;
      double acc = 0.0, absacc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = a[k] * b[k];
        acc += p;
        absacc += std::fabs(p);
      }
      double alpha = alpha_m[m] * alpha_n[n];
      double v = alpha * acc + (bias ? (double)bias[n] : 0.0);
      if (y64) y64[m * N + n] = v;
      if (T) T[m * N + n] = std::fabs(alpha) * absacc;
      if (y) y[m * N + n] = oracle_bf16_from_double(v);
    }
  }
}

// NVFP4 linear, both operands already quantized:
//   Y[m, n] = bf16( input_scale * weight_scale_2 * sum_k xhat[m,k] what[n,k] + bias[n] )
// with xhat = E2M1(xq) * E4M3(xs), what = E2M1(wq) * E4M3(ws), all in fp64.
// The two global scales multiply the whole sum (one per operand); the bias is added
// after scaling. Any of y, y64, T may be null. bias may be null.
int oracle_nvfp4_linear(const uint8_t* xq, const uint8_t* xs, int64_t M, int64_t K,
                        const uint8_t* wq, const uint8_t* ws, int64_t N,
                        float input_scale, float weight_scale_2, const float* bias,
                        uint16_t* y, double* y64, double* T) {
  if (M < 0 || N < 0 || K <= 0 || K % 16 != 0) return -1;
  std::vector<double> A((size_t)M * K), B((size_t)N * K);
  oracle_nvfp4_dequantize(xq, xs, M, K, A.data());
  oracle_nvfp4_dequantize(wq, ws, N, K, B.data());
  std::vector<double> am((size_t)M, (double)input_scale), an((size_t)N, (double)weight_scale_2);
  contract(A.data(), B.data(), M, K, N, am.data(), an.data(), bias, y, y64, T);
  return 0;
}

// The device-fallback semantics of the BFL page ("Kernels", last paragraph): the
// weight is dequantized and the activations are NOT quantized. Used only to check
// that activation quantization changes the result slightly.
int oracle_nvfp4_linear_unquantized_act(const uint16_t* x, int64_t M, int64_t K,
                                        const uint8_t* wq, const uint8_t* ws, int64_t N,
                                        float weight_scale_2, const float* bias,
                                        double* y64) {
  if (M < 0 || N < 0 || K <= 0 || K % 16 != 0) return -1;
  std::vector<double> A((size_t)M * K), B((size_t)N * K);
  for (int64_t i = 0; i < M * K; ++i) A[i] = (double)bf16_to_float(x[i]);
  oracle_nvfp4_dequantize(wq, ws, N, K, B.data());
  std::vector<double> am((size_t)M, 1.0), an((size_t)N, (double)weight_scale_2);
  contract(A.data(), B.data(), M, K, N, am.data(), an.data(), bias, nullptr, y64, nullptr);
  return 0;
}

// ---------------------------------------------------------------------------
// FP8 row-wise ("fp8r"): per row r of a bf16 matrix [R, K]
//   amax  = max_k |x|
//   scale = amax / 448        (fp32 division, one rounding)
//   scale == 0 -> codes 0x00
//   else       -> code = E4M3(x * (1/scale))   (fp32 reciprocal, fp32 multiply)
// Used for activations (rows = tokens) and weights (rows = output channels).
// ---------------------------------------------------------------------------
int oracle_fp8r_quantize_rows(const uint16_t* x, int64_t R, int64_t K,
                              uint8_t* q, float* scale) {
  if (R < 0 || K <= 0) return -1;
  (void)e4m3_magnitudes();
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; ++r) {
    const uint16_t* xr = x + r * K;
    float amax = 0.0f;
    for (int64_t k = 0; k < K; ++k) {
      float a = std::fabs(bf16_to_float(xr[k]));
      if (a > amax) amax = a;
    }
    float sc = amax / 448.0f;
    scale[r] = sc;
    if (sc == 0.0f) {
      for (int64_t k = 0; k < K; ++k) q[r * K + k] = 0;
    } else {
      float inv = 1.0f / sc;
      for (int64_t k = 0; k < K; ++k) q[r * K + k] = oracle_e4m3_encode(bf16_to_float(xr[k]) * inv);
    }
  }
  return 0;
}

// fp8r linear: Y[m, n] = bf16( xs[m] * ws[n] * sum_k E4M3(xq[m,k]) E4M3(wq[n,k]) + bias[n] )
// in fp64 (the row-wise scale_a[m] * scale_b[n] semantics of a scaled GEMM).
int oracle_fp8r_linear(const uint8_t* xq, const float* xs, int64_t M, int64_t K,
                       const uint8_t* wq, const float* ws, int64_t N, const float* bias,
                       uint16_t* y, double* y64, double* T) {
  if (M < 0 || N < 0 || K <= 0) return -1;
  std::vector<double> A((size_t)M * K), B((size_t)N * K);
  for (int64_t i = 0; i < M * K; ++i) A[i] = oracle_e4m3_decode(xq[i]);
  for (int64_t i = 0; i < N * K; ++i) B[i] = oracle_e4m3_decode(wq[i]);
  std::vector<double> am((size_t)M), an((size_t)N);
  for (int64_t m = 0; m < M; ++m) am[m] = (double)xs[m];
  for (int64_t n = 0; n < N; ++n) an[n] = (double)ws[n];
  contract(A.data(), B.data(), M, K, N, am.data(), an.data(), bias, y, y64, T);
  return 0;
}

// ---------------------------------------------------------------------------
// W4A16: NVFP4 weights with 16-bit activations. The 4-bit weight kernel family
// of "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers" (section
// "Introducing Nunchaku Lite", the W4A16 family: memory-bound modulation layers),
// taken with the weight format of "BFL (fp8r / nvfp4)" and the semantics that page
// gives for devices without the fused kernel ("Kernels", last paragraph): the
// weight is dequantized to the compute dtype (bf16) and the layer runs as a plain
// linear on unquantized activations.
//   what[n, k] = bf16( fp32( E2M1(q[n,k]) * E4M3(s[n, k/16]) * weight_scale_2 ) )
// The triple product is exact in fp64 (at most 2 + 4 + 24 significant bits); it is
// rounded once to fp32 (the dequantization arithmetic) and then to bf16 (the cast
// to the compute dtype).
// ---------------------------------------------------------------------------
int oracle_w4a16_dequantize_bf16(const uint8_t* q, const uint8_t* s, int64_t R, int64_t K,
                                 float weight_scale_2, uint16_t* out) {
  if (R < 0 || K <= 0 || K % 16 != 0) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t k = 0; k < K; ++k) {
      const uint8_t byte = q[r * (K / 2) + k / 2];
      const uint8_t nib = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      const double exact = oracle_e2m1_decode(nib) * oracle_e4m3_decode(s[r * (K / 16) + k / 16]) *
                           (double)weight_scale_2;
      const float w32 = (float)exact;  // one RN to fp32
      out[r * K + k] = oracle_bf16_from_double((double)w32);
    }
  }
  return 0;
}

// W4A16 linear: Y[m, n] = bf16( sum_k x[m,k] * what[n,k] + bias[n] ), the sum in
// fp64 in increasing k (the products of two bf16 values are exact), with the
// tolerance scale T[m, n] = sum_k |x[m,k] * what[n,k]|.
int oracle_w4a16_linear(const uint16_t* x, int64_t M, int64_t K, const uint8_t* wq,
                        const uint8_t* ws, int64_t N, float weight_scale_2, const float* bias,
                        uint16_t* y, double* y64, double* T) {
  if (M < 0 || N < 0 || K <= 0 || K % 16 != 0) return -1;
  std::vector<uint16_t> wb((size_t)N * K);
  oracle_w4a16_dequantize_bf16(wq, ws, N, K, weight_scale_2, wb.data());
  std::vector<double> A((size_t)M * K), B((size_t)N * K);
  for (int64_t i = 0; i < M * K; ++i) A[i] = (double)bf16_to_float(x[i]);
  for (int64_t i = 0; i < N * K; ++i) B[i] = (double)bf16_to_float(wb[i]);
  std::vector<double> am((size_t)M, 1.0), an((size_t)N, 1.0);
  contract(A.data(), B.data(), M, K, N, am.data(), an.data(), bias, y, y64, T);
  return 0;
}

// ---------------------------------------------------------------------------
// INT4 W4A4: the INT4 variant of the svdq_w4a4 kernel family ("Bringing Nunchaku
// 4-bit Diffusion Inference to Diffusers", section "Introducing Nunchaku Lite":
// 4-bit weights and activations, "available in INT4 and NVFP4 variants"), without
// the low-rank branch. The page gives no format; the reading: signed 4-bit integer
// codes in [-8, 7] with one fp32 scale per 64-element group along K, for the
// activations (quantized at run time) and the weights:
//   amax  = max over the group of |x|
//   scale = RN32(amax / 7)                    (the largest magnitude maps to 7)
//   scale == 0 -> all codes 0
//   else       -> q = clamp(RNE(RN32(x * RN32(1 / scale))), -8, 7)
// Codes are packed two per byte, element 2j in bits 3..0 of byte j (two's
// complement nibbles); scales are row-major [R, K/64].
// ---------------------------------------------------------------------------
int oracle_int4_quantize(const uint16_t* x, int64_t R, int64_t K, uint8_t* q, float* scale) {
  if (R < 0 || K <= 0 || K % 64 != 0) return -1;
  const int64_t G = K / 64;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < R; ++r) {
    for (int64_t g = 0; g < G; ++g) {
      const uint16_t* xg = x + r * K + g * 64;
      float amax = 0.0f;
      for (int i = 0; i < 64; ++i) {
        const float a = std::fabs(bf16_to_float(xg[i]));
        if (a > amax) amax = a;
      }
      const float sc = amax / 7.0f;  // one fp32 division
      scale[r * G + g] = sc;
      const float inv = sc == 0.0f ? 0.0f : 1.0f / sc;
      uint8_t* qg = q + r * (K / 2) + g * 32;
      for (int i = 0; i < 64; i += 2) {
        int c[2] = {0, 0};
        for (int e = 0; e < 2; ++e) {
          if (sc == 0.0f) continue;
          const float t = bf16_to_float(xg[i + e]) * inv;  // one fp32 multiply
          double rq = std::nearbyint(static_cast<double>(t));  // ties to even
          if (rq < -8.0) rq = -8.0;
          if (rq > 7.0) rq = 7.0;
          c[e] = static_cast<int>(rq);
        }
        qg[i / 2] = static_cast<uint8_t>((c[0] & 0xF) | ((c[1] & 0xF) << 4));
      }
    }
  }
  return 0;
}

static inline int int4_code(const uint8_t* q, int64_t k) {
  const int nib = (k % 2 == 0) ? (q[k / 2] & 0xF) : (q[k / 2] >> 4);
  return nib >= 8 ? nib - 16 : nib;
}

// INT4 linear:
//   Y[m, n] = bf16( sum_g xs[m,g] ws[n,g] sum_{k in group g} qx[m,k] qw[n,k] + bias[n] )
// the integer group sums exact, the scaled sum in fp64 in increasing g, with the
// tolerance scale T[m, n] = sum_g |xs[m,g] ws[n,g]| sum_{k in g} |qx qw|.
int oracle_int4_linear(const uint8_t* xq, const float* xs, int64_t M, int64_t K,
                       const uint8_t* wq, const float* ws, int64_t N, const float* bias,
                       uint16_t* y, double* y64, double* T) {
  if (M < 0 || N < 0 || K <= 0 || K % 64 != 0) return -1;
  const int64_t G = K / 64;
  std::vector<int8_t> A((size_t)M * K), B((size_t)N * K);
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k) A[m * K + k] = static_cast<int8_t>(int4_code(xq + m * (K / 2), k));
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) B[n * K + k] = static_cast<int8_t>(int4_code(wq + n * (K / 2), k));
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0, absacc = 0.0;
      for (int64_t g = 0; g < G; ++g) {
        int64_t isum = 0, iabs = 0;
        for (int64_t k = g * 64; k < g * 64 + 64; ++k) {
          const int64_t p = static_cast<int64_t>(A[m * K + k]) * B[n * K + k];
          isum += p;
          iabs += p < 0 ? -p : p;
        }
        const double sc = static_cast<double>(xs[m * G + g]) * static_cast<double>(ws[n * G + g]);
        acc += sc * static_cast<double>(isum);
        absacc += std::fabs(sc) * static_cast<double>(iabs);
      }
      const double v = acc + (bias ? static_cast<double>(bias[n]) : 0.0);
      if (y64) y64[m * N + n] = v;
      if (T) T[m * N + n] = absacc;
      if (y) y[m * N + n] = oracle_bf16_from_double(v);
    }
  }
  return 0;
}

}  // extern "C"
