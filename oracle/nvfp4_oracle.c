/*
 * CPU oracle for mm_bf16_fp4: out[m,n] = A[m,k](bf16) . dequant(W[n,k])^T with W in NVFP4.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, plain reference that the CUDA library
 * is checked against. Only the test suite, the smoke check and the benchmark's CPU-baseline
 * leg may load it. It shares no code, header, table or helper with the CUDA library.
 *
 * Sources:
 *  - "perf(gemm): split-K, occupancy, and m=1 stream-GEMV decode tactics for mm_bf16_fp4"
 *    (flashinfer PR #4038), Description: the op multiplies bf16 activations by nvfp4
 *    weights; the GEMV commit message: weights come in the canonical (N, K/2) packed layout
 *    with linear (row-major, unswizzled) E4M3 scales, one per 16 k.
 *  - The NVFP4 quantisation recipe this library targets: per 16-k block scale = block
 *    amax / 6 rounded to E4M3, global scale = tensor amax / (448 * 6), E2M1 codes packed two
 *    per byte. The pages name the format but not the recipe.
 *  - Element formats: OCP Microscaling Formats (MX) v1.0, FP4 E2M1 (bias 1, max 6, no
 *    inf/NaN); OCP 8-bit Floating Point (OFP8), E4M3 (bias 7, max 448, S.1111.111 = NaN).
 *
 * Readings where the sources are silent (each is a choice, listed with the design notes):
 *  - block scale is taken relative to the global scale: sf = (amax_b / 6) / gscale;
 *  - every rounding is round-to-nearest, ties to even; E4M3 and E2M1 saturate to max;
 *  - divisions are single fp32 IEEE divisions in the order written;
 *  - a code carries the sign of its input (a negative value that rounds to 0 gives 0x8);
 *  - a block whose fp32 denominator sf_val * gscale is 0 gets all-zero codes;
 *  - nibble order: byte j of a row holds code 2j in bits 0-3 and code 2j+1 in bits 4-7.
 *
 * Precision: the quantiser works in fp32 (the precision the recipe is stated in), the
 * dequantisation and the matmul in fp64, where every dequantised weight and every product
 * with a bf16 activation is exact.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---------------------------------------------------------------- element formats */

/* E2M1 decode from the bit fields: s | e1 e0 | m, bias 1. e == 0 is subnormal
 * (0 or 0.5); otherwise 2^(e-1) * (1 + m/2). OCP MX v1.0, FP4 E2M1. */
double orc_e2m1_decode(uint32_t code) {
  const int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  const double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

/* E4M3 decode from the bit fields: s | eeee | mmm, bias 7. e == 0 is subnormal
 * (m/8 * 2^-6); e == 15 && m == 7 is NaN; otherwise 2^(e-7) * (1 + m/8). OCP OFP8. */
double orc_e4m3_decode(uint32_t code) {
  const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) mag = ldexp(m / 8.0, -6);
  else mag = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* Round a finite magnitude ax >= 0 to the value grid of a binary minifloat with `mbits`
 * fraction bits and minimum normal exponent `emin`, round-to-nearest ties-to-even, then
 * clamp to `maxval` (saturating conversion). Works in double: for an fp32 input the
 * scaling by the power-of-two quantum is exact, so nearbyint() (current mode: nearest,
 * ties to even) performs the only rounding. */
static double round_minifloat(double ax, int mbits, int emin, double maxval) {
  if (ax == 0.0) return 0.0;
  int e;
  frexp(ax, &e);
  e -= 1; /* ax in [2^e, 2^(e+1)) */
  if (e < emin) e = emin; /* subnormals share the quantum of the lowest binade */
  const double quantum = ldexp(1.0, e - mbits);
  const double q = nearbyint(ax / quantum) * quantum;
  return q > maxval ? maxval : q;
}

/* Code bits of a magnitude v that lies on the grid (output of round_minifloat). */
static uint32_t minifloat_bits(double v, int mbits, int ebias) {
  const int emin = 1 - ebias;
  if (v == 0.0) return 0;
  int e;
  frexp(v, &e);
  e -= 1;
  if (e < emin) /* subnormal: exponent field 0, fraction = v / 2^(emin - mbits) */
    return (uint32_t)(v / ldexp(1.0, emin - mbits));
  const uint32_t frac = (uint32_t)((v / ldexp(1.0, e) - 1.0) * (double)(1 << mbits));
  return ((uint32_t)(e + ebias) << mbits) | frac;
}

/* fp32 -> E4M3 code, round to nearest even, saturate to +-448 (finite inputs). */
uint32_t orc_e4m3_encode(float x) {
  if (isnan(x)) return 0x7F;
  const double r = round_minifloat(fabs((double)x), 3, -6, 448.0);
  return (signbit(x) ? 0x80u : 0u) | minifloat_bits(r, 3, 7);
}

/* fp32 -> E2M1 code, round to nearest even, saturate to +-6; the sign bit follows x. */
uint32_t orc_e2m1_encode(float x) {
  const double r = round_minifloat(fabs((double)x), 1, 0, 6.0);
  return (signbit(x) ? 0x8u : 0u) | minifloat_bits(r, 1, 1);
}

/* bf16 bits -> double (exact: bf16 is the top half of an fp32). */
static double bf16_to_double(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

/* fp32 -> bf16 bits, round to nearest even (NaN kept quiet). */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40);
  const uint32_t lsb = (u >> 16) & 1u;
  return (uint16_t)((u + 0x7fffu + lsb) >> 16);
}

/* fp32 -> IEEE binary16 bits, round to nearest, ties to even (the optional f16 output of
 * PR #4038's commit covering fp16 output through the GEMV path). Written from the format
 * definition: the quantum of x's binade is 2^(e-10) for normal results (e >= -14) and 2^-24
 * below; x / quantum is exact in double, nearbyint rounds it half-to-even (the oracle is built
 * with the default rounding mode), and a result of 65536 or more is an overflow to +-inf. */
uint16_t orc_f32_to_f16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)(sign | 0x7e00u); /* NaN */
  const double x = fabs((double)f);
  if (x == 0.0) return sign;
  if (isinf(x)) return (uint16_t)(sign | 0x7c00u);
  int e2 = 0;
  frexp(x, &e2);           /* x = mant * 2^e2, mant in [0.5, 1): floor(log2 x) = e2 - 1 */
  int e = e2 - 1;
  const double q = e < -14 ? ldexp(1.0, -24) : ldexp(1.0, e - 10);
  const double nq = nearbyint(x / q);
  const double v = nq * q;
  if (v >= 65536.0) return (uint16_t)(sign | 0x7c00u);
  if (v < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)(v / ldexp(1.0, -24))); /* subnormal */
  frexp(v, &e2);
  e = e2 - 1;              /* the rounded value may have moved up one binade */
  const uint32_t mant = (uint32_t)(v / ldexp(1.0, e - 10)) - 1024u;
  return (uint16_t)(sign | (uint32_t)(e + 15) << 10 | mant);
}

/* --------------------------------------------------------------------- quantise */

/* Global scale: one fp32 division of the tensor amax by 448 * 6 = 2688 (exact in fp32). */
float orc_global_scale(const float* W, int64_t count) {
  float amax = 0.0f;
  for (int64_t i = 0; i < count; ++i) {
    const float a = fabsf(W[i]);
    if (a > amax) amax = a;
  }
  return amax / 2688.0f;
}

/* Quantise and pack one 16-element block given the fp32 global scale.
 * Writes 8 code bytes to q and returns the E4M3 scale code. */
static uint32_t quantise_block(const float* x, float gscale, uint8_t* q) {
  float bmax = 0.0f;
  for (int i = 0; i < 16; ++i) {
    const float a = fabsf(x[i]);
    if (a > bmax) bmax = a;
  }
  uint32_t sf_code = 0;
  if (gscale != 0.0f) {
    const float t = bmax / 6.0f;   /* block amax mapped onto E2M1's max */
    const float sf = t / gscale;   /* relative to the global scale */
    sf_code = orc_e4m3_encode(sf);
  }
  const float sf_val = (float)orc_e4m3_decode(sf_code); /* exact in fp32 */
  const float denom = sf_val * gscale;
  for (int i = 0; i < 16; i += 2) {
    uint32_t c0 = 0, c1 = 0;
    if (denom != 0.0f) {
      c0 = orc_e2m1_encode(x[i] / denom);
      c1 = orc_e2m1_encode(x[i + 1] / denom);
    }
    q[i / 2] = (uint8_t)(c0 | (c1 << 4));
  }
  return sf_code;
}

/* W fp32 [n, k] row-major -> Wq u8 [n, k/2], Wscale u8 [n, k/16], *gscale.
 * Returns 0, or -1 if k is not a multiple of 16. */
int orc_nvfp4_pack(const float* W, int64_t n, int64_t k, uint8_t* Wq, uint8_t* Wscale,
                   float* gscale) {
  if (k % 16 != 0 || n < 0 || k < 0) return -1;
  const float g = orc_global_scale(W, n * k);
  *gscale = g;
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j)
    for (int64_t b = 0; b < k / 16; ++b)
      Wscale[j * (k / 16) + b] =
          (uint8_t)quantise_block(W + j * k + b * 16, g, Wq + j * (k / 2) + b * 8);
  return 0;
}

/* ------------------------------------------------------------ dequant, matmul */

/* One row of dequant(W) in fp64: Wd[i] = e2m1(code_i) * e4m3(sf_(i/16)) * gscale. */
void orc_dequant_row(const uint8_t* Wq_row, const uint8_t* Ws_row, float gscale, int64_t k,
                     double* out) {
  for (int64_t i = 0; i < k; ++i) {
    const uint32_t byte = Wq_row[i / 2];
    const uint32_t code = (i % 2 == 0) ? (byte & 15u) : (byte >> 4);
    out[i] = orc_e2m1_decode(code) * orc_e4m3_decode(Ws_row[i / 16]) * (double)gscale;
  }
}

/* ref[r, c] = sum_i A[r, i] * dequant(W)[cols[c], i] in fp64, natural i order, for the
 * `ncols` weight rows listed in cols (all rows when cols == NULL, ncols == n).
 * A is bf16 bits [m, k]; ref is [m, ncols]. */
int orc_mm(const uint16_t* A, const uint8_t* Wq, const uint8_t* Wscale, float gscale,
           int64_t m, int64_t n, int64_t k, const int64_t* cols, int64_t ncols, double* ref) {
  if (k % 16 != 0) return -1;
  double* Ad = (double*)malloc(sizeof(double) * (size_t)(m * k > 0 ? m * k : 1));
  if (!Ad) return -2;
  for (int64_t i = 0; i < m * k; ++i) Ad[i] = bf16_to_double(A[i]);
  int bad = 0;
#pragma omp parallel reduction(| : bad)
  {
    double* wd = (double*)malloc(sizeof(double) * (size_t)(k > 0 ? k : 1));
    if (!wd) bad = 1;
#pragma omp for schedule(dynamic, 16)
    for (int64_t c = 0; c < ncols; ++c) {
      if (!wd) continue;
      const int64_t j = cols ? cols[c] : c;
      if (j < 0 || j >= n) { bad = 1; continue; }
      orc_dequant_row(Wq + j * (k / 2), Wscale + j * (k / 16), gscale, k, wd);
      for (int64_t r = 0; r < m; ++r) {
        double acc = 0.0;
        for (int64_t i = 0; i < k; ++i) acc += Ad[r * k + i] * wd[i];
        ref[r * ncols + c] = acc;
      }
    }
    free(wd);
  }
  free(Ad);
  return bad ? -3 : 0;
}

/* ------------------------------------------------------------ split-K reduce */

/* The fixed-order split-K reduction as a plain definition: for each output element,
 * s = ((p_0 + p_1) + p_2) + ... in fp32, then out = bf16_rn(s * gscale) (f16 == 0) or
 * f16_rn(s * gscale) (f16 != 0) with the product in fp32. partials is [S, m*n] fp32, out is
 * the output's bits [m*n]. */
void orc_splitk_reduce(const float* partials, int64_t S, int64_t mn, float gscale, int f16,
                       uint16_t* out) {
  for (int64_t e = 0; e < mn; ++e) {
    float s = partials[e];
    for (int64_t p = 1; p < S; ++p) s = s + partials[p * mn + e];
    const float v = s * gscale;
    out[e] = f16 ? orc_f32_to_f16(v) : orc_f32_to_bf16(v);
  }
}

int orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void orc_set_num_threads(int t) {
#ifdef _OPENMP
  if (t > 0) omp_set_num_threads(t);
#else
  (void)t;
#endif
}
