/*
 * q4_oracle.c -- plain, slow, CPU reference for affine 4-bit, group-32,
 * weight-only quantization and for dequantize-then-matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library; neither includes nor links
 * the other.
 *
 * What it follows.  The model card "personaplex-edge-q4" (section "Release
 * details") names the format: affine Q4, group size 32, BF16 activations, with
 * the packed weights consumed directly by a quantized matmul (opening
 * paragraph).  The Swift/MLX blog "NVIDIA PersonaPlex 7B on Apple Silicon"
 * (section "Depformer: per-step weight switching") shows the interface:
 * weight stored [out, in], per-row scales and biases, multiplied transposed,
 * with a given group size and bit width.  No page states the arithmetic, so
 * this file spells out the plainest reading of "affine, 4-bit, group 32":
 *
 *   per row n and group g (32 consecutive inputs k):
 *     mn, mx   = min, max of the group (exact: inputs are bf16)
 *     s32      = fp32(mx - mn) / 15      (IEEE fp32, round to nearest even)
 *     s        = bf16(s32), b = bf16(mn) (round to nearest even; b is exact)
 *     q        = 0 if s == 0, else clamp(rne((w - b) / s), 0, 15), in fp64
 *     w_hat    = s*q + b
 *   packing: byte k/2 of row n holds q[n,k] in bits 0..3 for even k and
 *            q[n,k+1] in bits 4..7; scales and biases are [N, K/32] bf16.
 *
 * The stored-size figure of the model card ("Packed language model 4.87 GiB"
 * for 8,371,408,896 parameters) fixes 5 bits per weight, i.e. 4-bit codes
 * plus a bf16 scale and a bf16 bias per 32 weights.
 *
 * All bf16 values cross this interface as their uint16 bit patterns.
 * Build flags: -O2 -ffp-contract=off (no fused multiply-add: every fp32/fp64
 * operation is a separately rounded IEEE operation).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OQ4_GROUP 32

enum {
  OQ4_OK = 0,
  OQ4_ERR_SHAPE = 2,
  OQ4_ERR_NONFINITE = 7,
};

/* ---- bf16 <-> binary64 ------------------------------------------------ */

double oq4_bf16_to_f64(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/*
 * Nearest bf16 to v, ties to even.  bf16 has an 8-bit significand and the
 * exponent range of binary32, so its subnormals are spaced 2^-133 apart.
 * The value is scaled by a power of two so that the bf16 spacing becomes 1,
 * rounded to an integer (nearbyint: ties to even in the default rounding
 * mode), and scaled back.  Every step but the rounding is exact.
 */
uint16_t oq4_bf16_from_f64(double v) {
  if (isnan(v)) return 0x7FC0;
  if (isinf(v)) return v > 0 ? 0x7F80 : 0xFF80;
  if (v == 0.0) return signbit(v) ? 0x8000 : 0x0000;
  int e;
  (void)frexp(v, &e);            /* |v| in [2^(e-1), 2^e) */
  int spacing_exp = e - 8;       /* 8 significant bits in that binade */
  if (spacing_exp < -133) spacing_exp = -133;
  double r = ldexp(nearbyint(ldexp(v, -spacing_exp)), spacing_exp);
  if (fabs(r) >= 0x1p128) return v > 0 ? 0x7F80 : 0xFF80;
  float f = (float)r;            /* exact: r fits 8 significant bits */
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return (uint16_t)(u >> 16);
}

/* ---- format size --------------------------------------------------------- */

/* Bytes of the packed form of an [N, K] weight: codes + scales + biases. */
int64_t oq4_packed_nbytes(int64_t N, int64_t K) {
  int64_t groups = N * (K / OQ4_GROUP);
  return N * K / 2 + groups * 2 /* scale */ + groups * 2 /* bias */;
}

/* ---- quantize ------------------------------------------------------------ */

static int quantize_group(const uint16_t* w, uint8_t* codes16, uint16_t* s_out,
                          uint16_t* b_out) {
  float mn = INFINITY, mx = -INFINITY;
  for (int i = 0; i < OQ4_GROUP; ++i) {
    float v = (float)oq4_bf16_to_f64(w[i]);
    if (!isfinite(v)) return OQ4_ERR_NONFINITE;
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  float range = mx - mn;              /* binary32 subtraction */
  float s32 = range / 15.0f;          /* binary32 division    */
  uint16_t sh = oq4_bf16_from_f64((double)s32);
  uint16_t bh = oq4_bf16_from_f64((double)mn);
  double s = oq4_bf16_to_f64(sh);
  double b = oq4_bf16_to_f64(bh);
  if (!isfinite(s)) return OQ4_ERR_NONFINITE;
  memset(codes16, 0, 16);
  for (int i = 0; i < OQ4_GROUP; ++i) {
    int q = 0;
    if (s != 0.0) {
      double t = (oq4_bf16_to_f64(w[i]) - b) / s;
      double r = nearbyint(t);
      if (r < 0.0) r = 0.0;
      if (r > 15.0) r = 15.0;
      q = (int)r;
    }
    codes16[i / 2] |= (uint8_t)(q << (4 * (i & 1)));
  }
  *s_out = sh;
  *b_out = bh;
  return OQ4_OK;
}

/*
 * W: [N, K] bf16 bits.  codes: [N, K/2] bytes.  scales, biases: [N, K/32].
 * Returns OQ4_ERR_SHAPE for K not a positive multiple of 32, and
 * OQ4_ERR_NONFINITE if any weight, or any group's scale, is not finite.
 */
int oq4_quantize(const uint16_t* W, int64_t N, int64_t K, uint8_t* codes,
                 uint16_t* scales, uint16_t* biases) {
  if (N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
  const int64_t G = K / OQ4_GROUP;
  int status = OQ4_OK;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      int st = quantize_group(W + n * K + g * OQ4_GROUP, codes + n * (K / 2) + g * 16,
                              scales + n * G + g, biases + n * G + g);
      if (st != OQ4_OK) {
#pragma omp atomic write
        status = st;
      }
    }
  }
  return status;
}

/* ---- dequantize ---------------------------------------------------------- */

static int code_at(const uint8_t* row_codes, int64_t k) {
  uint8_t byte = row_codes[k / 2];
  return (k & 1) ? (byte >> 4) : (byte & 0x0F);
}

/* w_hat = s*q + b in binary64 (the product is exact: 8 x 4 significant bits). */
static double dequant_value(const uint8_t* codes, const uint16_t* scales,
                            const uint16_t* biases, int64_t K, int64_t n, int64_t k) {
  const int64_t G = K / OQ4_GROUP;
  double s = oq4_bf16_to_f64(scales[n * G + k / OQ4_GROUP]);
  double b = oq4_bf16_to_f64(biases[n * G + k / OQ4_GROUP]);
  int q = code_at(codes + n * (K / 2), k);
  return s * (double)q + b;
}

/* Reconstructed weight rounded to bf16 (nearest, ties to even). */
int oq4_dequantize(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases,
                   int64_t N, int64_t K, uint16_t* W_out) {
  if (N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      W_out[n * K + k] = oq4_bf16_from_f64(dequant_value(codes, scales, biases, K, n, k));
  return OQ4_OK;
}

/* Reconstructed weight as binary64, not rounded. */
int oq4_dequantize_f64(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases,
                       int64_t N, int64_t K, double* W_out) {
  if (N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      W_out[n * K + k] = dequant_value(codes, scales, biases, K, n, k);
  return OQ4_OK;
}

/* ---- matmul: y = x . W_hat^T --------------------------------------------- */

/*
 * x: [M, K] bf16 bits.  Packed W: N rows.  rows: the nrows output columns to
 * compute (indices into 0..N-1), or NULL for all N in order.
 * y:      [M, nrows]  sum_k x[m,k] * w_hat[n,k]      (binary64)
 * absdot: [M, nrows]  sum_k |x[m,k] * w_hat[n,k]|    (binary64; may be NULL)
 * w_hat is the exact s*q + b, not rounded to bf16.
 */
int oq4_matmul_ref(const uint16_t* x, int64_t M, int64_t K, const uint8_t* codes,
                   const uint16_t* scales, const uint16_t* biases, int64_t N,
                   const int64_t* rows, int64_t nrows, double* y, double* absdot) {
  if (M < 0 || N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
  if (!rows) nrows = N;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows && (rows[r] < 0 || rows[r] >= N)) return OQ4_ERR_SHAPE;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t n = rows ? rows[r] : r;
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0, aacc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = oq4_bf16_to_f64(x[m * K + k]) *
                   dequant_value(codes, scales, biases, K, n, k);
        acc += p;
        aacc += fabs(p);
      }
      y[m * nrows + r] = acc;
      if (absdot) absdot[m * nrows + r] = aacc;
    }
  }
  return OQ4_OK;
}

/*
 * The same product taken group by group in the factored form
 *   y[m,n] = sum_g ( s[n,g] * sum_{k in g} x[m,k] q[n,k]  +  b[n,g] * sum_{k in g} x[m,k] ),
 * which equals the direct sum by distributivity.  Used only to cross-check
 * the direct form; all rows, binary64.
 */
int oq4_matmul_ref_factored(const uint16_t* x, int64_t M, int64_t K, const uint8_t* codes,
                            const uint16_t* scales, const uint16_t* biases, int64_t N,
                            double* y) {
  if (M < 0 || N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
  const int64_t G = K / OQ4_GROUP;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0;
      for (int64_t g = 0; g < G; ++g) {
        double xq = 0.0, xs = 0.0;
        for (int64_t k = g * OQ4_GROUP; k < (g + 1) * OQ4_GROUP; ++k) {
          double xv = oq4_bf16_to_f64(x[m * K + k]);
          xq += xv * (double)code_at(codes + n * (K / 2), k);
          xs += xv;
        }
        acc += oq4_bf16_to_f64(scales[n * G + g]) * xq + oq4_bf16_to_f64(biases[n * G + g]) * xs;
      }
      y[m * N + n] = acc;
    }
  }
  return OQ4_OK;
}

/* ---- 8-bit variant ---------------------------------------------------------
 *
 * The same affine rule with 8-bit codes: the pages compare a "standard 8-bit
 * conversion" of the model (TWX4 comparison page, opening section) and ship
 * an INT8 bundle (ONNX README, "All four variants"), without stating its
 * arithmetic.  The plainest reading keeps everything of the 4-bit rule but the
 * number of levels:
 *   s32 = fp32(mx - mn) / 255, s = bf16(s32), b = bf16(mn),
 *   q = 0 if s == 0, else clamp(rne((w - b) / s), 0, 255)  (binary64),
 *   w_hat = s*q + b (exact in binary64: 8 x 8 significant bits, plus b);
 * codes are one byte per weight, [N, K]; scales and biases [N, K/32] bf16.
 */

static int quantize_group_q8(const uint16_t* w, uint8_t* codes32, uint16_t* s_out, uint16_t* b_out) {
  float mn = INFINITY, mx = -INFINITY;
  for (int i = 0; i < OQ4_GROUP; ++i) {
    float v = (float)oq4_bf16_to_f64(w[i]);
    if (!isfinite(v)) return OQ4_ERR_NONFINITE;
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  float range = mx - mn;              /* binary32 subtraction */
  float s32 = range / 255.0f;         /* binary32 division    */
  uint16_t sh = oq4_bf16_from_f64((double)s32);
  uint16_t bh = oq4_bf16_from_f64((double)mn);
  double s = oq4_bf16_to_f64(sh);
  double b = oq4_bf16_to_f64(bh);
  if (!isfinite(s)) return OQ4_ERR_NONFINITE;
  for (int i = 0; i < OQ4_GROUP; ++i) {
    int q = 0;
    if (s != 0.0) {
      double r = nearbyint((oq4_bf16_to_f64(w[i]) - b) / s);
      if (r < 0.0) r = 0.0;
      if (r > 255.0) r = 255.0;
      q = (int)r;
    }
    codes32[i] = (uint8_t)q;
  }
  *s_out = sh;
  *b_out = bh;
  return OQ4_OK;
}

/* W: [N, K] bf16 bits -> codes [N, K] bytes, scales and biases [N, K/32]. */
int oq8_quantize(const uint16_t* W, int64_t N, int64_t K, uint8_t* codes, uint16_t* scales,
                 uint16_t* biases) {
  if (N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
  const int64_t G = K / OQ4_GROUP;
  int status = OQ4_OK;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    for (int64_t g = 0; g < G; ++g) {
      int st = quantize_group_q8(W + n * K + g * OQ4_GROUP, codes + n * K + g * OQ4_GROUP,
                                 scales + n * G + g, biases + n * G + g);
      if (st != OQ4_OK) {
#pragma omp atomic write
        status = st;
      }
    }
  }
  return status;
}

static double dequant_value_q8(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases,
                               int64_t K, int64_t n, int64_t k) {
  const int64_t G = K / OQ4_GROUP;
  double s = oq4_bf16_to_f64(scales[n * G + k / OQ4_GROUP]);
  double b = oq4_bf16_to_f64(biases[n * G + k / OQ4_GROUP]);
  return s * (double)codes[n * K + k] + b;
}

int oq8_dequantize(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases, int64_t N,
                   int64_t K, uint16_t* W_out) {
  if (N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      W_out[n * K + k] = oq4_bf16_from_f64(dequant_value_q8(codes, scales, biases, K, n, k));
  return OQ4_OK;
}

int oq8_dequantize_f64(const uint8_t* codes, const uint16_t* scales, const uint16_t* biases, int64_t N,
                       int64_t K, double* W_out) {
  if (N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k)
      W_out[n * K + k] = dequant_value_q8(codes, scales, biases, K, n, k);
  return OQ4_OK;
}

/* y = x . W_hat^T over the exact 8-bit w_hat; arguments as oq4_matmul_ref. */
int oq8_matmul_ref(const uint16_t* x, int64_t M, int64_t K, const uint8_t* codes, const uint16_t* scales,
                   const uint16_t* biases, int64_t N, const int64_t* rows, int64_t nrows, double* y,
                   double* absdot) {
  if (M < 0 || N < 0 || K <= 0 || K % OQ4_GROUP) return OQ4_ERR_SHAPE;
  if (!rows) nrows = N;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows && (rows[r] < 0 || rows[r] >= N)) return OQ4_ERR_SHAPE;
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t n = rows ? rows[r] : r;
    for (int64_t m = 0; m < M; ++m) {
      double acc = 0.0, aacc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        double p = oq4_bf16_to_f64(x[m * K + k]) * dequant_value_q8(codes, scales, biases, K, n, k);
        acc += p;
        aacc += fabs(p);
      }
      y[m * nrows + r] = acc;
      if (absdot) absdot[m * nrows + r] = aacc;
    }
  }
  return OQ4_OK;
}

/* Threads used by the OpenMP loops above (timing only; results do not depend
 * on it: every output element is computed by one thread in a fixed order). */
void oq4_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

int oq4_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
