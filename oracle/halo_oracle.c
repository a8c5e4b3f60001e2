/*
 * halo_oracle.c -- plain, slow CPU oracle for the Hadamard-rotated quantized
 * linear layer of "HALO: Hadamard-Assisted Lower-Precision Optimization for
 * LLMs" (arXiv 2501.02625).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  The CUDA product path
 * never links, loads or calls it, and it shares no source with that path.
 *
 * Every function restates one step of the method in fp64 with no blocking,
 * fusion or reordering beyond what the step's definition states:
 *
 *   - Walsh-Hadamard transform: Sylvester matrix H_n = H_1 (x) H_{n-1} with
 *     H_1 = [[1,1],[1,-1]]/sqrt(2), applied with the in-place butterflies
 *     (x[j], x[j+h]) <- (x[j]+x[j+h], x[j]-x[j+h]) for h = 1, 2, 4, ... and a
 *     final division by sqrt(n)  [QWHA page, sec. 2.1 "mathematical basis" and
 *     sec. 2.2 walsh_hadamard_transform].  Applied block-locally (blocks of b
 *     consecutive elements along the contraction dimension), the block-wise
 *     reading of the HALO blog page, sec. 5, and of the QWHA page, sec. 5.
 *   - Symmetric absmax quantiser: scale = max|x| / qmax, qmax = 2^(bits-1)-1,
 *     q = clip(round(x / scale), -qmax, qmax), round = half-to-even
 *     [QWHA page, sec. 2.2 quantize]; FP8 E4M3 as the alternative 8-bit type
 *     [HALO paper page, "key design": INT8 or FP8].
 *   - Low-precision GEMM with a wide accumulator, then a dequantising product
 *     with the row and column scales [HALO paper page, abstract: all large
 *     matmuls of forward and backward run in lower precision].
 *
 * Parity pins: every function here is checked by tests/test_oracle_pins.py
 * against something other than itself (dense Sylvester matrices, orthogonality,
 * involution, rotation invariance, quantiser bounds, torch's float8_e4m3fn
 * conversion, numpy int64 matmul, hand-worked golden fixtures).
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* bf16 widening: a bf16 value is the top 16 bits of an IEEE binary32.      */
/* ------------------------------------------------------------------------ */
double halo_oracle_bf16_to_f64(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

void halo_oracle_bf16_array_to_f64(const uint16_t* in, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = halo_oracle_bf16_to_f64(in[i]);
}

/* ------------------------------------------------------------------------ */
/* Walsh-Hadamard transform of one vector of length n (n a power of two),    */
/* natural (Sylvester) order, normalised so that the transform is orthogonal.*/
/* QWHA page, sec. 2.1 (definition) and sec. 2.2 (iterative butterflies).    */
/* ------------------------------------------------------------------------ */
void halo_oracle_fwht(double* x, int64_t n) {
  for (int64_t h = 1; h < n; h *= 2) {
    for (int64_t i = 0; i < n; i += 2 * h) {
      for (int64_t j = i; j < i + h; ++j) {
        double a = x[j];
        double b = x[j + h];
        x[j] = a + b;
        x[j + h] = a - b;
      }
    }
  }
  double root_n = sqrt((double)n);
  for (int64_t j = 0; j < n; ++j) x[j] = x[j] / root_n;
}

/* Block-local rotation of a bf16 matrix X[rows, cols] (row stride ld, in
 * elements) along the contiguous dimension: every run of blk consecutive
 * elements of a row is replaced by its Walsh-Hadamard transform.
 * Output: v[rows, cols] fp64, dense row-major. */
void halo_oracle_rotate_along_cols(const uint16_t* x, int64_t rows, int64_t cols,
                                   int64_t ld, int64_t blk, double* v) {
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) v[r * cols + c] = halo_oracle_bf16_to_f64(x[r * ld + c]);
    for (int64_t c0 = 0; c0 < cols; c0 += blk) halo_oracle_fwht(&v[r * cols + c0], blk);
  }
}

/* Block-local rotation of a bf16 matrix X[rows, cols] along dimension 0:
 * every run of blk consecutive rows of each column is replaced by its
 * Walsh-Hadamard transform.  Output: v[rows, cols] fp64, dense row-major
 * (same layout as the input; nothing is transposed). */
void halo_oracle_rotate_along_rows(const uint16_t* x, int64_t rows, int64_t cols,
                                   int64_t ld, int64_t blk, double* v) {
  double* col = (double*)malloc(sizeof(double) * (size_t)blk);
  for (int64_t c = 0; c < cols; ++c) {
    for (int64_t r0 = 0; r0 < rows; r0 += blk) {
      for (int64_t i = 0; i < blk; ++i) col[i] = halo_oracle_bf16_to_f64(x[(r0 + i) * ld + c]);
      halo_oracle_fwht(col, blk);
      for (int64_t i = 0; i < blk; ++i) v[(r0 + i) * cols + c] = col[i];
    }
  }
  free(col);
}

/* Random-sign variant of the two rotations above: every element is first
 * multiplied by the sign assigned to its position along the rotated
 * dimension (signs[c] for the contiguous dimension, signs[r] for dimension 0,
 * each +1 or -1), then transformed: H (D x) with D = diag(signs).  The same
 * signs on both GEMM operands keep the product, since (H D)^T (H D) = I
 * [HALO blog page sec. 4.2: every node seeds the Hadamard matrix alike]. */
void halo_oracle_rotate_signed_along_cols(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                          int64_t blk, const int8_t* signs, double* v) {
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c)
      v[r * cols + c] = (double)signs[c] * halo_oracle_bf16_to_f64(x[r * ld + c]);
    for (int64_t c0 = 0; c0 < cols; c0 += blk) halo_oracle_fwht(&v[r * cols + c0], blk);
  }
}

void halo_oracle_rotate_signed_along_rows(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                                          int64_t blk, const int8_t* signs, double* v) {
  double* col = (double*)malloc(sizeof(double) * (size_t)blk);
  for (int64_t c = 0; c < cols; ++c) {
    for (int64_t r0 = 0; r0 < rows; r0 += blk) {
      for (int64_t i = 0; i < blk; ++i)
        col[i] = (double)signs[r0 + i] * halo_oracle_bf16_to_f64(x[(r0 + i) * ld + c]);
      halo_oracle_fwht(col, blk);
      for (int64_t i = 0; i < blk; ++i) v[(r0 + i) * cols + c] = col[i];
    }
  }
  free(col);
}

/* ------------------------------------------------------------------------ */
/* OCP FP8 E4M3 ("fn": no infinities, max finite 448).  Sign, 4 exponent    */
/* bits with bias 7, 3 mantissa bits.  Exponent field 0 holds subnormals    */
/* m/8 * 2^-6; exponent field e >= 1 holds (1 + m/8) * 2^(e-7); the pattern */
/* S.1111.111 is NaN, so the largest finite value is 1.75 * 2^8 = 448.      */
/* ------------------------------------------------------------------------ */
double halo_oracle_e4m3_decode(uint8_t code) {
  int sign = (code >> 7) & 1;
  int e = (code >> 3) & 0xF;
  int m = code & 0x7;
  double mag;
  if (e == 0xF && m == 0x7) return NAN;
  if (e == 0)
    mag = ldexp((double)m / 8.0, -6);
  else
    mag = ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -mag : mag;
}

/* Round-to-nearest-even onto the E4M3 grid, saturating finite values above
 * 448 to 448 (the "satfinite" conversion).  NaN input gives the NaN code. */
uint8_t halo_oracle_e4m3_encode(double t) {
  if (isnan(t)) return 0x7F;
  uint8_t sign = signbit(t) ? 0x80 : 0x00;
  double a = fabs(t);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  /* Spacing of the grid around a: 2^-9 below 2^-6 (subnormals and the first
   * normal binade share it), else 2^(floor(log2 a) - 3). */
  double quantum;
  if (a < ldexp(1.0, -6)) {
    quantum = ldexp(1.0, -9);
  } else {
    int ex;
    frexp(a, &ex); /* a = f * 2^ex, f in [0.5, 1) -> floor(log2 a) = ex - 1 */
    quantum = ldexp(1.0, (ex - 1) - 3);
  }
  double r = nearbyint(a / quantum) * quantum; /* exact: division by 2^k */
  if (r > 448.0) r = 448.0;
  if (r == 0.0) return sign;
  uint8_t bits;
  if (r < ldexp(1.0, -6)) {
    bits = (uint8_t)(r / ldexp(1.0, -9)); /* subnormal: m in 1..7 */
  } else {
    int ex;
    frexp(r, &ex);
    int e = (ex - 1) + 7;                                      /* 1..15 */
    int m = (int)(r / ldexp(1.0, ex - 1) * 8.0) - 8;           /* 0..7  */
    bits = (uint8_t)((e << 3) | m);
  }
  return (uint8_t)(sign | bits);
}

/* Distance from t to the nearest rounding midpoint of the target grid,
 * relative to |t| (infinite when t is 0).  INT8 midpoints are the
 * half-integers; E4M3 midpoints lie halfway between adjacent grid values. */
double halo_oracle_boundary_distance(double t, int qtype) {
  double a = fabs(t);
  if (a == 0.0) return INFINITY;
  double d;
  if (qtype == 0) {
    double mid = floor(a) + 0.5;
    d = fabs(a - mid);
  } else {
    if (a >= 448.0) return INFINITY;
    double quantum;
    if (a < ldexp(1.0, -6)) {
      quantum = ldexp(1.0, -9);
    } else {
      int ex;
      frexp(a, &ex);
      quantum = ldexp(1.0, (ex - 1) - 3);
    }
    double mid = (floor(a / quantum) + 0.5) * quantum;
    d = fabs(a - mid);
  }
  return d / a;
}

/* Array forms of the two functions above (same arithmetic, element by element). */
void halo_oracle_e4m3_encode_array(const double* t, int64_t n, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = halo_oracle_e4m3_encode(t[i]);
}

void halo_oracle_e4m3_decode_array(const uint8_t* codes, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = halo_oracle_e4m3_decode(codes[i]);
}

void halo_oracle_boundary_distance_array(const double* t, int64_t n, int qtype, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = halo_oracle_boundary_distance(t[i], qtype);
}

/* ------------------------------------------------------------------------ */
/* Symmetric absmax quantisation (QWHA page sec. 2.2 quantize, read as      */
/* q = round(x / (absmax / qmax))).  One scale per group; a group is a row  */
/* (axis 0: v[g, :]) or a column (axis 1: v[:, g]) of v[rows, cols].         */
/*   qtype 0: INT8,  qmax 127, q = clip(round_half_even(t), -127, 127)       */
/*   qtype 1: E4M3,  qmax 448, q = e4m3_rne_satfinite(t)                     */
/* with t = v / s and s = (float)(absmax / qmax).  absmax = 0 gives s = 0    */
/* and all-zero codes.  Outputs: codes[rows, cols] (int8 or E4M3 bytes),     */
/* scales[groups] fp32, and t[rows, cols] (the pre-rounding values).         */
/* ------------------------------------------------------------------------ */
void halo_oracle_quantize(const double* v, int64_t rows, int64_t cols, int axis,
                          int qtype, uint8_t* codes, float* scales, double* t_out) {
  const double qmax = (qtype == 0) ? 127.0 : 448.0;
  const int64_t groups = (axis == 0) ? rows : cols;
  const int64_t len = (axis == 0) ? cols : rows;
  fesetround(FE_TONEAREST);
  for (int64_t g = 0; g < groups; ++g) {
    double amax = 0.0;
    for (int64_t i = 0; i < len; ++i) {
      int64_t idx = (axis == 0) ? g * cols + i : i * cols + g;
      double a = fabs(v[idx]);
      if (a > amax) amax = a;
    }
    float s = (float)(amax / qmax);
    scales[g] = s;
    for (int64_t i = 0; i < len; ++i) {
      int64_t idx = (axis == 0) ? g * cols + i : i * cols + g;
      double t = (s == 0.0f) ? 0.0 : v[idx] / (double)s;
      if (t_out) t_out[idx] = t;
      if (qtype == 0) {
        double q = nearbyint(t);
        if (q > 127.0) q = 127.0;
        if (q < -127.0) q = -127.0;
        codes[idx] = (uint8_t)(int8_t)q;
      } else {
        codes[idx] = halo_oracle_e4m3_encode(t);
      }
    }
  }
}

/* Stochastic-rounding variant of the quantiser [QWHA page, sec. 5].  Same
 * scale as above; the code of element idx rounds t = v / s to one of its
 * two grid neighbours lo <= t < hi, taking hi when u < (t - lo) / (hi - lo),
 * with u = rand[idx] / 65536 (16 caller-supplied random bits per element).
 * INT8 grid: the integers, clamped to +-127.  E4M3 grid: the E4M3 values,
 * saturating at 448 (|t| >= 448 gives +-448).  rand[] has the layout of v. */
static double e4m3_quantum(double a) {
  if (a < ldexp(1.0, -6)) return ldexp(1.0, -9);
  int ex;
  frexp(a, &ex);
  return ldexp(1.0, (ex - 1) - 3);
}

void halo_oracle_quantize_stochastic(const double* v, int64_t rows, int64_t cols, int axis, int qtype,
                                     const uint16_t* rand, uint8_t* codes, float* scales, double* t_out) {
  const double qmax = (qtype == 0) ? 127.0 : 448.0;
  const int64_t groups = (axis == 0) ? rows : cols;
  const int64_t len = (axis == 0) ? cols : rows;
  for (int64_t g = 0; g < groups; ++g) {
    double amax = 0.0;
    for (int64_t i = 0; i < len; ++i) {
      int64_t idx = (axis == 0) ? g * cols + i : i * cols + g;
      double a = fabs(v[idx]);
      if (a > amax) amax = a;
    }
    float s = (float)(amax / qmax);
    scales[g] = s;
    for (int64_t i = 0; i < len; ++i) {
      int64_t idx = (axis == 0) ? g * cols + i : i * cols + g;
      double t = (s == 0.0f) ? 0.0 : v[idx] / (double)s;
      double u = (double)rand[idx] / 65536.0;
      if (t_out) t_out[idx] = t;
      if (qtype == 0) {
        double lo = floor(t);
        double q = (u < t - lo) ? lo + 1.0 : lo;
        if (q > 127.0) q = 127.0;
        if (q < -127.0) q = -127.0;
        codes[idx] = (uint8_t)(int8_t)q;
      } else {
        double a = fabs(t);
        double mag;
        if (a >= 448.0) {
          mag = 448.0;
        } else {
          double quantum = e4m3_quantum(a);
          double lo = floor(a / quantum) * quantum;
          mag = (u < (a - lo) / quantum) ? lo + quantum : lo;
        }
        codes[idx] = halo_oracle_e4m3_encode(signbit(t) ? -mag : mag);
      }
    }
  }
}

/* ------------------------------------------------------------------------ */
/* GEMMs on codes.  C[i, j] = sum_k A[i, k] * B[j, k]; A[M, K], B[N, K]     */
/* dense row-major (contraction dimension contiguous).                      */
/* ------------------------------------------------------------------------ */
void halo_oracle_gemm_i8(const int8_t* a, const int8_t* b, int64_t m, int64_t n, int64_t k,
                         int64_t* c) {
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < m; ++i) {
    for (int64_t j = 0; j < n; ++j) {
      int64_t acc = 0;
      for (int64_t p = 0; p < k; ++p) acc += (int64_t)a[i * k + p] * (int64_t)b[j * k + p];
      c[i * n + j] = acc;
    }
  }
}

void halo_oracle_gemm_e4m3(const uint8_t* a, const uint8_t* b, int64_t m, int64_t n, int64_t k,
                           double* c) {
  double lut[256];
  for (int i = 0; i < 256; ++i) lut[i] = halo_oracle_e4m3_decode((uint8_t)i);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < m; ++i) {
    for (int64_t j = 0; j < n; ++j) {
      double acc = 0.0;
      for (int64_t p = 0; p < k; ++p) acc += lut[a[i * k + p]] * lut[b[j * k + p]];
      c[i * n + j] = acc;
    }
  }
}

/* Dequantising product: y[i, j] = acc[i, j] * s_a[i] * s_b[j] in fp64. */
void halo_oracle_dequant(const double* acc, const float* sa, const float* sb, int64_t m,
                         int64_t n, double* y) {
  for (int64_t i = 0; i < m; ++i)
    for (int64_t j = 0; j < n; ++j) y[i * n + j] = acc[i * n + j] * (double)sa[i] * (double)sb[j];
}

/* ------------------------------------------------------------------------ */
/* One rotated quantised GEMM, the unit every large matmul of the layer is   */
/* made of:  both operands rotated along the contraction dimension, each     */
/* quantised with one scale per non-contraction index, multiplied on codes   */
/* with a wide accumulator, dequantised with both scale vectors.             */
/*   a: A[M, K] given as bf16 rows of stride lda when a_kdim_contig, else as */
/*      A^T stored [K, M] (stride lda) and rotated along its dimension 0.    */
/*   b: likewise for B[N, K] (b_kdim_contig) or B^T stored [K, N].           */
/* Output y[M, N] fp64.                                                      */
/* ------------------------------------------------------------------------ */
static void rotate_quantize_operand(const uint16_t* x, int64_t outer, int64_t k, int64_t ld,
                                    int kdim_contig, int64_t blk, int qtype, uint8_t* codes_mk,
                                    float* scales) {
  /* Produces codes in [outer, k] order (contraction dimension contiguous). */
  if (kdim_contig) {
    double* v = (double*)malloc(sizeof(double) * (size_t)(outer * k));
    halo_oracle_rotate_along_cols(x, outer, k, ld, blk, v);
    halo_oracle_quantize(v, outer, k, 0, qtype, codes_mk, scales, NULL);
    free(v);
  } else {
    /* x holds X^T[k, outer]: rotate along its dim 0, one scale per column. */
    double* v = (double*)malloc(sizeof(double) * (size_t)(outer * k));
    uint8_t* c_ko = (uint8_t*)malloc((size_t)(outer * k));
    halo_oracle_rotate_along_rows(x, k, outer, ld, blk, v);
    halo_oracle_quantize(v, k, outer, 1, qtype, c_ko, scales, NULL);
    for (int64_t i = 0; i < outer; ++i)
      for (int64_t p = 0; p < k; ++p) codes_mk[i * k + p] = c_ko[p * outer + i];
    free(c_ko);
    free(v);
  }
}

void halo_oracle_rotated_qgemm(const uint16_t* a, int64_t lda, int a_kdim_contig,
                               const uint16_t* b, int64_t ldb, int b_kdim_contig, int64_t m,
                               int64_t n, int64_t k, int64_t blk, int qtype, double* y,
                               float* sa_out, float* sb_out) {
  uint8_t* aq = (uint8_t*)malloc((size_t)(m * k));
  uint8_t* bq = (uint8_t*)malloc((size_t)(n * k));
  float* sa = (float*)malloc(sizeof(float) * (size_t)m);
  float* sb = (float*)malloc(sizeof(float) * (size_t)n);
  double* acc = (double*)malloc(sizeof(double) * (size_t)(m * n));
  rotate_quantize_operand(a, m, k, lda, a_kdim_contig, blk, qtype, aq, sa);
  rotate_quantize_operand(b, n, k, ldb, b_kdim_contig, blk, qtype, bq, sb);
  if (qtype == 0) {
    int64_t* iacc = (int64_t*)malloc(sizeof(int64_t) * (size_t)(m * n));
    halo_oracle_gemm_i8((const int8_t*)aq, (const int8_t*)bq, m, n, k, iacc);
    for (int64_t i = 0; i < m * n; ++i) acc[i] = (double)iacc[i];
    free(iacc);
  } else {
    halo_oracle_gemm_e4m3(aq, bq, m, n, k, acc);
  }
  halo_oracle_dequant(acc, sa, sb, m, n, y);
  if (sa_out) memcpy(sa_out, sa, sizeof(float) * (size_t)m);
  if (sb_out) memcpy(sb_out, sb, sizeof(float) * (size_t)n);
  free(acc);
  free(sb);
  free(sa);
  free(bq);
  free(aq);
}

/* ------------------------------------------------------------------------ */
/* The linear layer (nn.Linear shapes X[M,K], W[N,K], Y = X W^T [M,N]).     */
/* HALO paper page, abstract: rotations placed in both passes so that all    */
/* three large matmuls run in low precision; each GEMM rotates both operands */
/* along its own contraction dimension.                                     */
/* ------------------------------------------------------------------------ */
/* Y[M, N] = X W^T: contraction over K, both operands K-contiguous. */
void halo_oracle_linear_fwd(const uint16_t* x, const uint16_t* w, int64_t m, int64_t n, int64_t k,
                            int64_t blk, int qtype, double* y) {
  halo_oracle_rotated_qgemm(x, k, 1, w, k, 1, m, n, k, blk, qtype, y, NULL, NULL);
}

/* dX[M, K] = dY W: contraction over N.  A = dY[M, N] (N contiguous);
 * B[K, N] = W^T, stored as W[N, K] and rotated along its dimension 0. */
void halo_oracle_linear_bwd_dx(const uint16_t* dy, const uint16_t* w, int64_t m, int64_t n,
                               int64_t k, int64_t blk, int qtype, double* dx) {
  halo_oracle_rotated_qgemm(dy, n, 1, w, k, 0, m, k, n, blk, qtype, dx, NULL, NULL);
}

/* dW[N, K] = dY^T X: contraction over M.  A[N, M] = dY^T stored as dY[M, N];
 * B[K, M] = X^T stored as X[M, K]; both rotated along their dimension 0. */
void halo_oracle_linear_bwd_dw(const uint16_t* dy, const uint16_t* x, int64_t m, int64_t n,
                               int64_t k, int64_t blk, int qtype, double* dw) {
  halo_oracle_rotated_qgemm(dy, n, 0, x, k, 0, n, k, m, blk, qtype, dw, NULL, NULL);
}

/* ------------------------------------------------------------------------ */
/* Group-wise scales (QWHA page sec. 3.1, the quantiser's group_quantize:    */
/* the values are cut into groups of group_size consecutive elements, each   */
/* group with its own scale max|x| / qmax; sec. 3.2 recommends 64 and sec. 6 */
/* 32-128).  Here a group runs along the GEMM's contraction dimension:       */
/*   along = 1: `group` consecutive elements of a row; scales[rows][cols/g]  */
/*   along = 0: `group` consecutive rows of a column;  scales[rows/g][cols]  */
/* Within a group: s = (float)(amax / qmax) and the element rule of          */
/* halo_oracle_quantize (round half to even and clamp to +-127, or E4M3).    */
/* rows (along 0) or cols (along 1) must be a multiple of group.             */
/* ------------------------------------------------------------------------ */
void halo_oracle_quantize_grouped(const double* v, int64_t rows, int64_t cols, int along, int64_t group,
                                  int qtype, uint8_t* codes, float* scales, double* t_out) {
  const double qmax = (qtype == 0) ? 127.0 : 448.0;
  const int64_t outer = (along == 1) ? rows : cols;          /* rows (along 1) or columns (along 0) */
  const int64_t ngroups = ((along == 1) ? cols : rows) / group;
  fesetround(FE_TONEAREST);
  for (int64_t o = 0; o < outer; ++o) {
    for (int64_t g = 0; g < ngroups; ++g) {
      double amax = 0.0;
      for (int64_t e = 0; e < group; ++e) {
        int64_t idx = (along == 1) ? o * cols + g * group + e : (g * group + e) * cols + o;
        double a = fabs(v[idx]);
        if (a > amax) amax = a;
      }
      float s = (float)(amax / qmax);
      if (along == 1)
        scales[o * ngroups + g] = s;
      else
        scales[g * cols + o] = s;
      for (int64_t e = 0; e < group; ++e) {
        int64_t idx = (along == 1) ? o * cols + g * group + e : (g * group + e) * cols + o;
        double t = (s == 0.0f) ? 0.0 : v[idx] / (double)s;
        if (t_out) t_out[idx] = t;
        if (qtype == 0) {
          double q = nearbyint(t);
          if (q > 127.0) q = 127.0;
          if (q < -127.0) q = -127.0;
          codes[idx] = (uint8_t)(int8_t)q;
        } else {
          codes[idx] = halo_oracle_e4m3_encode(t);
        }
      }
    }
  }
}

/* Product of group-quantised operands, both with the contraction dimension  */
/* contiguous: A codes [M, K] with scales sa[M][K/g], B codes [N, K] with    */
/* scales sb[N][K/g]:                                                        */
/*   y[i, j] = sum_G sa[i][G] * sb[j][G] * sum_{k in group G} a[i, k] b[j, k] */
/* Each group's sum is exact (int64 for INT8 codes, fp64 of the decoded E4M3 */
/* values); the rest in fp64.                                                */
void halo_oracle_gemm_grouped(const uint8_t* a, const float* sa, const uint8_t* b, const float* sb, int64_t m,
                              int64_t n, int64_t k, int64_t group, int qtype, double* y) {
  const int64_t ng = k / group;
  double lut[256];
  for (int i = 0; i < 256; ++i) lut[i] = halo_oracle_e4m3_decode((uint8_t)i);
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < m; ++i) {
    for (int64_t j = 0; j < n; ++j) {
      double sum = 0.0;
      for (int64_t g = 0; g < ng; ++g) {
        double part;
        if (qtype == 0) {
          int64_t acc = 0;
          for (int64_t p = g * group; p < (g + 1) * group; ++p)
            acc += (int64_t)(int8_t)a[i * k + p] * (int64_t)(int8_t)b[j * k + p];
          part = (double)acc;
        } else {
          part = 0.0;
          for (int64_t p = g * group; p < (g + 1) * group; ++p) part += lut[a[i * k + p]] * lut[b[j * k + p]];
        }
        sum += part * (double)sa[i * ng + g] * (double)sb[j * ng + g];
      }
      y[i * n + j] = sum;
    }
  }
}

int halo_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
