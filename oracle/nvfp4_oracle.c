/*
 * nvfp4_oracle.c -- plain scalar CPU oracle for the NVFP4 QAD hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * reference that the CUDA kernels are checked against.  Only the test suite,
 * the smoke check and the CPU-baseline leg of the benchmark may load it; the
 * product library never links, imports or calls it, and it shares no code,
 * header, table or constant generator with the CUDA sources.
 *
 * Sources followed (web pages on NVFP4 quantization-aware distillation):
 *  [FMT]  "NVIDIA AI bringt Nemotron-3-Nano-30B auf NVFP4 mit Quantization
 *         Conscious Distillation (QAD) ..." -- section "NVFP4-Format und warum
 *         es wichtig ist?" and "Wichtige Erkenntnisse": a 4-bit floating-point
 *         element, blocks of 16, an E4M3 (FP8) scale per block and an FP32
 *         scale per tensor.
 *  [MODE] "使用量化感知蒸馏技术构建Nemotron 3.5 Lightning NVFP4模型" --
 *         section "量化尺度处理策略": dynamic-scale QAD recomputes weight and
 *         activation scales from the max every step; frozen-scale QAD keeps
 *         the calibrated scales fixed and only updates the weights.
 *  [KD]   same page, "QAD的工作原理", and the Nemotron-3-Nano page "Von QAT zu
 *         QAD": the student is trained to match the frozen BF16 teacher's
 *         output-token distribution with a KL-divergence loss.
 *  [W4A4] "Qwen3.6-35B-A3B W4A4 NVFP4 ..." tutorial page, "为什么目标是 W4A4":
 *         activations are quantized to NVFP4 too, so the GEMM consumes two
 *         NVFP4 operands.
 *
 * Where the pages leave a step open, the reading taken is written next to the
 * step.  The E2M1 value set {0, .5, 1, 1.5, 2, 3, 4, 6} with a sign bit and
 * round-to-nearest-even are taken from the benchmark spec that names the
 * format; the pages only say "4-bit floating point".
 *
 * Precision: the quantizer steps (scale derivation, division, products) are
 * done in IEEE binary32 with round-to-nearest-even, one operation at a time,
 * because the kernels must reproduce the same integer codes; GEMM and KL sums
 * are done in binary64.  Build with -O2 -ffp-contract=off and without
 * -ffast-math so that every float operation is rounded exactly once.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_SHAPE 2

/* Scale modes, [MODE]. */
#define ORACLE_DYNAMIC 0       /* s_g and s_b derived from the data           */
#define ORACLE_FROZEN_GLOBAL 1 /* s_g given (activation amax frozen), s_b derived */
#define ORACLE_FROZEN_ALL 2    /* s_g and s_b both given (frozen weights)      */

/* ------------------------------------------------------------------------ */
/* Threads                                                                   */
/* ------------------------------------------------------------------------ */

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

/* ------------------------------------------------------------------------ */
/* E2M1: sign bit (bit 3) and a 3-bit magnitude index.                       */
/* ------------------------------------------------------------------------ */

/* Magnitude of each 3-bit index: exponent 2 bits, mantissa 1 bit, bias 1;
 * index 1 is the single subnormal (0.5). */
static const double E2M1_MAGNITUDE[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double oracle_e2m1_value(int code) {
  double m = E2M1_MAGNITUDE[code & 7];
  return (code & 8) ? -m : m;
}

/* Nearest E2M1 value to v by enumeration; |v| >= 6 saturates to 6; a tie
 * between two neighbours goes to the even index (even mantissa bit).  The
 * sign bit is copied from v, so a negative value that rounds to zero gives
 * code 8 (negative zero). */
int oracle_e2m1_encode(float v) {
  int sign = signbit(v) ? 8 : 0;
  double a = fabs((double)v);
  int best = 7;
  if (a < 6.0) {
    double best_dist = a; /* distance to index 0 */
    best = 0;
    for (int i = 1; i < 8; ++i) {
      double dist = fabs(a - E2M1_MAGNITUDE[i]);
      /* candidates are visited in increasing order, so a tie is always with
       * index i-1; keep i only if it is the even one. */
      if (dist < best_dist || (dist == best_dist && (i % 2) == 0)) {
        best = i;
        best_dist = dist;
      }
    }
  }
  return sign | best;
}

/* ------------------------------------------------------------------------ */
/* E4M3 ("fn" variant): bias 7, no infinities, 0x7F/0xFF are NaN, max 448.   */
/* ------------------------------------------------------------------------ */

double oracle_e4m3_value(int code) {
  int e = (code >> 3) & 15;
  int m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    mag = ldexp((double)m, -9); /* subnormal: m/8 * 2^(1-7) */
  else
    mag = ldexp(1.0 + m / 8.0, e - 7);
  return (code & 0x80) ? -mag : mag;
}

/* Nearest non-negative finite E4M3 code to t >= 0 by enumeration over the
 * 127 finite codes 0x00..0x7E, t >= 448 saturating to 448 (0x7E); ties go to
 * the even code (even mantissa bit).  Values below half of the smallest
 * subnormal round to +0. */
int oracle_e4m3_encode_nonneg(float t) {
  double a = (double)t;
  if (!(a < 448.0)) return 0x7E;
  int best = 0;
  double best_dist = a;
  for (int c = 1; c <= 0x7E; ++c) {
    double dist = fabs(a - oracle_e4m3_value(c));
    if (dist < best_dist || (dist == best_dist && (c % 2) == 0)) {
      best = c;
      best_dist = dist;
    }
  }
  return best;
}

/* ------------------------------------------------------------------------ */
/* bf16 rounding (8 significant bits, binary32 exponent range), RNE.         */
/* ------------------------------------------------------------------------ */

/* Round a double to the nearest bf16 value (ties to even significand) and
 * return its 16-bit pattern.  Written from the definition: the quantum at
 * magnitude 2^e (normal range) is 2^(e-7); below 2^-126 it is 2^-133. */
uint16_t oracle_bf16_round(double x) {
  if (isnan(x)) return 0x7FC0;
  int neg = signbit(x) ? 1 : 0;
  double a = fabs(x);
  double r;
  if (a == 0.0) {
    r = 0.0;
  } else {
    int e;
    (void)frexp(a, &e);      /* a = f * 2^e, f in [0.5, 1): a in [2^(e-1), 2^e) */
    int q = (e - 1) - 7;     /* quantum exponent of an 8-significant-bit value */
    if (q < -133) q = -133;  /* subnormal bf16 spacing */
    r = nearbyint(ldexp(a, -q)); /* default rounding mode: ties to even */
    r = ldexp(r, q);
  }
  /* largest finite bf16 is (2 - 2^-7) * 2^127; anything that rounded up to
   * 2^128 or beyond is +-inf */
  float f = (r >= ldexp(1.0, 128)) ? INFINITY : (float)r; /* exact: <= 8 significant bits */
  uint32_t bits;
  memcpy(&bits, &f, 4);
  uint16_t h = (uint16_t)(bits >> 16);
  if (neg) h |= 0x8000;
  return h;
}

/* oracle_bf16_round over an array: out[i] = bf16 pattern of x[i]. */
void oracle_bf16_round_array(const double* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_round(x[i]);
}

/* ------------------------------------------------------------------------ */
/* Quantize / dequantize, [FMT] + [MODE].                                    */
/* ------------------------------------------------------------------------ */

/* Per-tensor scale in dynamic mode: the decode scale s_g = amax / (6 * 448),
 * so that the largest block scale lands at the top of the E4M3 range and the
 * largest element at the top of the E2M1 range.  Reading: the pages name an
 * "FP32 scale per tensor"; this is the decode direction (x ~ q * s_b * s_g). */
float oracle_tensor_amax(const float* x, int64_t rows, int64_t cols, int64_t ld) {
  float amax = 0.0f;
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      float a = fabsf(x[r * ld + c]);
      if (a > amax) amax = a;
    }
  return amax;
}

float oracle_global_scale_from_amax(float amax) {
  return amax / 2688.0f; /* 2688 = 6 * 448 */
}

/* Quantize a rows x cols binary32 matrix (row stride ld elements) into packed
 * E2M1 codes [rows][cols/2] (even element in the low nibble), E4M3 block
 * scales [rows][cols/16] (blocks of 16 along the contiguous last dimension)
 * and the per-tensor scale *s_g.
 *   DYNAMIC        : *s_g = amax/2688 (output), s_b computed (output)
 *   FROZEN_GLOBAL  : *s_g given,                 s_b computed (output)
 *   FROZEN_ALL     : *s_g given,                 s_b given    (input)
 * Block scale: s_b = E4M3_RNE_sat( a_b / (6 * s_g) ), where a_b is the block
 * max |x| and 6*s_g is first rounded to binary32; s_b = 0 when s_g == 0.
 * Element code: d = value(s_b) * s_g (binary32); code = E2M1_RNE_sat(x / d),
 * the quotient rounded to binary32 first; every code of a block with d == 0
 * is +0. */
int oracle_quantize(const float* x, int64_t rows, int64_t cols, int64_t ld, int mode,
                    float* s_g, uint8_t* s_b, uint8_t* codes) {
  if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols) return ORACLE_ERR_SHAPE;
  if (!s_g || (rows > 0 && (!x || !s_b || !codes))) return ORACLE_ERR_ARG;
  if (mode == ORACLE_DYNAMIC) *s_g = oracle_global_scale_from_amax(oracle_tensor_amax(x, rows, cols, ld));
  else if (mode != ORACLE_FROZEN_GLOBAL && mode != ORACLE_FROZEN_ALL) return ORACLE_ERR_ARG;
  const float sg = *s_g;
  const int64_t nblk = cols / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nblk; ++b) {
      const float* xb = x + r * ld + b * 16;
      int sb;
      if (mode == ORACLE_FROZEN_ALL) {
        sb = s_b[r * nblk + b];
      } else if (sg == 0.0f) {
        sb = 0;
      } else {
        float ab = 0.0f;
        for (int i = 0; i < 16; ++i)
          if (fabsf(xb[i]) > ab) ab = fabsf(xb[i]);
        float denom = 6.0f * sg; /* rounded to binary32 */
        float t = ab / denom;    /* rounded to binary32 */
        sb = oracle_e4m3_encode_nonneg(t);
        s_b[r * nblk + b] = (uint8_t)sb;
      }
      float d = (float)oracle_e4m3_value(sb) * sg; /* binary32 product */
      uint8_t* cb = codes + r * (cols / 2) + b * 8;
      for (int j = 0; j < 8; ++j) {
        int lo = 0, hi = 0;
        if (d != 0.0f) {
          float q0 = xb[2 * j] / d;     /* binary32 quotient */
          float q1 = xb[2 * j + 1] / d;
          lo = oracle_e2m1_encode(q0);
          hi = oracle_e2m1_encode(q1);
        }
        cb[j] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
  return ORACLE_OK;
}

/* Dequantize: x_hat = value(code) * d with d = value(s_b) * s_g, each product
 * rounded to binary32; written as binary32 (out_f32) and/or as bf16 bits
 * rounded to nearest even (out_bf16).  Either output may be NULL. */
int oracle_dequantize(const uint8_t* codes, const uint8_t* s_b, float s_g, int64_t rows,
                      int64_t cols, float* out_f32, uint16_t* out_bf16) {
  if (rows < 0 || cols < 0 || cols % 16 != 0) return ORACLE_ERR_SHAPE;
  const int64_t nblk = cols / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t c = 0; c < cols; ++c) {
      int byte = codes[r * (cols / 2) + c / 2];
      int code = (c % 2 == 0) ? (byte & 15) : (byte >> 4);
      float d = (float)oracle_e4m3_value(s_b[r * nblk + c / 16]) * s_g;
      float v = (float)oracle_e2m1_value(code) * d;
      if (out_f32) out_f32[r * cols + c] = v;
      if (out_bf16) out_bf16[r * cols + c] = oracle_bf16_round((double)v);
    }
  }
  return ORACLE_OK;
}

/* Fake quantization (simulated quantization in the student forward pass,
 * [KD]/[MODE]): dequantize(quantize(x)).  Scales follow `mode` exactly as in
 * oracle_quantize and are returned through s_g / s_b. */
int oracle_fake_quant(const float* x, int64_t rows, int64_t cols, int64_t ld, int mode, float* s_g,
                      uint8_t* s_b, uint8_t* codes_scratch, float* out_f32, uint16_t* out_bf16) {
  int st = oracle_quantize(x, rows, cols, ld, mode, s_g, s_b, codes_scratch);
  if (st != ORACLE_OK) return st;
  return oracle_dequantize(codes_scratch, s_b, *s_g, rows, cols, out_f32, out_bf16);
}

/* ------------------------------------------------------------------------ */
/* MSE block-scale calibration for frozen-scale QAD.                          */
/* ------------------------------------------------------------------------ */

/* Frozen-scale QAD starts from scales an MSE calibration chose (Nemotron 3.5
 * Lightning article, "量化尺度处理策略"); the page gives no formula beyond
 * "MSE".  Reading: with the tensor scale s_g given, every block's E4M3 scale
 * is the code c (all 127 finite non-negative codes, in increasing order)
 * whose fake quantization of the block has the least squared error
 *   err(c) = sum_i (x_i - x^_i)^2,  x^_i = value(q_i) * d,  d = value(c) * s_g,
 *   q_i = E2M1_RNE_sat(x_i / d)  (q_i = 0 for every i when d == 0),
 * each operation in binary32 with one rounding, the sum accumulated in
 * element order as err = fma(diff, diff, err); the smallest code wins a tie.
 * s_b: rows x cols/16 (output); err_out (may be NULL): the least error per
 * block. */
int oracle_calibrate_mse(const float* x, int64_t rows, int64_t cols, int64_t ld, float s_g, uint8_t* s_b,
                         float* err_out) {
  if (rows < 0 || cols < 0 || cols % 16 != 0 || ld < cols) return ORACLE_ERR_SHAPE;
  if (rows > 0 && (!x || !s_b)) return ORACLE_ERR_ARG;
  const int64_t nblk = cols / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nblk; ++b) {
      const float* xb = x + r * ld + b * 16;
      int best = 0;
      float best_err = INFINITY;
      for (int c = 0; c < 127; ++c) {
        const float d = (float)oracle_e4m3_value(c) * s_g; /* binary32 product */
        float err = 0.0f;
        for (int i = 0; i < 16; ++i) {
          float xh = 0.0f;
          if (d != 0.0f) {
            const float q = xb[i] / d; /* binary32 quotient */
            xh = (float)oracle_e2m1_value(oracle_e2m1_encode(q)) * d;
          }
          const float diff = xb[i] - xh;
          err = fmaf(diff, diff, err);
        }
        if (err < best_err) {
          best_err = err;
          best = c;
        }
      }
      s_b[r * nblk + b] = (uint8_t)best;
      if (err_out) err_out[r * nblk + b] = best_err;
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Block-scale layout used by the block-scaled tensor-core MMA.             */
/* ------------------------------------------------------------------------ */

/* Byte offset of block scale (row r, 16-block kb) in the tensor-core layout:
 * the scale matrix is cut into tiles of 128 rows x 4 blocks (512 bytes),
 * tiles ordered with the block index fastest; inside a tile, row r and block
 * kb sit at (r % 32) * 16 + ((r / 32) % 4) * 4 + (kb % 4).  `cols` is the
 * element count of a row, so a row holds cols/16 blocks, padded to 4. */
int64_t oracle_swizzled_scale_offset(int64_t r, int64_t kb, int64_t cols) {
  int64_t kchunks = (cols / 16 + 3) / 4;
  int64_t tile = (r / 128) * kchunks + kb / 4;
  int64_t rr = r % 128;
  return tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (kb % 4);
}

/* Scatter row-major block scales [rows][cols/16] into the layout above; the
 * padding bytes (rows up to a multiple of 128, blocks up to a multiple of 4)
 * are set to 0. */
int oracle_swizzle_scales(const uint8_t* s_b, int64_t rows, int64_t cols, uint8_t* out) {
  if (rows < 0 || cols < 0 || cols % 16 != 0) return ORACLE_ERR_SHAPE;
  int64_t nblk = cols / 16;
  int64_t total = ((rows + 127) / 128) * 128 * ((nblk + 3) / 4) * 4;
  memset(out, 0, (size_t)total);
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t kb = 0; kb < nblk; ++kb) out[oracle_swizzled_scale_offset(r, kb, cols)] = s_b[r * nblk + kb];
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* W4A4 GEMM, [W4A4]: C = (s_gA * s_gB) * sum_k (vA * s_bA)(vB * s_bB).      */
/* ------------------------------------------------------------------------ */

/* A is M x K, B is N x K (both quantized along K, row-major codes and
 * row-major block scales); C[m][n] = sum_k A_hat[m][k] * B_hat[n][k], i.e.
 * A_hat * B_hat^T, accumulated in binary64 (each product is exact there).
 * Rows are independent, so they are split across threads. */
int oracle_gemm_w4a4(const uint8_t* a_codes, const uint8_t* a_sb, float a_sg,
                     const uint8_t* b_codes, const uint8_t* b_sb, float b_sg,
                     int64_t M, int64_t N, int64_t K, double* c) {
  if (M < 0 || N < 0 || K < 0 || K % 16 != 0) return ORACLE_ERR_SHAPE;
  const int64_t kb = K / 16;
  const double alpha = (double)a_sg * (double)b_sg;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        int ba = a_codes[m * (K / 2) + k / 2];
        int bb = b_codes[n * (K / 2) + k / 2];
        int qa = (k % 2 == 0) ? (ba & 15) : (ba >> 4);
        int qb = (k % 2 == 0) ? (bb & 15) : (bb >> 4);
        double xa = oracle_e2m1_value(qa) * oracle_e4m3_value(a_sb[m * kb + k / 16]);
        double xb = oracle_e2m1_value(qb) * oracle_e4m3_value(b_sb[n * kb + k / 16]);
        acc += xa * xb;
      }
      c[m * N + n] = alpha * acc;
    }
  }
  return ORACLE_OK;
}

/* Same sum for a subset of A's rows: rows[i] selects the A row written to
 * c[i][*].  Used to check large products on sampled rows. */
int oracle_gemm_w4a4_rows(const uint8_t* a_codes, const uint8_t* a_sb, float a_sg,
                          const uint8_t* b_codes, const uint8_t* b_sb, float b_sg,
                          int64_t N, int64_t K, const int64_t* rows, int64_t nrows, double* c) {
  if (N < 0 || K < 0 || K % 16 != 0 || nrows < 0) return ORACLE_ERR_SHAPE;
  const int64_t kb = K / 16;
  const double alpha = (double)a_sg * (double)b_sg;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t i = 0; i < nrows; ++i) {
    int64_t m = rows[i];
    for (int64_t n = 0; n < N; ++n) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        int ba = a_codes[m * (K / 2) + k / 2];
        int bb = b_codes[n * (K / 2) + k / 2];
        int qa = (k % 2 == 0) ? (ba & 15) : (ba >> 4);
        int qb = (k % 2 == 0) ? (bb & 15) : (bb >> 4);
        double xa = oracle_e2m1_value(qa) * oracle_e4m3_value(a_sb[m * kb + k / 16]);
        double xb = oracle_e2m1_value(qb) * oracle_e4m3_value(b_sb[n * kb + k / 16]);
        acc += xa * xb;
      }
      c[i * N + n] = alpha * acc;
    }
  }
  return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* KL-divergence distillation loss, [KD].                                    */
/* ------------------------------------------------------------------------ */

/* Log-softmax of u = z / T for one row, in binary64: log p = u - lse(u),
 * lse = m + log(sum exp(u - m)) with m = max u. */
static void log_softmax_row(const double* z, int64_t V, double T, double* logp) {
  double m = -INFINITY;
  for (int64_t v = 0; v < V; ++v)
    if (z[v] / T > m) m = z[v] / T;
  double s = 0.0;
  for (int64_t v = 0; v < V; ++v) s += exp(z[v] / T - m);
  double lse = m + log(s);
  for (int64_t v = 0; v < V; ++v) logp[v] = z[v] / T - lse;
}

/* Forward KL(p_t || p_s) per row with p = softmax(z / T):
 *   row_kl[i] = sum_v p_t[v] * (log p_t[v] - log p_s[v])
 *   *loss     = (1/N) * sum_i row_kl[i]            (summed in row order)
 *   grad[i][v]= grad_scale * (p_s[v] - p_t[v]) / T (d loss_i / d z_s, optional)
 * Teacher and student are rows x V with row stride ld.  Reading: no T^2
 * factor and a mean over tokens (the pages state neither).  `work` must hold
 * 2*V doubles per thread (threads * 2 * V); rows are split across threads. */
int oracle_kl(const double* teacher, const double* student, int64_t rows, int64_t V, int64_t ld,
              double T, double grad_scale, double* row_kl, double* loss, double* grad,
              double* work, int threads) {
  if (rows < 0 || V <= 0 || ld < V || !(T > 0.0)) return ORACLE_ERR_SHAPE;
  if (threads < 1) threads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(threads)
  for (int64_t i = 0; i < rows; ++i) {
    int tid = 0;
#ifdef _OPENMP
    tid = omp_get_thread_num();
#endif
    double* lpt = work + (size_t)tid * 2 * V;
    double* lps = lpt + V;
    log_softmax_row(teacher + i * ld, V, T, lpt);
    log_softmax_row(student + i * ld, V, T, lps);
    double kl = 0.0;
    for (int64_t v = 0; v < V; ++v) kl += exp(lpt[v]) * (lpt[v] - lps[v]);
    row_kl[i] = kl;
    if (grad)
      for (int64_t v = 0; v < V; ++v) grad[i * V + v] = grad_scale * (exp(lps[v]) - exp(lpt[v])) / T;
  }
  if (loss) {
    double acc = 0.0;
    for (int64_t i = 0; i < rows; ++i) acc += row_kl[i];
    *loss = rows > 0 ? acc / (double)rows : 0.0;
  }
  return ORACLE_OK;
}
