/*
 * mx_oracle.c -- plain fp64 CPU oracle for MXFP8 block scaling of SiTU-GLU
 * outputs.
 *
 * TEST INFRASTRUCTURE ONLY, like situ_oracle.c (built into the same library).
 * The CUDA path shares no code, header or constant with it.
 *
 * The block format is the OCP Microscaling Formats (MX) Specification v1.0
 * (public; the pages only name the MXFP8 and NVFP4 recipes that were tested
 * -- Megatron-LM PR #6673, "Test results"):
 *   * MXFP8 = blocks of 32 elements, each element an FP8 E4M3 code, the block
 *     sharing one E8M0 scale X = 2^(S - 127), S = 0..254 (S = 255 is NaN).
 *   * E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits; no infinities;
 *     S.1111.111 is NaN, so the largest normal is 1.75 * 2^8 = 448; exponent
 *     field 0 holds the subnormals m/8 * 2^-6.
 *   * Conversion of a block of reals V_i (the spec's FP32-vector-to-MX
 *     conversion): shared exponent e = floor(log2(max_i |V_i|)) - emax,
 *     emax = 8 (the exponent of E4M3's largest normal); X = 2^e; each
 *     P_i = V_i / X rounded to nearest-even E4M3, clamped to +-448.
 * A second scale rule (the no-clamp rule, rule 1 below) takes the smallest
 * e with max_i |V_i| / 2^e <= 448, so that no element is clamped.
 *
 * Readings (where the spec leaves a choice to the implementation): a block
 * whose largest magnitude is 0 takes e = -127 (the smallest scale); e is
 * clamped to [-127, 127]; a block holding a NaN or an infinity gets the NaN
 * scale (255) and NaN element codes.
 *
 * Pinned by tests/test_oracle_pins.py (torch's float8_e4m3fn conversion and
 * decoding, the spec's closed forms, the scale rules' defining inequalities,
 * planted mutants 14-19).
 */
#include <math.h>
#include <stdint.h>

#ifndef SITU_ORACLE_MUTANT
#define SITU_ORACLE_MUTANT 0
#endif

#define MX_BLOCK 32
#define E4M3_MAX 448.0 /* 1.75 * 2^8 */
#define E4M3_EMAX 8
#define MX_RULE_OCP 0
#define MX_RULE_CEIL 1
#define MX_SCALE_NAN 128 /* returned by situ_oracle_mx_scale_exp for a NaN scale */

/* Round a non-negative real to the nearest E4M3 magnitude, ties to even,
 * clamped to 448; returns the 7-bit magnitude code. */
static int e4m3_magnitude_code(double a) {
#if SITU_ORACLE_MUTANT == 16
  if (a >= 464.0) return 0x7F; /* planted: overflow to NaN instead of clamping */
#endif
  if (a >= E4M3_MAX) return 0x7E;
  /* spacing of E4M3 values near a: 2^(k - 3) in the binade [2^k, 2^(k+1)),
   * k >= -6; the subnormals below 2^-6 are 2^-9 apart. */
  int k;
#if SITU_ORACLE_MUTANT == 18
  if (a < ldexp(1.0, -6)) {
    k = -7; /* planted: subnormal spacing 2^-10 */
  } else {
#else
  if (a < ldexp(1.0, -6)) {
    k = -6;
  } else {
#endif
    int ex;
    frexp(a, &ex); /* a = f 2^ex, f in [0.5, 1) */
    k = ex - 1;
  }
  const double q = ldexp(1.0, k - 3);
#if SITU_ORACLE_MUTANT == 17
  const double n = round(a / q); /* planted: ties away from zero */
#else
  const double n = rint(a / q); /* a / q is exact; rint rounds ties to even */
#endif
  const double v = n * q;
  if (v == 0.0) return 0;
  if (v >= E4M3_MAX) return 0x7E;
  if (v < ldexp(1.0, -6)) return (int)(v / ldexp(1.0, -9)); /* subnormal: m 2^-9 */
  int ex;
  const double f = frexp(v, &ex); /* v = (2 f) 2^(ex - 1) */
  const int e_field = (ex - 1) + 7;
  const int m = (int)((2.0 * f - 1.0) * 8.0);
  return (e_field << 3) | m;
}

/* E4M3 code of x: round to nearest even, clamp to +-448 (infinities too);
 * NaN -> 0x7F. */
int situ_oracle_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  return (signbit(x) ? 0x80 : 0) | e4m3_magnitude_code(fabs(x));
}

/* Value of an E4M3 code (NaN for S.1111.111). */
double situ_oracle_e4m3_decode(int code) {
  const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ldexp((double)m, -9);
  else
    v = ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* Shared exponent e of a block whose largest magnitude is amax (X = 2^e), or
 * MX_SCALE_NAN.  rule 0: floor(log2 amax) - 8; rule 1: smallest e with
 * amax <= 448 2^e.  Clamped to [-127, 127]; amax = 0 gives -127. */
int situ_oracle_mx_scale_exp(double amax, int rule) {
  if (isnan(amax) || isinf(amax)) return MX_SCALE_NAN;
  if (amax == 0.0) return -127;
  int ex;
  frexp(amax, &ex);
  const int k = ex - 1; /* floor(log2 amax), exact */
#if SITU_ORACLE_MUTANT == 15
  int e = k - (E4M3_EMAX - 1); /* planted: emax 7 */
#elif SITU_ORACLE_MUTANT == 14
  int e = (amax == ldexp(1.0, k)) ? k - E4M3_EMAX : k + 1 - E4M3_EMAX; /* planted: ceil(log2) */
#else
  int e = k - E4M3_EMAX;
#endif
  if (rule == MX_RULE_CEIL) {
    /* amax >= 2^k > 448 2^(k - 9), so e = k - 8 or k - 7 */
#if SITU_ORACLE_MUTANT == 19
    if (amax >= ldexp(E4M3_MAX, e)) e += 1; /* planted: >= at the boundary */
#else
    if (amax > ldexp(E4M3_MAX, e)) e += 1;
#endif
  }
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* MXFP8 quantisation of v[rows, cols] (row pitch v_stride elements): blocks of
 * 32 consecutive columns of a row.  codes[rows, cols] (row pitch cols) and
 * scales[rows, cols / 32] (row pitch cols / 32) receive the E4M3 codes and
 * the E8M0 scale bytes e + 127 (255 for NaN).  Returns 0, or -1 when cols is
 * not a multiple of 32. */
int situ_oracle_mxfp8_quantize(const double *v, int64_t rows, int64_t cols, int64_t v_stride, int rule,
                               uint8_t *codes, uint8_t *scales) {
  if (cols % MX_BLOCK != 0 || rows < 0) return -1;
  const int64_t nblk = cols / MX_BLOCK;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nblk; ++b) {
      const double *blk = v + r * v_stride + b * MX_BLOCK;
      double amax = 0.0;
      int special = 0;
      for (int i = 0; i < MX_BLOCK; ++i) {
        if (isnan(blk[i]) || isinf(blk[i])) special = 1;
        else if (fabs(blk[i]) > amax) amax = fabs(blk[i]);
      }
      const int e = special ? MX_SCALE_NAN : situ_oracle_mx_scale_exp(amax, rule);
      scales[r * nblk + b] = (uint8_t)(e == MX_SCALE_NAN ? 255 : e + 127);
      for (int i = 0; i < MX_BLOCK; ++i)
        codes[r * cols + b * MX_BLOCK + i] =
            (uint8_t)(e == MX_SCALE_NAN ? 0x7F : situ_oracle_e4m3_encode(blk[i] / ldexp(1.0, e)));
    }
  }
  return 0;
}

/* situ_oracle_e4m3_encode over n values. */
void situ_oracle_e4m3_encode_n(const double *x, int64_t n, uint8_t *codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)situ_oracle_e4m3_encode(x[i]);
}

/* ---- NVFP4 --------------------------------------------------------------
 * The NVFP4 recipe named beside MXFP8 (Megatron-LM PR #6673, "Test results";
 * the format is NVIDIA's public NVFP4 definition, not on the pages):
 *   * elements are FP4 E2M1 codes: sign, 2 exponent bits (bias 1), 1 mantissa
 *     bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinities or NaN;
 *   * every 16 consecutive elements of a row share one FP8 E4M3 scale s_b;
 *   * the tensor has one fp32 scale: with A = max |V| over the tensor,
 *     S_enc = 448 * 6 / A (S_enc = 1 when A = 0), and the decoded value of a
 *     code q in block b is q * s_b / S_enc.
 * Conversion, read plainly in exact arithmetic with one rounding per stored
 * number: s_b = E4M3(amax_b * S_enc / 6) (nearest even, clamped to 448);
 * q_i = E2M1(V_i * S_enc / s_b) (nearest even, clamped to +-6); a block whose
 * scale code is zero gets zero codes.  A NaN or infinite value gives the NaN
 * block scale (0x7F) and zero codes (E2M1 has no NaN). */

#define E2M1_MAX 6.0

/* E2M1 code (4 bits: sign << 3 | magnitude code) of x, nearest even, clamped to 6. */
int situ_oracle_e2m1_encode(double x) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  if (isnan(x)) return 0;
  const int s = signbit(x) ? 8 : 0;
  double a = fabs(x);
  if (a >= E2M1_MAX) return s | 7;
  int best = 0;
  for (int k = 1; k < 8; ++k) {
    const double dk = fabs(a - mag[k]), db = fabs(a - mag[best]);
#if SITU_ORACLE_MUTANT == 32
    if (dk <= db) best = k; /* planted: ties to the larger magnitude */
#else
    if (dk < db || (dk == db && (k & 1) == 0)) best = k; /* ties to the even code */
#endif
  }
  return s | best;
}

void situ_oracle_e2m1_encode_n(const double *x, int64_t n, uint8_t *codes) {
  for (int64_t i = 0; i < n; ++i) codes[i] = (uint8_t)situ_oracle_e2m1_encode(x[i]);
}

double situ_oracle_e2m1_decode(int code) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  const double v = mag[code & 7];
  return (code & 8) ? -v : v;
}

/* Per-tensor encode scale S_enc of a tensor with largest magnitude amax. */
double situ_oracle_nvfp4_tensor_scale(double amax) {
  if (!(amax > 0.0) || isinf(amax)) return 1.0;
#if SITU_ORACLE_MUTANT == 34
  return 1.0; /* planted: no tensor scale */
#elif SITU_ORACLE_MUTANT == 35
  return E4M3_MAX / amax; /* planted: the E2M1 range left out */
#elif SITU_ORACLE_MUTANT == 36
  return amax / (E4M3_MAX * E2M1_MAX); /* planted: inverted */
#else
  return E4M3_MAX * E2M1_MAX / amax;
#endif
}

/* NVFP4 quantisation of v[rows, cols] (row pitch v_stride): codes[rows, cols]
 * (one 4-bit code per byte here, unpacked), block scale codes [rows, cols /
 * 16] (E4M3), with the tensor scale s_enc given.  Returns 0, or -1 when cols
 * is not a multiple of 16. */
int situ_oracle_nvfp4_quantize(const double *v, int64_t rows, int64_t cols, int64_t v_stride, double s_enc,
                               uint8_t *codes, uint8_t *scales) {
  if (cols % 16 != 0 || rows < 0) return -1;
  const int64_t nblk = cols / 16;
  for (int64_t r = 0; r < rows; ++r) {
    for (int64_t b = 0; b < nblk; ++b) {
      const double *blk = v + r * v_stride + b * 16;
      double amax = 0.0;
      int special = 0;
      for (int i = 0; i < 16; ++i) {
        if (isnan(blk[i]) || isinf(blk[i])) special = 1;
        else if (fabs(blk[i]) > amax) amax = fabs(blk[i]);
      }
      int sc;
      if (special) {
        sc = 0x7F;
      } else {
#if SITU_ORACLE_MUTANT == 33
        sc = situ_oracle_e4m3_encode(amax * s_enc / 4.0); /* planted: divided by 4 instead of 6 */
#else
        sc = situ_oracle_e4m3_encode(amax * s_enc / E2M1_MAX);
#endif
      }
      scales[r * nblk + b] = (uint8_t)sc;
      const double sb = special ? 0.0 : situ_oracle_e4m3_decode(sc);
      for (int i = 0; i < 16; ++i)
        codes[r * cols + b * 16 + i] = (uint8_t)((sb > 0.0) ? situ_oracle_e2m1_encode(blk[i] * s_enc / sb) : 0);
    }
  }
  return 0;
}
