/*
 * fc2_oracle.c -- plain fp64 CPU oracle for the FC2 data-gradient GEMM
 * followed by the SiTU-GLU backward (the "dSiTU in the dgrad GEMM" form).
 *
 * TEST INFRASTRUCTURE ONLY, like situ_oracle.c (built into the same library).
 * The CUDA path shares no code, header or constant with it.
 *
 * Megatron-LM PR #6673, "Test results": the fused grouped-MLP path was
 * validated forward and backward with a dSiTU correction in the cuDNN
 * frontend.  In the backward of Y -> FC2, the activation's upstream gradient
 * is FC2's data gradient, so the fused form computes, for a token row r of
 * expert e (rows [off[e], off[e+1])) and FC2 weight W2_e [H, I] (passed
 * transposed, W2T_e [I, H]):
 *     dY[r, i]  = sum_h dOut[r, h] W2_e[h, i] = sum_h dOut[r, h] W2T_e[i, h]
 *     dG[r, i]  = dY w[r] T_u(U) T_g'(G)           (NeMo `_situ_bwd_core`)
 *     dU[r, i]  = dY w[r] T_g(G) T_u'(U)
 *     dw[r]     = sum_i dY T_g(G) T_u(U)
 * with G, U the halves of the saved gate_up row and T_g, T_u and their
 * derivatives from situ_oracle.c.  Plain fp64 sums in index order.
 *
 * Pinned by tests/test_oracle_pins.py (fsum dot products with 50-digit
 * element derivatives, exact agreement with the pinned activation backward
 * on bf16-exact dY, per-expert calls; planted mutants 29-31).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifndef SITU_ORACLE_MUTANT
#define SITU_ORACLE_MUTANT 0
#endif

void situ_oracle_gate(double g, double beta, double *t_g, double *dt_g, double *dt_g_mag);
void situ_oracle_up(double u, int has_linear_beta, double linear_beta, double *t_u, double *dt_u);

static double fc2_bf16(const uint16_t *base, int64_t index) {
  uint32_t bits = (uint32_t)base[index] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

static int64_t fc2_expert_of(const int64_t *off, int64_t experts, int64_t r) {
  for (int64_t e = 0; e < experts; ++e)
    if (off[e] <= r && r < off[e + 1]) return e;
  return -1;
}

/*
 * For the selected token rows (rows == NULL: 0..nrows-1), packed by row:
 *   dgu   [nrows, 2 inter]  dG then dU
 *   dw    [nrows]
 *   dy    [nrows, inter] or NULL: the unrounded FC2 data gradient
 *   err   [nrows, 2 inter] or NULL: error scales of dG, dU -- the
 *         accumulation |dY/d(dY)| sum_h |dOut W2T| plus, for dG, the
 *         uncancelled magnitude |dY w T_u| (|t1| + |t2|) of T_g'
 *   dw_err [nrows] or NULL: sum_i |dY T_g T_u| + sum_i |T_g T_u| sum_h |dOut W2T|
 * Inputs: dout bf16 [T, >= hidden] (pitch ldo); w2t bf16 [experts * inter,
 * >= hidden] (pitch ldw; expert e's rows e*inter ..); gate_up bf16 [T, >=
 * 2 inter] (pitch ldg); rw fp32 [T] or NULL (w = 1).  A row outside every
 * expert gets NaN.  Returns 0, or -1 on a bad argument.
 */
int situ_oracle_fc2_dgrad(const uint16_t *dout, int64_t ldo, int64_t hidden, const uint16_t *w2t, int64_t ldw,
                          int64_t inter, const int64_t *offsets, int64_t experts, const uint16_t *gate_up,
                          int64_t ldg, const float *rw, double beta, int has_linear_beta, double linear_beta,
                          const int64_t *rows, int64_t nrows, double *dgu, double *dw, double *dy, double *err,
                          double *dw_err) {
  if (!dout || !w2t || !offsets || !gate_up || !dgu || !dw || hidden <= 0 || inter <= 0 || experts <= 0 ||
      nrows < 0 || ldo < hidden || ldw < hidden || ldg < 2 * inter)
    return -1;
  for (int64_t j = 0; j < nrows; ++j) {
    const int64_t r = rows ? rows[j] : j;
    const int64_t e = fc2_expert_of(offsets, experts, r);
    const double w = rw ? (double)rw[r] : 1.0;
    double acc = 0.0, acc_mag = 0.0, acc_err = 0.0;
    for (int64_t i = 0; i < inter; ++i) {
      if (e < 0) {
        dgu[j * 2 * inter + i] = dgu[j * 2 * inter + inter + i] = NAN;
        if (dy) dy[j * inter + i] = NAN;
        if (err) err[j * 2 * inter + i] = err[j * 2 * inter + inter + i] = NAN;
        continue;
      }
      const uint16_t *wrow = w2t + (e * inter + i) * ldw;
      double d = 0.0, s = 0.0;
      for (int64_t h = 0; h < hidden; ++h) {
#if SITU_ORACLE_MUTANT == 29
        const double p = fc2_bf16(dout, r * ldo + h) * fc2_bf16(w2t, (e * inter + h % inter) * ldw + i); /* planted: W2 read untransposed */
#else
        const double p = fc2_bf16(dout, r * ldo + h) * fc2_bf16(wrow, h);
#endif
        d += p;
        s += fabs(p);
      }
      const double g = fc2_bf16(gate_up, r * ldg + i), u = fc2_bf16(gate_up, r * ldg + inter + i);
      double t_g, dt_g, dt_g_mag, t_u, dt_u;
      situ_oracle_gate(g, beta, &t_g, &dt_g, &dt_g_mag);
      situ_oracle_up(u, has_linear_beta, linear_beta, &t_u, &dt_u);
#if SITU_ORACLE_MUTANT == 30
      dgu[j * 2 * inter + i] = d * t_u * dt_g; /* planted: routing weight dropped from dG */
#else
      dgu[j * 2 * inter + i] = d * w * t_u * dt_g;
#endif
      dgu[j * 2 * inter + inter + i] = d * w * t_g * dt_u;
      if (dy) dy[j * inter + i] = d;
      if (err) {
        err[j * 2 * inter + i] = fabs(w * t_u * dt_g) * s + fabs(d * w * t_u) * dt_g_mag;
        err[j * 2 * inter + inter + i] = fabs(w * t_g * dt_u) * s;
      }
#if SITU_ORACLE_MUTANT == 31
      acc += t_g * t_u; /* planted: the upstream gradient dropped from dw */
#else
      acc += d * t_g * t_u;
#endif
      acc_mag += fabs(d * t_g * t_u);
      acc_err += fabs(t_g * t_u) * s;
    }
    dw[j] = e < 0 ? NAN : acc;
    if (dw_err) dw_err[j] = e < 0 ? NAN : acc_mag + acc_err;
  }
  return 0;
}
