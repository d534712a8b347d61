/*
 * fc1_oracle.c -- plain fp64 CPU oracle for FC1 followed by SiTU-GLU, the
 * fused grouped-GEMM form.
 *
 * TEST INFRASTRUCTURE ONLY, like situ_oracle.c (built into the same library).
 * The CUDA path shares no code, header or constant with it.
 *
 * Megatron-LM PR #6673, "Design": with a SiTU-capable cuDNN frontend, FC1's
 * grouped GEMM and the SiTU-GLU activation run as one fused grouped-MLP
 * operation; without it Transformer Engine runs GroupedLinear ->
 * ScaledSiTUGLU -> GroupedLinear.  Either way the activation's input is FC1's
 * output, so what the fused operation computes is the composition, for a
 * token row r routed to expert e (rows [off[e], off[e+1]) of X):
 *     gate_up[r, n] = sum_k X[r, k] W1_e[n, k]     n < 2I (gate rows, then up rows)
 *     Y[r, i]       = T_g(gate_up[r, i]) T_u(gate_up[r, I + i]) w[r]
 * with T_g, T_u the element functions of situ_oracle.c (Megatron-LM PR #6673,
 * "Activation"; NeMo `_situ_fwd_core`: gate first, up second, routing weight
 * last).  Each dot product is a plain fp64 sum in k order (no blocking), and
 * gate_up is never rounded to a storage type.
 *
 * Pinned by tests/test_oracle_pins.py: Python fsum dot products with mpmath
 * element values on a tiny grouped case, exact agreement with the pinned
 * activation oracle when every gate_up value is a bf16 number, per-expert
 * calls against the grouped call, and planted mutants 20-23.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifndef SITU_ORACLE_MUTANT
#define SITU_ORACLE_MUTANT 0
#endif

void situ_oracle_gate(double g, double beta, double *t_g, double *dt_g, double *dt_g_mag);
void situ_oracle_up(double u, int has_linear_beta, double linear_beta, double *t_u, double *dt_u);

static double bf16_value(const uint16_t *base, int64_t index) {
  uint32_t bits = (uint32_t)base[index] << 16; /* bf16 is the top half of an fp32 word */
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Expert owning token row r: the e with off[e] <= r < off[e+1]; -1 if none. */
static int64_t expert_of(const int64_t *off, int64_t experts, int64_t r) {
  for (int64_t e = 0; e < experts; ++e) {
#if SITU_ORACLE_MUTANT == 23
    if (off[e] <= r && r <= off[e + 1]) return e; /* planted: a boundary row goes to the earlier expert */
#else
    if (off[e] <= r && r < off[e + 1]) return e;
#endif
  }
  return -1;
}

/* sum_k x[k] w[k] (and sum_k |x[k] w[k]|) over the hidden axis, k in order. */
static void dot(const uint16_t *x, const uint16_t *w, int64_t hidden, double *s, double *s_abs) {
  double acc = 0.0, mag = 0.0;
#if SITU_ORACLE_MUTANT == 22
  hidden -= 1; /* planted: the last product dropped */
#endif
  for (int64_t k = 0; k < hidden; ++k) {
    const double p = bf16_value(x, k) * bf16_value(w, k);
    acc += p;
    mag += fabs(p);
  }
  *s = acc;
  *s_abs = mag;
}

/*
 * Y for the selected token rows (rows == NULL: rows 0..nrows-1).
 *   x        bf16 [T, >= hidden], row pitch ldx elements
 *   w1       bf16 [experts * 2I, >= hidden], row pitch ldw: expert e's gate
 *            rows are e*2I .. e*2I+I-1, its up rows e*2I+I .. e*2I+2I-1
 *   offsets  [experts + 1], non-decreasing, rows of expert e = [off[e], off[e+1])
 *   rw       fp32 [T] per-row routing weights, or NULL for w = 1
 * Outputs (packed by selected row):
 *   y        [nrows, inter]
 *   err      [nrows, inter] or NULL: |dY/dG| sum_k |x w_g| + |dY/dU| sum_k |x w_u|,
 *            the scale of the error an accumulation of the products can make
 *   gate_up  [nrows, 2 inter] or NULL: the unrounded FC1 output
 * A row that belongs to no expert gets NaN.  Returns 0, or -1 on a bad argument.
 */
int situ_oracle_fc1_fwd(const uint16_t *x, int64_t ldx, int64_t hidden, const uint16_t *w1, int64_t ldw,
                        int64_t inter, const int64_t *offsets, int64_t experts, const int64_t *rows, int64_t nrows,
                        const float *rw, double beta, int has_linear_beta, double linear_beta, double *y, double *err,
                        double *gate_up) {
  if (!x || !w1 || !offsets || !y || hidden <= 0 || inter <= 0 || experts <= 0 || nrows < 0 || ldx < hidden ||
      ldw < hidden)
    return -1;
  for (int64_t j = 0; j < nrows; ++j) {
    const int64_t r = rows ? rows[j] : j;
    int64_t e = expert_of(offsets, experts, r);
    for (int64_t i = 0; i < inter; ++i) {
      if (e < 0) {
        y[j * inter + i] = NAN;
        if (err) err[j * inter + i] = NAN;
        if (gate_up) gate_up[j * 2 * inter + i] = gate_up[j * 2 * inter + inter + i] = NAN;
        continue;
      }
#if SITU_ORACLE_MUTANT == 20
      const int64_t we = (e + 1) % experts; /* planted: the next expert's weights */
#else
      const int64_t we = e;
#endif
      const uint16_t *wg = w1 + (we * 2 * inter + i) * ldw;
#if SITU_ORACLE_MUTANT == 21
      const uint16_t *wu = w1 + (we * 2 * inter + i) * ldw; /* planted: gate rows used for up */
#else
      const uint16_t *wu = w1 + (we * 2 * inter + inter + i) * ldw;
#endif
      double g, g_abs, u, u_abs;
      dot(x + r * ldx, wg, hidden, &g, &g_abs);
      dot(x + r * ldx, wu, hidden, &u, &u_abs);
      double t_g, dt_g, dt_g_mag, t_u, dt_u;
      situ_oracle_gate(g, beta, &t_g, &dt_g, &dt_g_mag);
      situ_oracle_up(u, has_linear_beta, linear_beta, &t_u, &dt_u);
      const double w = rw ? (double)rw[r] : 1.0;
      y[j * inter + i] = t_g * t_u * w;
      if (err) err[j * inter + i] = fabs(t_u * w) * dt_g_mag * g_abs + fabs(t_g * w * dt_u) * u_abs;
      if (gate_up) {
        gate_up[j * 2 * inter + i] = g;
        gate_up[j * 2 * inter + inter + i] = u;
      }
    }
  }
  return 0;
}
