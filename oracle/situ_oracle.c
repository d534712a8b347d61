/*
 * situ_oracle.c -- plain fp64 CPU oracle for the routing-weighted SiTU-GLU
 * forward and its analytic backward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  The CUDA path in
 * ffn_gated_activation_b200/ shares no code, header or constant with it.
 *
 * What it computes (each function below names the passage it follows):
 *
 *   Megatron-LM PR #6673 "[Dev] Add SiTU-GLU through Transformer Engine",
 *   section "Activation" (Kimi K3 report, Equation 12):
 *       T_g = beta1 * tanh(G / beta1) * sigmoid(G)
 *       T_u = beta2 * tanh(U / beta2)
 *       Y   = T_g * T_u
 *   NeMo AutoModel API, nemo_automodel.components.models.kimi_k3.situ,
 *   `_situ_fwd_core` (Returns): the routed form situ(g) * up(u0) * w, with
 *   `linear_beta` optional (None => the up branch is the identity), and
 *   `_WeightedSiTUFunction.forward` (gate in the first half of the last
 *   axis of gate_up, up in the second).
 *   `_situ_bwd_core` / `_WeightedSiTUFunction.backward`: analytic gradients
 *   d_g, d_u of that chain, and the routing-weight reduction `red`, taken
 *   here as the per-row sum over the intermediate axis of go * T_g * T_u
 *   (d Y / d w = T_g * T_u for a row-aligned weight).
 *
 * Every value is evaluated in IEEE double from inputs converted exactly
 * (bf16 and fp32 are subsets of double).  No blocking, fusion or
 * reordering: one element at a time, in the pages' notation.
 *
 * Parity pins: see tests/test_oracle_pins.py (closed forms, invariants,
 * the SwiGLU limit against a library SiLU, finite differences, float64
 * autograd, 50-digit values, brute-force sums, and planted mutants built
 * from this file with -DSITU_ORACLE_MUTANT=n that the pins must reject).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifndef SITU_ORACLE_MUTANT
#define SITU_ORACLE_MUTANT 0 /* 0 = the oracle; n > 0 = a planted mistake */
#endif

#define ORACLE_DTYPE_BF16 0
#define ORACLE_DTYPE_F32 1
#define ORACLE_RW_ROW 0    /* w[row * stride]              ([T, 1])   */
#define ORACLE_RW_SCALAR 1 /* w[0] on every row            (one value) */
#define ORACLE_RW_COL 2    /* w[col * stride] on every row ([I])       */
#define ORACLE_RW_FULL 3   /* w[row * stride + col]        ([T, I])    */

/* ---- exact input conversion ------------------------------------------ */

static double load_value(const void *base, int dtype, int64_t index) {
  if (dtype == ORACLE_DTYPE_BF16) {
    /* bf16 is the top 16 bits of an fp32 word: widening is exact. */
    uint16_t half = ((const uint16_t *)base)[index];
    uint32_t bits = (uint32_t)half << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float *)base)[index];
}

/* ---- the scalar building blocks ---------------------------------------- */

/* Logistic sigmoid 1 / (1 + exp(-x)), evaluated on the side whose exp()
 * argument is non-positive so that neither branch overflows. */
static double sigmoid(double x) {
  if (x >= 0.0) return 1.0 / (1.0 + exp(-x));
  double e = exp(x);
  return e / (1.0 + e);
}

/* sech^2(a) = 1 - tanh^2(a), written as 4E / (1 + E)^2 with E = exp(-2|a|):
 * equal in exact arithmetic, and it keeps its value (e.g. 3.7e-13 at
 * a = 15) where 1 - tanh(a)^2 would round to zero. */
static double sech2(double a) {
#if SITU_ORACLE_MUTANT == 11
  double e = exp(-fabs(a)); /* planted: wrong factor in the exponent */
#else
  double e = exp(-2.0 * fabs(a));
#endif
  return 4.0 * e / ((1.0 + e) * (1.0 + e));
}

/* Gate branch T_g(g) = beta * tanh(g / beta) * sigmoid(g) and its
 * derivative (Megatron-LM PR #6673, "Activation", first line; NeMo
 * `_situ_bwd_core` for the analytic gradient).  Product rule:
 *   d/dg [beta tanh(g/beta)] = sech^2(g/beta)
 *   d/dg sigmoid(g)          = sigmoid(g) (1 - sigmoid(g))
 *   T_g'(g) = sech^2(g/beta) sigmoid(g) + beta tanh(g/beta) sigmoid(g) (1 - sigmoid(g))
 * 1 - sigmoid(g) is evaluated as sigmoid(-g) (exact identity, no cancellation).
 * Also returns the uncancelled magnitude of T_g' (sum of the absolute
 * values of its two terms), used to scale the tolerance where they cancel. */
void situ_oracle_gate(double g, double beta, double *t_g, double *dt_g, double *dt_g_mag) {
  double a = g / beta;
  double th = tanh(a);
#if SITU_ORACLE_MUTANT == 4
  double s = sigmoid(-g); /* planted: sigmoid of the wrong sign */
#else
  double s = sigmoid(g);
#endif
  double one_minus_s = sigmoid(-g);
  double term1 = sech2(a) * s;
#if SITU_ORACLE_MUTANT == 1
  double term2 = 0.0; /* planted: dropped product-rule term */
#elif SITU_ORACLE_MUTANT == 2
  double term2 = -beta * th * s * one_minus_s; /* planted: wrong sign */
#else
  double term2 = beta * th * s * one_minus_s;
#endif
  if (t_g) *t_g = beta * th * s;
  if (dt_g) *dt_g = term1 + term2;
  if (dt_g_mag) *dt_g_mag = fabs(term1) + fabs(term2);
}

/* Up branch T_u(u) = beta_L * tanh(u / beta_L), or T_u = u when no
 * linear beta is given (Megatron-LM PR #6673, "Activation", second line;
 * NeMo `_situ_fwd_core`: "Optional bounded-linear beta applied to the up
 * branch").  Derivative sech^2(u / beta_L), or 1. */
void situ_oracle_up(double u, int has_linear_beta, double linear_beta, double *t_u, double *dt_u) {
#if SITU_ORACLE_MUTANT == 10
  has_linear_beta = 0; /* planted: the optional clamp is ignored */
#endif
  if (!has_linear_beta) {
    if (t_u) *t_u = u;
    if (dt_u) *dt_u = 1.0;
    return;
  }
#if SITU_ORACLE_MUTANT == 3
  double a = u * linear_beta; /* planted: transposed operand of the divide */
#else
  double a = u / linear_beta;
#endif
  if (t_u) *t_u = linear_beta * tanh(a);
  if (dt_u) *dt_u = sech2(a);
}

/* ---- row helpers -------------------------------------------------------- */

static int64_t row_index(const int64_t *rows, int64_t k) { return rows ? rows[k] : k; }

/* Routing weight of element (row, col): the weight tensor broadcast against
 * the [T, I] output (NeMo `_WeightedSiTUFunction.forward`, parameter
 * routing_weights: row-aligned [..., 1] or broadcastable). */
static double routing_weight(int rw_dtype, const void *rw, int rw_mode, int64_t rw_stride, int64_t row,
                             int64_t col) {
  switch (rw_mode) {
    case ORACLE_RW_SCALAR: return load_value(rw, rw_dtype, 0);
#if SITU_ORACLE_MUTANT == 13
    case ORACLE_RW_COL: return load_value(rw, rw_dtype, row * rw_stride); /* planted: row for column */
#else
    case ORACLE_RW_COL: return load_value(rw, rw_dtype, col * rw_stride);
#endif
    case ORACLE_RW_FULL: return load_value(rw, rw_dtype, row * rw_stride + col);
    default: return load_value(rw, rw_dtype, row * rw_stride);
  }
}

/* Gate is the first half of a gate_up row, up the second half
 * (NeMo `_WeightedSiTUFunction.forward`, parameter gate_up). */
static void load_pair(int dtype, const void *gate_up, int64_t gu_stride, int64_t inter,
                      int64_t row, int64_t i, double *g, double *u) {
#if SITU_ORACLE_MUTANT == 8
  *u = load_value(gate_up, dtype, row * gu_stride + i); /* planted: halves swapped */
  *g = load_value(gate_up, dtype, row * gu_stride + inter + i);
#elif SITU_ORACLE_MUTANT == 12
  *g = load_value(gate_up, dtype, row * 2 * inter + i); /* planted: row stride ignored */
  *u = load_value(gate_up, dtype, row * 2 * inter + inter + i);
  (void)gu_stride;
#else
  *g = load_value(gate_up, dtype, row * gu_stride + i);
  *u = load_value(gate_up, dtype, row * gu_stride + inter + i);
#endif
}

/* Neumaier's compensated summation (Neumaier 1974): running sum plus a
 * correction term that collects the low-order bits each add loses. */
typedef struct {
  double sum, comp;
} neumaier_t;

static void neumaier_add(neumaier_t *acc, double x) {
  double t = acc->sum + x;
  if (fabs(acc->sum) >= fabs(x))
    acc->comp += (acc->sum - t) + x;
  else
    acc->comp += (x - t) + acc->sum;
  acc->sum = t;
}

static double neumaier_value(const neumaier_t *acc) { return acc->sum + acc->comp; }

/* ---- forward ------------------------------------------------------------ */

/* Y[k, i] = T_g(G[r, i]) * T_u(U[r, i]) * w[r] for each selected row r =
 * rows[k] (rows == NULL selects rows 0..nrows-1).  Output y is packed
 * [nrows, inter].  NeMo `_situ_fwd_core` (Returns: situ(g) * up(u0) * w).
 * Returns 0, or -1 on a bad argument. */
int situ_oracle_fwd(int dtype, const void *gate_up, int64_t gu_stride, int64_t inter,
                    const int64_t *rows, int64_t nrows,
                    int rw_dtype, const void *rw, int rw_mode, int64_t rw_stride,
                    double beta, int has_linear_beta, double linear_beta, double *y) {
  if (!gate_up || !rw || !y || inter <= 0 || nrows < 0 || gu_stride < 2 * inter) return -1;
  for (int64_t k = 0; k < nrows; ++k) {
    int64_t r = row_index(rows, k);
    for (int64_t i = 0; i < inter; ++i) {
      double g, u, t_g, t_u;
      double w = routing_weight(rw_dtype, rw, rw_mode, rw_stride, r, i);
      load_pair(dtype, gate_up, gu_stride, inter, r, i, &g, &u);
      situ_oracle_gate(g, beta, &t_g, NULL, NULL);
      situ_oracle_up(u, has_linear_beta, linear_beta, &t_u, NULL);
#if SITU_ORACLE_MUTANT == 5
      y[k * inter + i] = t_g * t_u; /* planted: routing weight dropped */
#else
      y[k * inter + i] = t_g * t_u * w;
#endif
    }
  }
  return 0;
}

/* ---- backward ----------------------------------------------------------- */

/* Analytic gradients of Y = T_g(G) T_u(U) w for each selected row, given
 * the upstream gradient go (NeMo `_situ_bwd_core`, `_WeightedSiTUFunction
 * .backward`):
 *   dG[k, i] = go * w * T_u * T_g'
 *   dU[k, i] = go * w * T_g * T_u'
 *   dw[k]    = sum_i go * T_g * T_u          (Neumaier-compensated)
 * Optional error scales for the tolerance (any of them may be NULL):
 *   cg[k, i] = |go * w * T_u| * (|term1| + |term2| of T_g')
 *   sw[k]    = sum_i |go * T_g * T_u|
 * Outputs dg, du, cg are packed [nrows, inter]; dw, sw are [nrows].
 * Returns 0, or -1 on a bad argument. */
int situ_oracle_bwd(int dtype, const void *gate_up, int64_t gu_stride, int64_t inter,
                    const int64_t *rows, int64_t nrows,
                    int rw_dtype, const void *rw, int rw_mode, int64_t rw_stride,
                    double beta, int has_linear_beta, double linear_beta,
                    const void *grad_out, int64_t go_stride,
                    double *dg, double *du, double *dw, double *cg, double *sw) {
  if (!gate_up || !rw || !grad_out || inter <= 0 || nrows < 0 || gu_stride < 2 * inter ||
      go_stride < inter)
    return -1;
  for (int64_t k = 0; k < nrows; ++k) {
    int64_t r = row_index(rows, k);
    neumaier_t red = {0.0, 0.0};
    neumaier_t mag = {0.0, 0.0};
    for (int64_t i = 0; i < inter; ++i) {
      double g, u, t_g, dt_g, dt_g_mag, t_u, dt_u;
      double w = routing_weight(rw_dtype, rw, rw_mode, rw_stride, r, i);
      load_pair(dtype, gate_up, gu_stride, inter, r, i, &g, &u);
      double go = load_value(grad_out, dtype, r * go_stride + i);
      situ_oracle_gate(g, beta, &t_g, &dt_g, &dt_g_mag);
      situ_oracle_up(u, has_linear_beta, linear_beta, &t_u, &dt_u);
#if SITU_ORACLE_MUTANT == 6
      double d_g = go * w * t_g * dt_g; /* planted: T_g where T_u belongs */
#else
      double d_g = go * w * t_u * dt_g;
#endif
#if SITU_ORACLE_MUTANT == 7
      double d_u = go * w * t_u * dt_u; /* planted: T_u where T_g belongs */
#else
      double d_u = go * w * t_g * dt_u;
#endif
#if SITU_ORACLE_MUTANT == 9
      double term = t_g * t_u; /* planted: upstream gradient dropped */
#else
      double term = go * t_g * t_u;
#endif
      if (dg) dg[k * inter + i] = d_g;
      if (du) du[k * inter + i] = d_u;
      if (cg) cg[k * inter + i] = fabs(go * w * t_u) * dt_g_mag;
      neumaier_add(&red, term);
      neumaier_add(&mag, fabs(term));
    }
    if (dw) dw[k] = neumaier_value(&red);
    if (sw) sw[k] = neumaier_value(&mag);
  }
  return 0;
}

/* Gradient of a per-column routing weight w[i] (shape [I], broadcast over
 * the rows): d w[i] = sum over rows r of go * T_g * T_u, for every column,
 * each in one compensated sum; mag[i] receives the sum of absolute terms
 * (may be NULL).  For a full [T, I] weight the gradient is the term
 * go * T_g * T_u itself, element by element: situ_oracle_bwd's per-row sums
 * are those terms summed over each row. */
int situ_oracle_dw_columns(int dtype, const void *gate_up, int64_t gu_stride, int64_t inter, int64_t tokens,
                           double beta, int has_linear_beta, double linear_beta, const void *grad_out,
                           int64_t go_stride, double *colsum, double *colmag) {
  if (!gate_up || !grad_out || !colsum || inter <= 0 || tokens < 0 || gu_stride < 2 * inter || go_stride < inter)
    return -1;
  for (int64_t i = 0; i < inter; ++i) {
    neumaier_t red = {0.0, 0.0};
    neumaier_t mag = {0.0, 0.0};
    for (int64_t r = 0; r < tokens; ++r) {
      double g, u, t_g, t_u;
      load_pair(dtype, gate_up, gu_stride, inter, r, i, &g, &u);
      double go = load_value(grad_out, dtype, r * go_stride + i);
      situ_oracle_gate(g, beta, &t_g, NULL, NULL);
      situ_oracle_up(u, has_linear_beta, linear_beta, &t_u, NULL);
      neumaier_add(&red, go * t_g * t_u);
      neumaier_add(&mag, fabs(go * t_g * t_u));
    }
    colsum[i] = neumaier_value(&red);
    if (colmag) colmag[i] = neumaier_value(&mag);
  }
  return 0;
}

/* The weight-gradient terms go * T_g * T_u of each selected row, packed
 * [nrows, inter]: the gradient of a full [T, I] routing weight. */
int situ_oracle_dw_terms(int dtype, const void *gate_up, int64_t gu_stride, int64_t inter, const int64_t *rows,
                         int64_t nrows, double beta, int has_linear_beta, double linear_beta, const void *grad_out,
                         int64_t go_stride, double *terms) {
  if (!gate_up || !grad_out || !terms || inter <= 0 || nrows < 0 || gu_stride < 2 * inter || go_stride < inter)
    return -1;
  for (int64_t k = 0; k < nrows; ++k) {
    int64_t r = row_index(rows, k);
    for (int64_t i = 0; i < inter; ++i) {
      double g, u, t_g, t_u;
      load_pair(dtype, gate_up, gu_stride, inter, r, i, &g, &u);
      double go = load_value(grad_out, dtype, r * go_stride + i);
      situ_oracle_gate(g, beta, &t_g, NULL, NULL);
      situ_oracle_up(u, has_linear_beta, linear_beta, &t_u, NULL);
      terms[k * inter + i] = go * t_g * t_u;
    }
  }
  return 0;
}

/* Gradient of a single routing weight broadcast to every row: autograd's
 * sum-to-shape of d(Y)/d(w) * go over all rows and columns, i.e. the sum of
 * go * T_g * T_u over the whole [tokens, inter] block, in one compensated
 * sum.  *total_mag receives the sum of absolute terms (may be NULL). */
int situ_oracle_dw_scalar(int dtype, const void *gate_up, int64_t gu_stride, int64_t inter,
                          int64_t tokens, double beta, int has_linear_beta, double linear_beta,
                          const void *grad_out, int64_t go_stride, double *total, double *total_mag) {
  if (!gate_up || !grad_out || !total || inter <= 0 || tokens < 0 || gu_stride < 2 * inter ||
      go_stride < inter)
    return -1;
  neumaier_t red = {0.0, 0.0};
  neumaier_t mag = {0.0, 0.0};
  for (int64_t r = 0; r < tokens; ++r) {
    for (int64_t i = 0; i < inter; ++i) {
      double g, u, t_g, t_u;
      load_pair(dtype, gate_up, gu_stride, inter, r, i, &g, &u);
      double go = load_value(grad_out, dtype, r * go_stride + i);
      situ_oracle_gate(g, beta, &t_g, NULL, NULL);
      situ_oracle_up(u, has_linear_beta, linear_beta, &t_u, NULL);
      neumaier_add(&red, go * t_g * t_u);
      neumaier_add(&mag, fabs(go * t_g * t_u));
    }
  }
  *total = neumaier_value(&red);
  if (total_mag) *total_mag = neumaier_value(&mag);
  return 0;
}

/* Array forms of the two branch functions, for the pin tests. */
void situ_oracle_gate_n(int64_t n, const double *g, double beta, double *t_g, double *dt_g, double *dt_g_mag) {
  for (int64_t k = 0; k < n; ++k)
    situ_oracle_gate(g[k], beta, t_g ? t_g + k : NULL, dt_g ? dt_g + k : NULL, dt_g_mag ? dt_g_mag + k : NULL);
}

void situ_oracle_up_n(int64_t n, const double *u, int has_linear_beta, double linear_beta, double *t_u, double *dt_u) {
  for (int64_t k = 0; k < n; ++k)
    situ_oracle_up(u[k], has_linear_beta, linear_beta, t_u ? t_u + k : NULL, dt_u ? dt_u + k : NULL);
}

/* Identifies which build this is: 0 for the oracle, n for planted mutant n. */
int situ_oracle_mutant_id(void) { return SITU_ORACLE_MUTANT; }
