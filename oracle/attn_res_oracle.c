/*
 * attn_res_oracle.c -- plain fp64 CPU oracle for the attention-residual
 * mixing core.
 *
 * TEST INFRASTRUCTURE ONLY, like situ_oracle.c (built into the same library).
 * The CUDA path shares no code, header or constant with it.
 *
 * NeMo AutoModel API, kimi_k3.situ, `_attn_res_core(values, norm_weight,
 * proj_weight, variance_epsilon, out_dtype)`: the fp32 attention-residual
 * mixing chain over values [tokens, blocks + 1, hidden] (the block residuals
 * with the current prefix sum appended along axis 1, as `_apply_attn_res`
 * stacks them), an RMSNorm weight [hidden], a squeezed projection weight
 * [hidden], and the RMSNorm epsilon; the weighted combine is a multiply and
 * sum of prob [tokens, 1, blocks + 1] with the values.  Read plainly, for
 * token t and source b:
 *     k[t, b, :] = RMSNorm(values[t, b, :]) = values[t, b, :] / sqrt(mean_h values^2 + eps) * norm_weight
 *     logit[t, b] = sum_h k[t, b, h] proj_weight[h]      (the projection to one score)
 *     prob[t, :]  = softmax over b of logit[t, :]
 *     out[t, h]   = sum_b prob[t, b] values[t, b, h]        (the raw values)
 * The RMSNorm definition is not on the pages; this is its standard form.
 * Sources may come from two arrays: `blocks` stored sums and, optionally, the
 * current prefix sum as the last source (what `_apply_attn_res` passes).
 *
 * Pinned by tests/test_oracle_pins.py (torch's rms_norm and softmax in
 * float64, invariants, and planted mutants 24-28).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#ifndef SITU_ORACLE_MUTANT
#define SITU_ORACLE_MUTANT 0
#endif

#define AR_DTYPE_BF16 0
#define AR_DTYPE_F32 1
#define AR_MAX_SOURCES 64

static double ar_value(const void *base, int dtype, int64_t index) {
  if (dtype == AR_DTYPE_BF16) {
    uint32_t bits = (uint32_t)((const uint16_t *)base)[index] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
  }
  return (double)((const float *)base)[index];
}

/* Element h of source b of token t. */
static double source_value(const void *blocks, int64_t nblocks, int64_t block_row_stride, int64_t block_stride,
                           const void *prefix, int64_t prefix_row_stride, int dtype, int64_t t, int64_t b,
                           int64_t h) {
  if (b < nblocks) return ar_value(blocks, dtype, t * block_row_stride + b * block_stride + h);
  return ar_value(prefix, dtype, t * prefix_row_stride + h);
}

/*
 * out[k, h] for the selected tokens t = rows[k] (rows == NULL: 0..nrows-1),
 * packed [nrows, hidden]; mag[k, h] (or NULL) = sum_b prob[b] |values[t, b, h]|,
 * the scale of the combine's rounding error; prob[k, b] (or NULL) packed
 * [nrows, sources].  Returns 0, or -1 on a bad argument.
 */
int situ_oracle_attn_res(const void *blocks, int64_t nblocks, int64_t block_row_stride, int64_t block_stride,
                         const void *prefix, int64_t prefix_row_stride, int dtype, int64_t hidden,
                         const void *norm_weight, int norm_dtype, const void *proj_weight, int proj_dtype, double eps,
                         const int64_t *rows, int64_t nrows, double *out, double *mag, double *prob) {
  const int64_t sources = nblocks + (prefix ? 1 : 0);
  if (sources < 1 || sources > AR_MAX_SOURCES || hidden <= 0 || nrows < 0 || !out || !norm_weight ||
      !proj_weight || (nblocks > 0 && !blocks) || eps < 0.0)
    return -1;
  for (int64_t k = 0; k < nrows; ++k) {
    const int64_t t = rows ? rows[k] : k;
    double logit[AR_MAX_SOURCES], p[AR_MAX_SOURCES];
    for (int64_t b = 0; b < sources; ++b) {
      double ss = 0.0;
      for (int64_t h = 0; h < hidden; ++h) {
        const double x = source_value(blocks, nblocks, block_row_stride, block_stride, prefix, prefix_row_stride,
                                      dtype, t, b, h);
        ss += x * x;
      }
#if SITU_ORACLE_MUTANT == 24
      const double inv = 1.0 / sqrt(ss + eps); /* planted: sum instead of mean */
#elif SITU_ORACLE_MUTANT == 25
      const double inv = 1.0 / sqrt(ss / (double)hidden); /* planted: epsilon dropped */
#else
      const double inv = 1.0 / sqrt(ss / (double)hidden + eps);
#endif
      double score = 0.0;
      for (int64_t h = 0; h < hidden; ++h) {
        const double x = source_value(blocks, nblocks, block_row_stride, block_stride, prefix, prefix_row_stride,
                                      dtype, t, b, h);
#if SITU_ORACLE_MUTANT == 26
        const double key = x * inv; /* planted: norm weight not applied */
#else
        const double key = x * inv * ar_value(norm_weight, norm_dtype, h);
#endif
        score += key * ar_value(proj_weight, proj_dtype, h);
      }
      logit[b] = score;
    }
    /* softmax over the sources, shifted by the largest logit (exact identity) */
    double mx = logit[0];
    for (int64_t b = 1; b < sources; ++b)
      if (logit[b] > mx) mx = logit[b];
    double z = 0.0;
    for (int64_t b = 0; b < sources; ++b) {
#if SITU_ORACLE_MUTANT == 27
      p[b] = exp(logit[b]); /* planted: no shift (overflows for large logits) */
#else
      p[b] = exp(logit[b] - mx);
#endif
      z += p[b];
    }
    for (int64_t b = 0; b < sources; ++b) {
      p[b] /= z;
      if (prob) prob[k * sources + b] = p[b];
    }
    for (int64_t h = 0; h < hidden; ++h) {
      double acc = 0.0, m = 0.0;
      for (int64_t b = 0; b < sources; ++b) {
        double x = source_value(blocks, nblocks, block_row_stride, block_stride, prefix, prefix_row_stride, dtype, t,
                                b, h);
#if SITU_ORACLE_MUTANT == 28
        x = x / sqrt(1.0 + x * x); /* planted: a transformed value combined instead of the raw one */
#endif
        acc += p[b] * x;
        m += p[b] * fabs(x);
      }
      out[k * hidden + h] = acc;
      if (mag) mag[k * hidden + h] = m;
    }
  }
  return 0;
}
