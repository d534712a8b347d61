/*
 * situ_glu.h -- C ABI of the B200 (sm_100a) routing-weighted SiTU-GLU library
 * (libsitu_glu.so).
 *
 * The operation (Megatron-LM PR #6673 "[Dev] Add SiTU-GLU through Transformer
 * Engine", section "Activation"; NeMo AutoModel API
 * nemo_automodel.components.models.kimi_k3.situ, `_situ_fwd_core`):
 *
 *     G = gate_up[:, 0:I]          (gate half, first)
 *     U = gate_up[:, I:2I]         (up half, second)
 *     T_g = beta * tanh(G / beta) * sigmoid(G)
 *     T_u = linear_beta * tanh(U / linear_beta)      (T_u = U without a linear beta)
 *     Y   = T_g * T_u * w          (w: routing weight of the row)
 *
 * and its analytic backward (NeMo `_situ_bwd_core`,
 * `_WeightedSiTUFunction.backward`), which recomputes the fp32 chain from the
 * saved low-precision inputs only:
 *
 *     dG  = go * w * T_u * T_g'
 *     dU  = go * w * T_g * T_u'
 *     d_w = sum over the I columns of go * T_g * T_u     (per row)
 *
 * Conventions shared by every entry point:
 *   - All functions are extern "C", never throw, and are thread-safe.
 *   - Matrices are row-major with an explicit row stride in ELEMENTS.  Leading
 *     batch dimensions are flattened into `tokens` by the caller.
 *   - All tensor pointers are DEVICE pointers on the CUDA device that is
 *     current on the calling thread.  The caller owns every buffer; the
 *     library allocates nothing and keeps no state except a cached SM count
 *     per device and the launch cap set by situ_glu_set_max_ctas().
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *     stream) and the call returns without synchronising.  Errors raised while
 *     the kernels run surface at the caller's next synchronisation.
 *   - Arguments are validated on the host before anything is launched; on any
 *     non-OK status nothing was enqueued and no output was touched.
 *     situ_glu_last_error() then describes the failure.
 *   - Arithmetic is fp32 in registers; each output is rounded once,
 *     round-to-nearest-even, to its storage dtype.
 */
#ifndef SITU_GLU_H_
#define SITU_GLU_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SITU_GLU_ABI_VERSION 8

typedef enum situ_status {
  SITU_OK = 0,
  SITU_ERR_INVALID_ARG = 1, /* NULL pointer, bad size, stride, beta, enum or aliasing */
  SITU_ERR_UNSUPPORTED = 2, /* a valid request the library does not implement         */
  SITU_ERR_MISALIGNED = 3,  /* a base address or row pitch is not 16-byte aligned     */
  SITU_ERR_CUDA = 4         /* the CUDA runtime reported an error at launch           */
} situ_status_t;

/* Storage dtype of a tensor.  bf16 = IEEE binary32 truncated to its upper 16
 * bits (the torch.bfloat16 layout). */
typedef enum situ_dtype {
  SITU_DTYPE_BF16 = 0,
  SITU_DTYPE_F32 = 1
} situ_dtype_t;

/* How the routing weights line up with the rows (NeMo `_situ_rw_is_row_aligned`
 * and `_WeightedSiTUFunction.forward`, parameter routing_weights: "row-aligned
 * with shape [..., k] matching gate_up's leading dimensions (typically
 * [tokens, 1]) or broadcastable against them"). */
typedef enum situ_rw_mode {
  SITU_RW_ROW = 0,    /* one weight per row: w[row * rw_stride], gradient per row   */
  SITU_RW_SCALAR = 1, /* one weight for every row: w[0]                             */
  SITU_RW_NONE = 2,   /* unweighted SiTU-GLU (w = 1; Megatron-LM PR #6673 "Design":
                         the TE SiTUGLU op / `situlu`).  rw and d_rw must be NULL. */
  SITU_RW_COL = 3,    /* one weight per column, shared by every row: w[i], contiguous
                         [inter]; its gradient is the sum over rows (needs workspace) */
  SITU_RW_FULL = 4    /* one weight per element: w[r * rw_stride + i], [tokens, >= inter]
                         (rw_stride = row pitch in elements); gradient per element */
} situ_rw_mode_t;

/*
 * Forward: out[r, i] = T_g(G[r, i]) * T_u(U[r, i]) * w[r].
 * Defined by: Megatron-LM PR #6673, section "Activation" (T_g, T_u, Y);
 * NeMo kimi_k3.situ `_situ_fwd_core` ("situ(g) * up(u0) * w") and
 * `_WeightedSiTUFunction.forward` (gate first half, up second half;
 * optional linear_beta).
 *
 *   gate_up            [tokens, >= 2*inter] in `dtype`, row pitch gate_up_row_stride
 *                      elements.  Read only.
 *   dtype              SITU_DTYPE_BF16 or SITU_DTYPE_F32 (also the dtype of out).
 *   tokens             rows, >= 0.  0 returns SITU_OK and launches nothing.
 *   inter              I, > 0.  inter * sizeof(dtype) must be a multiple of 16
 *                      (bf16: I % 8 == 0, fp32: I % 4 == 0).
 *   rw, rw_dtype       routing weights (bf16 or fp32), laid out per rw_mode;
 *                      rw_stride (elements): SITU_RW_ROW >= 0 (0 repeats w[0] on
 *                      every row, as an expanded tensor does); SITU_RW_FULL the
 *                      row pitch, >= inter; ignored otherwise.  SITU_RW_COL and
 *                      SITU_RW_FULL read the weights of one 16-byte vector of
 *                      gate_up in one piece: rw (and the FULL row pitch) must
 *                      be aligned to min(16, 16 / sizeof(dtype) * sizeof(rw_dtype))
 *                      bytes -- 16, or 8 for bf16 weights with fp32 gate_up.
 *                      SITU_RW_COL supports inter <= 16384.
 *   beta               gate beta, finite and > 0 (Megatron-LM PR #6673
 *                      "Design": finite positive betas).  Kimi-K3 default 4.
 *   has_linear_beta    0: T_u = U.  1: linear_beta is used, finite and > 0
 *                      (Kimi-K3 default 25).
 *   out                [tokens, >= inter] in `dtype`, row pitch out_row_stride
 *                      elements.  Written; must not overlap any input.
 *   stream             cudaStream_t.
 * Alignment: gate_up and out 16-byte aligned, row pitches multiples of 16
 * bytes; rw aligned to its element size.  Otherwise SITU_ERR_MISALIGNED.
 */
situ_status_t situ_glu_fwd(const void *gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                           int64_t gate_up_row_stride,
                           const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                           int64_t rw_stride,
                           double beta, int has_linear_beta, double linear_beta,
                           void *out, int64_t out_row_stride,
                           void *stream);

/*
 * Backward: recomputes T_g, T_u and their derivatives in fp32 from gate_up and
 * rw (the only saved inputs: NeMo `_WeightedSiTUFunction`, "saves only the
 * low-precision inputs") and writes, in one pass over HBM,
 *   d_gate_up[r, 0:I]  = go * w * T_u * T_g'
 *   d_gate_up[r, I:2I] = go * w * T_g * T_u'
 *   d_rw               = sum over columns of go * T_g * T_u: per row for
 *                        SITU_RW_ROW; summed over every row as well for
 *                        SITU_RW_SCALAR (autograd's sum to the weight's shape);
 *                        per column, summed over rows, for SITU_RW_COL; the
 *                        term go * T_g * T_u itself for SITU_RW_FULL.
 * Defined by: NeMo kimi_k3.situ `_situ_bwd_core` (d_g, d_u, red; want_drw)
 * and `_WeightedSiTUFunction.backward` (returns d_gate_up, d_routing_weights).
 *
 *   grad_out           [tokens, >= inter] in `dtype`, row pitch grad_out_row_stride.
 *   d_gate_up          [tokens, >= 2*inter] in `dtype`, row pitch
 *                      d_gate_up_row_stride.  Written; must not overlap any input.
 *   d_rw               NULL: the routing-weight gradient is not wanted and no
 *                      reduction runs (`want_drw` = false).  Otherwise in
 *                      rw_dtype, shaped like rw: element r at d_rw[r * d_rw_stride]
 *                      (row mode), one element (scalar mode), [inter] contiguous
 *                      (column mode, sums over rows), or element (r, i) at
 *                      d_rw[r * d_rw_stride + i] (full mode; d_rw_stride >= inter,
 *                      base and row pitch aligned like rw's).  Must be NULL for
 *                      SITU_RW_NONE.
 *   workspace          scratch for SITU_RW_SCALAR and SITU_RW_COL with
 *                      d_rw != NULL: at least situ_glu_bwd_workspace_bytes()
 *                      bytes, 16-byte aligned, device memory owned by the caller,
 *                      contents ignored on entry and undefined on exit.  May be
 *                      NULL when that query returns 0.
 * Other arguments as for situ_glu_fwd.  Per-row reductions run in a fixed
 * order, so every output is bitwise reproducible for a given build, shape and
 * load path, whatever the launch size.  dG and dU do not depend on the load
 * path either; d_rw's summation order does, within its rounding.
 */
situ_status_t situ_glu_bwd(const void *gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                           int64_t gate_up_row_stride,
                           const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                           int64_t rw_stride,
                           double beta, int has_linear_beta, double linear_beta,
                           const void *grad_out, int64_t grad_out_row_stride,
                           void *d_gate_up, int64_t d_gate_up_row_stride,
                           void *d_rw, int64_t d_rw_stride,
                           void *workspace, size_t workspace_bytes,
                           void *stream);

/* Bytes of workspace situ_glu_bwd (and situ_glu_bwd_mxfp8) needs with
 * want_drw != 0: tokens * 4 for SITU_RW_SCALAR (one partial per row),
 * ceil(tokens / 16) * inter * 4 for SITU_RW_COL (one partial per column per
 * chunk of 16 rows), each rounded up to 256; otherwise 0.  Non-positive
 * tokens or inter give 0. */
size_t situ_glu_bwd_workspace_bytes(int64_t tokens, int64_t inter, situ_rw_mode_t rw_mode, int want_drw);

/* ---- MXFP8 outputs ---------------------------------------------------------
 * Block-scaled FP8 outputs in the OCP Microscaling Formats (MX) v1.0 layout,
 * the format of the MXFP8 recipe the SiTU-GLU integration was tested with
 * (Megatron-LM PR #6673, "Test results"; the format itself is the public OCP
 * specification): every 32 consecutive elements of a row share one E8M0
 * scale byte S (X = 2^(S - 127); S = 255 is NaN) and each element is an FP8
 * E4M3 code (bias 7, largest normal 448, S.1111.111 NaN) of value / X,
 * rounded to nearest even.  The values are quantised from the kernel's fp32
 * results, never rounded to bf16 first.  A block holding a NaN or an
 * infinity gets S = 255 and NaN codes. */
typedef enum situ_mx_rule {
  SITU_MX_RULE_OCP = 0,  /* shared exponent floor(log2 amax) - 8, elements clamped to +-448
                            (the OCP MX conversion)                                          */
  SITU_MX_RULE_CEIL = 1  /* smallest exponent e with amax <= 448 * 2^e: no element clamps     */
} situ_mx_rule_t;        /* both at least -127 (S >= 0); amax = 0 gives S = 0                  */

/*
 * Forward with an MXFP8 Y: as situ_glu_fwd, but Y is written as
 *   y_data   [tokens, >= inter] E4M3 codes, row pitch y_data_row_stride BYTES
 *            (a multiple of 16; y_data 16-byte aligned);
 *   y_scale  [tokens, >= inter / 32] scale bytes, row pitch y_scale_row_stride
 *            bytes; byte b of a row scales columns [32 b, 32 b + 32).
 * inter must be a multiple of 32 (SITU_ERR_INVALID_ARG otherwise).  Routing
 * weights: SITU_RW_ROW, SITU_RW_SCALAR or SITU_RW_NONE (SITU_ERR_UNSUPPORTED
 * for the element-wise forms).  Neither output may overlap an input or the
 * other.  Other arguments and errors as for situ_glu_fwd.
 */
situ_status_t situ_glu_fwd_mxfp8(const void *gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                                 int64_t gate_up_row_stride,
                                 const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                                 int64_t rw_stride,
                                 double beta, int has_linear_beta, double linear_beta,
                                 void *y_data, int64_t y_data_row_stride,
                                 void *y_scale, int64_t y_scale_row_stride,
                                 situ_mx_rule_t rule, void *stream);

/*
 * Backward with an MXFP8 d_gate_up: as situ_glu_bwd, but d_gate_up is written
 * as E4M3 codes d_gate_up_data [tokens, >= 2 inter] (dG in columns [0, I), dU
 * in [I, 2I); row pitch in BYTES, a multiple of 16, base 16-byte aligned) and
 * scale bytes d_gate_up_scale [tokens, >= 2 inter / 32] (dG blocks first).
 * The routing-weight gradient (d_rw, workspace) is exactly as in situ_glu_bwd.
 * Same restrictions as situ_glu_fwd_mxfp8.
 */
situ_status_t situ_glu_bwd_mxfp8(const void *gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                                 int64_t gate_up_row_stride,
                                 const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                                 int64_t rw_stride,
                                 double beta, int has_linear_beta, double linear_beta,
                                 const void *grad_out, int64_t grad_out_row_stride,
                                 void *d_gate_up_data, int64_t d_gate_up_data_row_stride,
                                 void *d_gate_up_scale, int64_t d_gate_up_scale_row_stride,
                                 situ_mx_rule_t rule,
                                 void *d_rw, int64_t d_rw_stride,
                                 void *workspace, size_t workspace_bytes,
                                 void *stream);

/*
 * Forward with an NVFP4 Y (NVIDIA's NVFP4 format, the other block-scaled
 * recipe the integration was tested with -- Megatron-LM PR #6673, "Test
 * results"; the format is NVIDIA's public definition): with A the largest
 * finite |Y| of the call and S_enc = 448 * 6 / A (1 when A is 0 or not finite),
 *   y_scale  [tokens, >= inter / 16] E4M3 codes s_b = E4M3(amax_b S_enc / 6)
 *            of every 16 consecutive elements of a row (0x7F for a block
 *            holding NaN or infinity); row pitch y_scale_row_stride bytes
 *   y_data   [tokens, >= inter / 2] bytes of packed FP4 E2M1 codes of
 *            Y S_enc / s_b (nearest even, clamped to +-6), element 2k in the
 *            low nibble of byte k; row pitch y_data_row_stride bytes (a
 *            multiple of 4, base 4-byte aligned)
 *   amax     device fp32: A.  amax_given = 0: the library computes it first
 *            (a pass that reads gate_up once more) and writes it here;
 *            amax_given = 1: the caller's A is used (e.g. from an earlier
 *            step, or a maximum reduced over the ranks that hold the shards
 *            of one tensor); block scales and codes saturate (448, +-6) where
 *            it is below the call's own maximum; amax_given = 2: only A is
 *            computed and written (y_data and y_scale may be NULL), the first
 *            half of a sharded tensor's two-step coding.
 * A consumer decodes code q of block b as q * s_b * A / 2688.  inter must be a
 * multiple of 16; routing weights per row, broadcast or none.  Other
 * arguments and errors as for situ_glu_fwd.
 */
situ_status_t situ_glu_fwd_nvfp4(const void *gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                                 int64_t gate_up_row_stride,
                                 const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                                 int64_t rw_stride,
                                 double beta, int has_linear_beta, double linear_beta,
                                 void *y_data, int64_t y_data_row_stride,
                                 void *y_scale, int64_t y_scale_row_stride,
                                 float *amax, int amax_given, void *stream);

/*
 * Backward with an NVFP4 d_gate_up (format as for situ_glu_fwd_nvfp4; the
 * NVFP4 recipe's backward, Megatron-LM PR #6673, "Test results"): with A the
 * largest finite |dG|, |dU| of the call (one tensor scale S_enc = 2688 / A for
 * the whole d_gate_up),
 *   d_gate_up_data   [tokens, >= inter] bytes: dG's packed E2M1 codes
 *                    (inter / 2 bytes), then dU's; row pitch a multiple of 4,
 *                    base 4-byte aligned
 *   d_gate_up_scale  [tokens, >= 2 inter / 16] E4M3 block scales: dG's, then dU's
 *   amax / amax_given as for situ_glu_fwd_nvfp4 (amax_given = 0: a first pass
 *                    over gate_up and grad_out computes A; 2: only A, with
 *                    d_rw NULL)
 * d_rw, workspace and every other argument and error as for situ_glu_bwd
 * (per-row, broadcast or no routing weights); inter a multiple of 16.
 */
situ_status_t situ_glu_bwd_nvfp4(const void *gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                                 int64_t gate_up_row_stride,
                                 const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                                 int64_t rw_stride,
                                 double beta, int has_linear_beta, double linear_beta,
                                 const void *grad_out, int64_t grad_out_row_stride,
                                 void *d_gate_up_data, int64_t d_gate_up_data_row_stride,
                                 void *d_gate_up_scale, int64_t d_gate_up_scale_row_stride,
                                 float *amax, int amax_given,
                                 void *d_rw, int64_t d_rw_stride,
                                 void *workspace, size_t workspace_bytes, void *stream);

/* ---- FC1 grouped GEMM + SiTU-GLU --------------------------------------------
 * Megatron-LM PR #6673, "Design": with a SiTU-capable cuDNN frontend FC1's
 * grouped GEMM and SiTU-GLU run as one fused operation.  For token row r of
 * expert e (rows [offsets[e], offsets[e+1]) of x):
 *   G[r, i] = sum_k x[r, k] w1[e 2I + i, k],  U[r, i] = sum_k x[r, k] w1[e 2I + I + i, k]
 *   y[r, i] = T_g(G) T_u(U) w[r]                (as situ_glu_fwd, from fp32 G, U)
 * The products accumulate in fp32 on the tensor cores; G and U are never
 * written.
 *
 *   x         bf16 [tokens, >= hidden], row pitch x_row_stride elements
 *   w1        bf16 [experts * 2 inter, >= hidden], row pitch w1_row_stride:
 *             expert e's inter gate rows, then its inter up rows
 *   offsets   DEVICE int64 [experts + 1], non-decreasing; each value is
 *             clamped to [0, tokens] (a decreasing pair is an empty expert).
 *             Rows outside every expert are not written.  Overlapping ranges
 *             (non-monotone offsets) leave those rows unspecified.
 *   rw        per-row (SITU_RW_ROW), broadcast (SITU_RW_SCALAR) or no
 *             (SITU_RW_NONE) routing weights, as for situ_glu_fwd
 *   y         bf16 [tokens, >= inter], row pitch y_row_stride; must not
 *             overlap an input
 * hidden must be a multiple of 64, inter of 128, experts in [1, 1024]
 * (SITU_ERR_UNSUPPORTED otherwise); x, w1, y 16-byte aligned with row pitches
 * of a multiple of 16 bytes, offsets 8-byte aligned.  tokens == 0 launches
 * nothing.  The kernel uses the whole tensor memory and about 200 KiB of
 * shared memory of each SM it runs on; every internal wait is bounded and an
 * expired wait is reported by situ_glu_device_status.
 */
situ_status_t situ_glu_fc1_fwd(const void *x, int64_t tokens, int64_t hidden, int64_t x_row_stride,
                               const void *w1, int64_t experts, int64_t inter, int64_t w1_row_stride,
                               const int64_t *offsets,
                               const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                               int64_t rw_stride,
                               double beta, int has_linear_beta, double linear_beta,
                               void *y, int64_t y_row_stride,
                               void *stream);

/* ---- FC2 data gradient + SiTU-GLU backward --------------------------------------
 * The backward of the fused grouped MLP at the activation (Megatron-LM PR
 * #6673, "Test results": the fused path's backward with a dSiTU correction):
 * FC2's data gradient is the activation's upstream gradient, so for token row
 * r of expert e
 *   dY[r, i]            = sum_h dout[r, h] W2_e[h, i]       (fp32 on the tensor cores, never written)
 *   d_gate_up[r, i]     = dY w[r] T_u(U) T_g'(G)            (as situ_glu_bwd with grad_out = dY)
 *   d_gate_up[r, I + i] = dY w[r] T_g(G) T_u'(U)
 *   d_rw[r]             = sum_i dY T_g(G) T_u(U)
 * with G, U the halves of the saved gate_up row.
 *
 *   dout        bf16 [tokens, >= hidden], row pitch dout_row_stride
 *   w2t         bf16 [experts * inter, >= hidden]: FC2's weight W2_e [hidden,
 *               inter] TRANSPOSED (row e * inter + i holds W2_e[:, i])
 *   offsets     DEVICE int64 [experts + 1], as for situ_glu_fc1_fwd
 *   gate_up     bf16 [tokens, >= 2 inter], the forward's saved FC1 output
 *   rw, rw_dtype, rw_stride  per-row routing weights (SITU_RW_ROW) or none
 *               (SITU_RW_NONE: rw and d_rw NULL); other modes SITU_ERR_UNSUPPORTED
 *   d_gate_up   bf16 [tokens, >= 2 inter]; d_rw (rw_dtype, stride d_rw_stride)
 *               or NULL when not wanted
 *   workspace   >= situ_glu_fc2_dgrad_workspace_bytes() bytes (per-row,
 *               per-256-column-tile d_rw partials, added in tile order)
 * hidden a multiple of 64, inter of 256, experts in [1, 1024]; alignment and
 * offsets rules as for situ_glu_fc1_fwd.  Rows outside every expert are not
 * written.
 */
situ_status_t situ_glu_fc2_dgrad_bwd(const void *dout, int64_t tokens, int64_t hidden, int64_t dout_row_stride,
                                     const void *w2t, int64_t experts, int64_t inter, int64_t w2t_row_stride,
                                     const int64_t *offsets,
                                     const void *gate_up, int64_t gate_up_row_stride,
                                     const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                                     int64_t rw_stride,
                                     double beta, int has_linear_beta, double linear_beta,
                                     void *d_gate_up, int64_t d_gate_up_row_stride,
                                     void *d_rw, int64_t d_rw_stride,
                                     void *workspace, size_t workspace_bytes,
                                     void *stream);

/* Bytes of workspace situ_glu_fc2_dgrad_bwd needs: tokens * (inter / 256) * 4
 * rounded up to 256 when want_drw != 0, else 0. */
size_t situ_glu_fc2_dgrad_workspace_bytes(int64_t tokens, int64_t inter, int want_drw);

/* ---- Attention-residual mixing core -------------------------------------------
 * NeMo AutoModel API, kimi_k3.situ, `_attn_res_core` ("fp32 attention-residual
 * mixing chain") and `_apply_attn_res` (mix the current [tokens, hidden] sum
 * with the stored [tokens, blocks, hidden] sums).  For token t, with sources
 * b = 0 .. S-1 the nblocks stored sums followed by the prefix sum (if given):
 *   logit[b] = sum_h x_b[h] / sqrt(mean_h x_b^2 + eps) * norm_weight[h] * proj_weight[h]
 *   out[h]   = sum_b softmax_b(logit)[b] x_b[h]
 * in fp32 (RMSNorm in its standard form; the projection is the squeezed
 * [hidden] weight of a hidden -> 1 linear layer).
 *
 *   blocks            stored sums, dtype; element (t, b, h) at
 *                     blocks[t * block_row_stride + b * block_stride + h];
 *                     may be NULL when nblocks == 0
 *   prefix            current sum [tokens, >= hidden] (row pitch
 *                     prefix_row_stride), the last source; NULL: none
 *   dtype             storage of blocks and prefix (bf16 or fp32)
 *   norm_weight, proj_weight  [hidden] in their own dtypes
 *   variance_epsilon  RMSNorm epsilon, finite and >= 0
 *   out               [tokens, >= hidden] in out_dtype, row pitch
 *                     out_row_stride; must not overlap an input
 * 1 <= S <= 16 and hidden <= 32768 (SITU_ERR_UNSUPPORTED otherwise); hidden *
 * sizeof(dtype) a multiple of 16; sources and out 16-byte aligned with row
 * (and source) pitches of a multiple of 16 bytes.  Results do not depend on
 * the launch size.
 */
situ_status_t situ_attn_res_fwd(const void *blocks, int64_t nblocks, int64_t block_row_stride,
                                int64_t block_stride, const void *prefix, int64_t prefix_row_stride,
                                situ_dtype_t dtype, int64_t tokens, int64_t hidden,
                                const void *norm_weight, situ_dtype_t norm_dtype,
                                const void *proj_weight, situ_dtype_t proj_dtype,
                                double variance_epsilon,
                                void *out, situ_dtype_t out_dtype, int64_t out_row_stride,
                                void *stream);

/* Static, human-readable name of a status code. */
const char *situ_glu_status_string(situ_status_t status);

/* Description of the most recent non-OK status returned on the calling thread
 * ("" if none).  The pointer stays valid until the thread's next call. */
const char *situ_glu_last_error(void);

/* SITU_GLU_ABI_VERSION of the built library. */
int situ_glu_abi_version(void);

/* Upper bound on the CTAs of each launch (0 = automatic: SM count times the
 * CTAs per SM the occupancy calculator allows).  Results do not depend on it;
 * it exists for tuning and to check that.  Process-wide; returns the previous
 * value, or -1 (and changes nothing) for a negative argument. */
int situ_glu_set_max_ctas(int max_ctas);

/* How the kernels read HBM.  0 (default): every thread loads its own 16-byte
 * vectors into registers, the CTA's next row while it computes the current
 * one.  1: one lane per CTA streams chunks of rows into a shared-memory ring
 * with TMA bulk copies (cp.async.bulk) and the other warps compute from it.
 * Both paths run the same arithmetic, so results are bitwise identical; on
 * B200 the direct path measured faster on every workload.  Process-wide;
 * returns the previous value, or -1 (and changes nothing) for any other
 * argument. */
int situ_glu_set_load_path(int path);

/* Status word the kernels set on the current device when one of their
 * bounded waits (on a shared-memory stage, 2 s at most) expires: 0 = none
 * has, 1 = a wait expired and that launch's outputs are not valid.  A kernel
 * whose wait expires returns instead of hanging.  Synchronises the device
 * first; a nonzero `clear` resets the word.  Returns -1 if the CUDA runtime
 * reports an error. */
int situ_glu_device_status(int clear);

/* Test hook for the bounded waits above: enqueues on `stream` one thread
 * block that waits, with the limit `limit_ns` (1 to 10^10 ns) instead of the
 * kernels' 2 s, on a shared-memory mbarrier that nothing completes.  The wait
 * runs out, the block sets the status word to 1 and returns, as a kernel
 * whose staged copy never lands would; nothing faults and the context stays
 * usable.  SITU_ERR_INVALID_ARG (nothing enqueued) for a limit outside that
 * range. */
situ_status_t situ_glu_wait_probe(int64_t limit_ns, void *stream);

/*
 * Backward without caller scratch.  Same arguments and results as
 * situ_glu_bwd, minus `workspace` and `workspace_bytes`.  The pages describe
 * no counterpart of this entry point: it exists for callers that cannot
 * allocate device memory where they run the backward (an engine that
 * reserves all of HBM at start-up and gives its kernels only planned
 * buffers, or a C caller without a CUDA allocator).  Two modes need
 * scratch when d_rw != NULL, and in both it comes from a fixed 1 MiB array
 * inside this library instead of a caller workspace: a routing weight
 * broadcast to every row (SITU_RW_SCALAR: one fp32 partial per row) and a
 * per-column weight (SITU_RW_COL: one fp32 partial per column per chunk of
 * 16 rows).
 *   - Limit: the bytes situ_glu_bwd_workspace_bytes reports must not exceed
 *     1 MiB (1048576): tokens * 4 for SITU_RW_SCALAR, i.e. at most 262144
 *     rows; ceil(tokens / 16) * inter * 4 for SITU_RW_COL, each rounded up
 *     to 256 (at inter = 4096: at most 1024 rows).  More returns
 *     SITU_ERR_UNSUPPORTED before anything is launched.  Other modes need no
 *     scratch and have no limit beyond situ_glu_bwd's.
 *   - Allocates nothing (no cudaMalloc, cudaFree or allocating library call).
 *     The array exists once per GPU that loads the library, until exit.
 *   - The first call on a device looks up the array's device address (with
 *     that device current) and caches it for the life of the process; make
 *     that first call before any stream capture.  cudaDeviceReset discards
 *     the device's copy of the array, and the cached address with it: do not
 *     call this entry point on a device after resetting it.
 *   - Every call shares the one array, and it keeps whatever the last call
 *     left in it (nothing in it has to start at zero).  Calls whose kernels
 *     overlap on the GPU -- on different streams, or from different threads
 *     -- race on it and give undefined results; serialise them.
 */
situ_status_t situ_glu_bwd_no_alloc(const void *gate_up, situ_dtype_t dtype, int64_t tokens,
                                    int64_t inter, int64_t gate_up_row_stride,
                                    const void *rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                                    int64_t rw_stride,
                                    double beta, int has_linear_beta, double linear_beta,
                                    const void *grad_out, int64_t grad_out_row_stride,
                                    void *d_gate_up, int64_t d_gate_up_row_stride,
                                    void *d_rw, int64_t d_rw_stride,
                                    void *stream);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* SITU_GLU_H_ */
