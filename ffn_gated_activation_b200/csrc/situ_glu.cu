// situ_glu.cu -- routing-weighted SiTU-GLU forward and fused analytic backward
// for B200 (sm_100a), behind the C ABI declared in include/situ_glu.h.
//
// The operation (Megatron-LM PR #6673 "[Dev] Add SiTU-GLU through Transformer
// Engine", section "Activation"; NeMo AutoModel kimi_k3.situ `_situ_fwd_core`,
// `_situ_bwd_core`):
//   T_g = beta tanh(G/beta) sigmoid(G),  T_u = beta_L tanh(U/beta_L) (or U),
//   Y = T_g T_u w,
//   dG = go w T_u T_g',  dU = go w T_g T_u',  d_w = sum_i go T_g T_u.
//
// The path is bound by HBM bandwidth (a few bytes per element, no contraction),
// so the kernels are streaming kernels: 16-byte vector loads and stores with
// streaming cache hints, one CTA per row at a time, a grid of (SMs x resident
// CTAs) that strides over rows, fp32 arithmetic in registers.  Tensor cores
// play no part.
//
// Arithmetic.  With E = exp(-x) for x >= 0 every transcendental of the chain is
// a rational function of a few exponentials:
//   tanh(|a|)  = (1 - E_t) / (1 + E_t),        E_t = exp(-2|a|)
//   sech^2(a)  = 4 E_t / (1 + E_t)^2
//   sigmoid(g) = 1 / (1 + E_s)  (g >= 0)   or   E_s / (1 + E_s)  (g < 0),  E_s = exp(-|g|)
//   sigmoid(g) (1 - sigmoid(g)) = E_s / (1 + E_s)^2
// All factors (1 + E) lie in (1, 2], so the denominators of a whole element
// are multiplied together and inverted with ONE reciprocal.  For beta = 4,
// E_s = E_t^2 (beta = 2: E_s = E_t; beta = 1: E_t = E_s^2), so the gate needs
// one exponential.  The forward then costs 3 MUFU operations per element
// (two exp2, one reciprocal) and the backward the same.  1 - E_t loses
// relative accuracy as x -> 0; below a threshold it is taken from the Taylor
// series of 1 - exp(-x) instead.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "situ_glu.h"

namespace {

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------

constexpr float kNegLog2e = -1.4426950408889634f;  // -log2(e)
constexpr int kMaxThreads = 256;                   // CTA size ceiling
constexpr int kVecBytes = 16;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Read-only streaming load (no L1 allocation) and evict-first store: every
// byte is touched once.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ void st_stream(void* p, const uint4& v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// Storage types.  A 16-byte vector holds 8 bf16 or 4 fp32 values.
struct Bf16 {
  static constexpr int kPerVec = 8;
  __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);           // element 2k: low half
      f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);  // element 2k+1: high half
    }
  }
  __device__ __forceinline__ static uint4 pack(const float (&f)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)  // cvt packs its first source into the high half
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(w[k]) : "f"(f[2 * k + 1]), "f"(f[2 * k]));
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

struct F32 {
  static constexpr int kPerVec = 4;
  __device__ __forceinline__ static void unpack(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
  }
  __device__ __forceinline__ static uint4 pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};

// 1 - exp(-x) for x >= 0, given E = ex2 approximation of exp(-x).  Where x is
// small, 1 - E cancels; there the Taylor series x - x^2/2 + x^3/6 - ... is
// used.  bf16 outputs: series to x^4 below x = 1/16 (truncation < 2^-22
// relative; 1 - E above it is within ~2^-19).  fp32 outputs: series to x^6
// below x = 1/4 (truncation < 2^-24; 1 - E above it within ~2^-21).
template <typename S>
__device__ __forceinline__ float one_minus_exp_neg(float x, float E);

template <>
__device__ __forceinline__ float one_minus_exp_neg<Bf16>(float x, float E) {
  float p = fmaf(x, -1.0f / 24.0f, 1.0f / 6.0f);
  p = fmaf(p, x, -0.5f);
  p = fmaf(p, x, 1.0f);
  return x < 0.0625f ? p * x : 1.0f - E;
}

template <>
__device__ __forceinline__ float one_minus_exp_neg<F32>(float x, float E) {
  float p = fmaf(x, -1.0f / 720.0f, 1.0f / 120.0f);
  p = fmaf(p, x, -1.0f / 24.0f);
  p = fmaf(p, x, 1.0f / 6.0f);
  p = fmaf(p, x, -0.5f);
  p = fmaf(p, x, 1.0f);
  return x < 0.25f ? p * x : 1.0f - E;
}

// How the two gate exponentials relate for the given beta.
enum GateMode : int {
  kGateGeneric = 0,  // two independent exponentials
  kGateSquare = 1,   // beta = 4: E_s = E_t^2
  kGateEqual = 2,    // beta = 2: E_s = E_t
  kGateRoot = 3,     // beta = 1: E_t = E_s^2
};

struct Coeffs {
  float beta;      // gate beta
  float lb;        // linear beta (unused without one)
  float neg_kt;    // -2 log2(e) / beta: E_t = 2^(|g| neg_kt)
  float xt_scale;  // 2 / beta: series argument x_t = 2|g| / beta
  float neg_ku;    // -2 log2(e) / beta_L
  float xu_scale;  // 2 / beta_L
  float bb;        // beta * beta_L (beta without a linear beta)
};

struct GateExp {
  float Et;   // exp(-2|g|/beta)
  float Es;   // exp(-|g|)
  float emt;  // 1 - Et, accurate
};

template <int GATE, typename S>
__device__ __forceinline__ GateExp gate_exp(float g, const Coeffs& c) {
  const float ag = fabsf(g);
  GateExp r;
  if (GATE == kGateSquare) {
    r.Et = ex2_approx(ag * c.neg_kt);
    r.Es = r.Et * r.Et;
  } else if (GATE == kGateEqual) {
    r.Et = ex2_approx(ag * c.neg_kt);
    r.Es = r.Et;
  } else if (GATE == kGateRoot) {
    r.Es = ex2_approx(ag * kNegLog2e);
    r.Et = r.Es * r.Es;
  } else {
    r.Et = ex2_approx(ag * c.neg_kt);
    r.Es = ex2_approx(ag * kNegLog2e);
  }
  r.emt = one_minus_exp_neg<S>(ag * c.xt_scale, r.Et);
  return r;
}

// Forward of one element.  wbb = w * beta * beta_L (w * beta without one).
template <int GATE, bool HAS_LB, typename S>
__device__ __forceinline__ float situ_fwd_elem(float g, float u, float wbb, const Coeffs& c) {
  const GateExp e = gate_exp<GATE, S>(g, c);
  const float sig = g < 0.0f ? e.Es : 1.0f;    // sigmoid(g) * (1 + E_s)
  float num = copysignf(e.emt, g) * sig;        // T_g * (1 + E_t)(1 + E_s) / beta
  float den = (1.0f + e.Et) * (1.0f + e.Es);
  if (HAS_LB) {
    const float au = fabsf(u);
    const float Eu = ex2_approx(au * c.neg_ku);
    const float emu = one_minus_exp_neg<S>(au * c.xu_scale, Eu);
    num *= copysignf(emu, u);                   // T_u * (1 + E_u) / beta_L
    den *= 1.0f + Eu;
  } else {
    num *= u;
  }
  return num * wbb * rcp_approx(den);
}

// Backward of one element: writes dG, dU and returns go * T_g * T_u.
template <int GATE, bool HAS_LB, typename S>
__device__ __forceinline__ float situ_bwd_elem(float g, float u, float go, float gow, const Coeffs& c,
                                               float& dg, float& du) {
  const GateExp e = gate_exp<GATE, S>(g, c);
  const float sig = g < 0.0f ? e.Es : 1.0f;
  const float tb = c.beta * copysignf(e.emt, g);  // beta tanh(g/beta) (1 + E_t)
  const float tg = tb * sig;                        // T_g * A
  const float opt = 1.0f + e.Et, ops = 1.0f + e.Es;
  const float A = opt * ops;
  // T_g' A^2 = [sech^2(g/beta) sigmoid(g)] A^2 + [beta tanh(g/beta) sigmoid(1 - sigmoid)] A^2
  //          = 4 E_t sig (1 + E_s)            + tb (1 + E_t) E_s
  const float ng = 4.0f * e.Et * sig * ops + tb * opt * e.Es;
  if (HAS_LB) {
    const float au = fabsf(u);
    const float Eu = ex2_approx(au * c.neg_ku);
    const float tu = c.lb * copysignf(one_minus_exp_neg<S>(au * c.xu_scale, Eu), u);  // T_u * B
    const float B = 1.0f + Eu;
    const float AB = A * B;
    const float R = rcp_approx(AB * AB);  // 1 / (A^2 B^2)
    dg = gow * tu * ng * (B * R);          // go w T_u T_g'
    du = gow * tg * (4.0f * Eu) * (A * R);  // go w T_g sech^2(u / beta_L)
    return go * tg * tu * (AB * R);        // go T_g T_u
  } else {
    const float R = rcp_approx(A * A);
    dg = gow * u * ng * R;
    const float AR = A * R;                // 1 / A
    du = gow * tg * AR;
    return go * tg * u * AR;
  }
}

// Routing weight of a row.
struct RwArgs {
  const void* rw;
  int64_t stride;
  int mode;  // situ_rw_mode_t
  int bf16;  // storage dtype is bf16
};

__device__ __forceinline__ float load_rw(const RwArgs& a, int64_t row) {
  if (a.mode == SITU_RW_NONE) return 1.0f;
  const int64_t idx = a.mode == SITU_RW_ROW ? row * a.stride : 0;
  if (a.bf16) {
    const uint16_t h = __ldg(reinterpret_cast<const unsigned short*>(a.rw) + idx);
    return __uint_as_float(static_cast<uint32_t>(h) << 16);
  }
  return __ldg(reinterpret_cast<const float*>(a.rw) + idx);
}

// Sum over the CTA, in an order fixed by blockDim alone.  The result is valid
// in thread 0.  `slot` must alternate between two buffers from one call to
// the next so that a single barrier per call suffices.
__device__ __forceinline__ float block_sum(float v, float* slot) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) slot[warp] = v;
  __syncthreads();
  float total = 0.0f;
  if (warp == 0) {
    total = lane < static_cast<int>(blockDim.x >> 5) ? slot[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  return total;
}

// ---------------------------------------------------------------------------
// Kernels
// ---------------------------------------------------------------------------

struct FwdArgs {
  const char* gate_up;
  int64_t gu_pitch;  // bytes
  char* out;
  int64_t out_pitch;
  RwArgs rw;
  int64_t tokens;
  int half_bytes;  // inter * element size: offset of the up half
  int vpr;         // 16-byte vectors per half row
  Coeffs c;
};

template <typename S, int GATE, bool HAS_LB>
__global__ void __launch_bounds__(kMaxThreads) situ_glu_fwd_kernel(const FwdArgs a) {
  constexpr int N = S::kPerVec;
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    const char* gu = a.gate_up + row * a.gu_pitch;
    char* out = a.out + row * a.out_pitch;
    const float wbb = load_rw(a.rw, row) * a.c.bb;
    for (int j = threadIdx.x; j < a.vpr; j += blockDim.x) {
      const int off = j * kVecBytes;
      float g[N], u[N], y[N];
      S::unpack(ld_stream(gu + off), g);
      S::unpack(ld_stream(gu + a.half_bytes + off), u);
#pragma unroll
      for (int k = 0; k < N; ++k) y[k] = situ_fwd_elem<GATE, HAS_LB, S>(g[k], u[k], wbb, a.c);
      st_stream(out + off, S::pack(y));
    }
  }
}

struct BwdArgs {
  const char* gate_up;
  int64_t gu_pitch;
  const char* grad_out;
  int64_t go_pitch;
  char* d_gate_up;
  int64_t dgu_pitch;
  RwArgs rw;
  void* d_rw;          // row mode: per-row output (stride d_rw_stride)
  int64_t d_rw_stride;
  float* partials;     // scalar mode: per-row partial sums (workspace)
  int want_drw;
  int64_t tokens;
  int half_bytes;
  int vpr;
  Coeffs c;
};

__device__ __forceinline__ void store_rw_grad(void* base, int64_t idx, int bf16, float v) {
  if (bf16) {
    reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
  } else {
    reinterpret_cast<float*>(base)[idx] = v;
  }
}

template <typename S, int GATE, bool HAS_LB>
__global__ void __launch_bounds__(kMaxThreads) situ_glu_bwd_kernel(const BwdArgs a) {
  constexpr int N = S::kPerVec;
  __shared__ float red[2][kMaxThreads / 32];
  int parity = 0;
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    const char* gu = a.gate_up + row * a.gu_pitch;
    const char* go_row = a.grad_out + row * a.go_pitch;
    char* dgu = a.d_gate_up + row * a.dgu_pitch;
    const float w = load_rw(a.rw, row);
    float acc = 0.0f;
    for (int j = threadIdx.x; j < a.vpr; j += blockDim.x) {
      const int off = j * kVecBytes;
      float g[N], u[N], go[N], dg[N], du[N];
      S::unpack(ld_stream(gu + off), g);
      S::unpack(ld_stream(gu + a.half_bytes + off), u);
      S::unpack(ld_stream(go_row + off), go);
#pragma unroll
      for (int k = 0; k < N; ++k)
        acc += situ_bwd_elem<GATE, HAS_LB, S>(g[k], u[k], go[k], go[k] * w, a.c, dg[k], du[k]);
      st_stream(dgu + off, S::pack(dg));
      st_stream(dgu + a.half_bytes + off, S::pack(du));
    }
    if (a.want_drw) {  // uniform over the launch
      const float total = block_sum(acc, red[parity]);
      parity ^= 1;
      if (threadIdx.x == 0) {
        if (a.rw.mode == SITU_RW_SCALAR)
          a.partials[row] = total;
        else
          store_rw_grad(a.d_rw, row * a.d_rw_stride, a.rw.bf16, total);
      }
    }
  }
}

// Broadcast routing weight: sum the per-row partials in a fixed order.
constexpr int kFinalizeThreads = 1024;

__global__ void __launch_bounds__(kFinalizeThreads)
    situ_glu_dw_scalar_finalize_kernel(const float* partials, int64_t tokens, void* d_rw, int bf16) {
  __shared__ float red[kFinalizeThreads / 32];
  float s = 0.0f;
  for (int64_t r = threadIdx.x; r < tokens; r += blockDim.x) s += partials[r];
  const float total = block_sum(s, red);
  if (threadIdx.x == 0) store_rw_grad(d_rw, 0, bf16, total);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

thread_local char tl_last_error[512] = "";

situ_status_t fail(situ_status_t status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(tl_last_error, sizeof tl_last_error, fmt, ap);
  va_end(ap);
  return status;
}

std::atomic<int> g_max_ctas{0};

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];

situ_status_t device_sm_count(int* sms) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
  if (dev >= 0 && dev < kMaxDevices) {
    const int cached = g_sm_count[dev].load(std::memory_order_relaxed);
    if (cached > 0) {
      *sms = cached;
      return SITU_OK;
    }
  }
  int n = 0;
  err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (err != cudaSuccess || n <= 0)
    return fail(SITU_ERR_CUDA, "cudaDeviceGetAttribute(SM count): %s", cudaGetErrorString(err));
  if (dev >= 0 && dev < kMaxDevices) g_sm_count[dev].store(n, std::memory_order_relaxed);
  *sms = n;
  return SITU_OK;
}

bool finite_positive(double x) { return std::isfinite(x) && x > 0.0; }

int elem_size(situ_dtype_t d) { return d == SITU_DTYPE_BF16 ? 2 : 4; }

bool valid_dtype(int d) { return d == SITU_DTYPE_BF16 || d == SITU_DTYPE_F32; }

// Byte range [lo, hi) spanned by a row-pitched matrix.
struct Span {
  uintptr_t lo, hi;
};

Span matrix_span(const void* base, int64_t rows, int64_t pitch_elems, int64_t width_elems, int es) {
  const uintptr_t lo = reinterpret_cast<uintptr_t>(base);
  const uint64_t bytes = (static_cast<uint64_t>(rows - 1) * pitch_elems + width_elems) * es;
  return {lo, lo + bytes};
}

bool overlap(const Span& a, const Span& b) { return a.lo < b.hi && b.lo < a.hi; }

// rows * pitch + width fits in int64 bytes.
bool span_fits(int64_t rows, int64_t pitch, int64_t width, int es) {
  const int64_t limit = INT64_MAX / es - width;
  return rows <= 1 || (pitch <= limit / (rows - 1));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int64_t kMaxInter = int64_t(1) << 28;

// Checks common to fwd and bwd.  Fills coefficients and the gate mode.
situ_status_t check_common(situ_dtype_t dtype, int64_t tokens, int64_t inter, int64_t gu_stride,
                           const void* rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                           int64_t rw_stride, double beta, int has_lb, double lb, Coeffs* c,
                           int* gate_mode) {
  if (!valid_dtype(dtype)) return fail(SITU_ERR_INVALID_ARG, "dtype %d is not a situ_dtype_t", (int)dtype);
  if (rw_mode != SITU_RW_ROW && rw_mode != SITU_RW_SCALAR && rw_mode != SITU_RW_NONE)
    return fail(SITU_ERR_INVALID_ARG, "rw_mode %d is not a situ_rw_mode_t", (int)rw_mode);
  if (rw_mode != SITU_RW_NONE && !valid_dtype(rw_dtype))
    return fail(SITU_ERR_INVALID_ARG, "rw_dtype %d is not a situ_dtype_t", (int)rw_dtype);
  if (tokens < 0) return fail(SITU_ERR_INVALID_ARG, "tokens = %lld < 0", (long long)tokens);
  if (inter <= 0) return fail(SITU_ERR_INVALID_ARG, "inter = %lld <= 0", (long long)inter);
  if (inter > kMaxInter)
    return fail(SITU_ERR_UNSUPPORTED, "inter = %lld exceeds %lld", (long long)inter, (long long)kMaxInter);
  if (!finite_positive(beta)) return fail(SITU_ERR_INVALID_ARG, "beta must be finite and > 0");
  if (has_lb != 0 && has_lb != 1) return fail(SITU_ERR_INVALID_ARG, "has_linear_beta must be 0 or 1");
  if (has_lb && !finite_positive(lb)) return fail(SITU_ERR_INVALID_ARG, "linear_beta must be finite and > 0");
  if (gu_stride < 2 * inter) return fail(SITU_ERR_INVALID_ARG, "gate_up_row_stride < 2 * inter");
  if (rw_mode == SITU_RW_NONE) {
    if (rw != nullptr) return fail(SITU_ERR_INVALID_ARG, "rw must be NULL for SITU_RW_NONE");
  } else if (tokens > 0 && rw == nullptr) {
    return fail(SITU_ERR_INVALID_ARG, "rw is NULL");
  }
  if (rw_mode == SITU_RW_ROW && rw_stride < 0) return fail(SITU_ERR_INVALID_ARG, "rw_stride < 0");
  const int es = elem_size(dtype);
  if ((inter * es) % kVecBytes != 0)
    return fail(SITU_ERR_MISALIGNED, "inter * element size (%lld bytes) is not a multiple of 16",
                (long long)(inter * es));

  const double kLog2e = 1.4426950408889634;
  c->beta = static_cast<float>(beta);
  c->neg_kt = static_cast<float>(-2.0 * kLog2e / beta);
  c->xt_scale = static_cast<float>(2.0 / beta);
  c->lb = has_lb ? static_cast<float>(lb) : 1.0f;
  c->neg_ku = has_lb ? static_cast<float>(-2.0 * kLog2e / lb) : 0.0f;
  c->xu_scale = has_lb ? static_cast<float>(2.0 / lb) : 0.0f;
  c->bb = static_cast<float>(has_lb ? beta * lb : beta);
  *gate_mode = beta == 4.0 ? kGateSquare : beta == 2.0 ? kGateEqual : beta == 1.0 ? kGateRoot : kGateGeneric;
  return SITU_OK;
}

int choose_threads(int vpr) {
  const int per_thread = (vpr + kMaxThreads - 1) / kMaxThreads;
  const int nt = (vpr + per_thread - 1) / per_thread;
  return (nt + 31) / 32 * 32;
}

situ_status_t launch_grid(const void* kernel, int threads, int64_t tokens, int* grid) {
  int sms = 0;
  situ_status_t st = device_sm_count(&sms);
  if (st != SITU_OK) return st;
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, 0);
  if (err != cudaSuccess || per_sm <= 0)
    return fail(SITU_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(err));
  int64_t g = static_cast<int64_t>(sms) * per_sm;
  const int cap = g_max_ctas.load(std::memory_order_relaxed);
  if (cap > 0 && g > cap) g = cap;
  if (g > tokens) g = tokens;
  *grid = static_cast<int>(g);
  return SITU_OK;
}

situ_status_t check_launch(const char* what) {
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(err));
  return SITU_OK;
}

using FwdKernel = void (*)(FwdArgs);
using BwdKernel = void (*)(BwdArgs);

template <typename S, bool LB>
FwdKernel pick_fwd_gate(int gate) {
  switch (gate) {
    case kGateSquare: return situ_glu_fwd_kernel<S, kGateSquare, LB>;
    case kGateEqual: return situ_glu_fwd_kernel<S, kGateEqual, LB>;
    case kGateRoot: return situ_glu_fwd_kernel<S, kGateRoot, LB>;
    default: return situ_glu_fwd_kernel<S, kGateGeneric, LB>;
  }
}

FwdKernel pick_fwd(situ_dtype_t dtype, int gate, bool lb) {
  if (dtype == SITU_DTYPE_BF16) return lb ? pick_fwd_gate<Bf16, true>(gate) : pick_fwd_gate<Bf16, false>(gate);
  return lb ? pick_fwd_gate<F32, true>(gate) : pick_fwd_gate<F32, false>(gate);
}

template <typename S, bool LB>
BwdKernel pick_bwd_gate(int gate) {
  switch (gate) {
    case kGateSquare: return situ_glu_bwd_kernel<S, kGateSquare, LB>;
    case kGateEqual: return situ_glu_bwd_kernel<S, kGateEqual, LB>;
    case kGateRoot: return situ_glu_bwd_kernel<S, kGateRoot, LB>;
    default: return situ_glu_bwd_kernel<S, kGateGeneric, LB>;
  }
}

BwdKernel pick_bwd(situ_dtype_t dtype, int gate, bool lb) {
  if (dtype == SITU_DTYPE_BF16) return lb ? pick_bwd_gate<Bf16, true>(gate) : pick_bwd_gate<Bf16, false>(gate);
  return lb ? pick_bwd_gate<F32, true>(gate) : pick_bwd_gate<F32, false>(gate);
}

}  // namespace

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------

extern "C" {

situ_status_t situ_glu_fwd(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                           int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype,
                           situ_rw_mode_t rw_mode, int64_t rw_stride, double beta, int has_linear_beta,
                           double linear_beta, void* out, int64_t out_row_stride, void* stream) {
  tl_last_error[0] = '\0';
  Coeffs c;
  int gate = kGateGeneric;
  situ_status_t st = check_common(dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                  rw_stride, beta, has_linear_beta, linear_beta, &c, &gate);
  if (st != SITU_OK) return st;
  if (out_row_stride < inter) return fail(SITU_ERR_INVALID_ARG, "out_row_stride < inter");
  if (tokens == 0) return SITU_OK;
  if (gate_up == nullptr || out == nullptr) return fail(SITU_ERR_INVALID_ARG, "gate_up or out is NULL");
  const int es = elem_size(dtype);
  if (!span_fits(tokens, gate_up_row_stride, 2 * inter, es) || !span_fits(tokens, out_row_stride, inter, es) ||
      (rw_mode == SITU_RW_ROW && !span_fits(tokens, rw_stride, 1, elem_size(rw_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  if (!aligned(gate_up, 16) || !aligned(out, 16) || (gate_up_row_stride * es) % 16 != 0 ||
      (out_row_stride * es) % 16 != 0)
    return fail(SITU_ERR_MISALIGNED, "gate_up/out base or row pitch not 16-byte aligned");
  if (rw_mode != SITU_RW_NONE && !aligned(rw, elem_size(rw_dtype)))
    return fail(SITU_ERR_MISALIGNED, "rw not aligned to its element size");
  const Span s_out = matrix_span(out, tokens, out_row_stride, inter, es);
  if (overlap(s_out, matrix_span(gate_up, tokens, gate_up_row_stride, 2 * inter, es)))
    return fail(SITU_ERR_INVALID_ARG, "out overlaps gate_up");
  if (rw_mode == SITU_RW_ROW && overlap(s_out, matrix_span(rw, tokens, rw_stride, 1, elem_size(rw_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "out overlaps rw");
  if (rw_mode == SITU_RW_SCALAR && overlap(s_out, matrix_span(rw, 1, 1, 1, elem_size(rw_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "out overlaps rw");

  FwdArgs a;
  a.gate_up = static_cast<const char*>(gate_up);
  a.gu_pitch = gate_up_row_stride * es;
  a.out = static_cast<char*>(out);
  a.out_pitch = out_row_stride * es;
  a.rw = {rw, rw_stride, static_cast<int>(rw_mode), rw_dtype == SITU_DTYPE_BF16 ? 1 : 0};
  a.tokens = tokens;
  a.half_bytes = static_cast<int>(inter * es);
  a.vpr = static_cast<int>(inter * es / kVecBytes);
  a.c = c;
  if (rw_mode == SITU_RW_NONE) a.rw.bf16 = 0;

  FwdKernel k = pick_fwd(dtype, gate, has_linear_beta != 0);
  const int threads = choose_threads(a.vpr);
  int grid = 0;
  st = launch_grid(reinterpret_cast<const void*>(k), threads, tokens, &grid);
  if (st != SITU_OK) return st;
  k<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return check_launch("situ_glu_fwd");
}

size_t situ_glu_bwd_workspace_bytes(int64_t tokens, situ_rw_mode_t rw_mode, int want_drw) {
  if (tokens <= 0 || rw_mode != SITU_RW_SCALAR || !want_drw) return 0;
  const uint64_t bytes = static_cast<uint64_t>(tokens) * sizeof(float);
  return static_cast<size_t>((bytes + 255) / 256 * 256);
}

situ_status_t situ_glu_bwd(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                           int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype,
                           situ_rw_mode_t rw_mode, int64_t rw_stride, double beta, int has_linear_beta,
                           double linear_beta, const void* grad_out, int64_t grad_out_row_stride,
                           void* d_gate_up, int64_t d_gate_up_row_stride, void* d_rw, int64_t d_rw_stride,
                           void* workspace, size_t workspace_bytes, void* stream) {
  tl_last_error[0] = '\0';
  Coeffs c;
  int gate = kGateGeneric;
  situ_status_t st = check_common(dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                  rw_stride, beta, has_linear_beta, linear_beta, &c, &gate);
  if (st != SITU_OK) return st;
  if (grad_out_row_stride < inter) return fail(SITU_ERR_INVALID_ARG, "grad_out_row_stride < inter");
  if (d_gate_up_row_stride < 2 * inter) return fail(SITU_ERR_INVALID_ARG, "d_gate_up_row_stride < 2 * inter");
  if (rw_mode == SITU_RW_NONE && d_rw != nullptr)
    return fail(SITU_ERR_INVALID_ARG, "d_rw must be NULL for SITU_RW_NONE");
  const bool want_drw = d_rw != nullptr;
  if (want_drw && rw_mode == SITU_RW_ROW && d_rw_stride < 1) return fail(SITU_ERR_INVALID_ARG, "d_rw_stride < 1");
  const size_t ws_needed = situ_glu_bwd_workspace_bytes(tokens, rw_mode, want_drw ? 1 : 0);
  if (tokens == 0) {
    // The gradient of a broadcast weight over zero rows is zero; nothing else
    // is written.  That store is the one piece of work an empty call does.
    if (want_drw && rw_mode == SITU_RW_SCALAR) {
      if (!aligned(d_rw, elem_size(rw_dtype))) return fail(SITU_ERR_MISALIGNED, "d_rw not aligned");
      cudaError_t err = cudaMemsetAsync(d_rw, 0, elem_size(rw_dtype), static_cast<cudaStream_t>(stream));
      if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    }
    return SITU_OK;
  }
  if (gate_up == nullptr || grad_out == nullptr || d_gate_up == nullptr)
    return fail(SITU_ERR_INVALID_ARG, "gate_up, grad_out or d_gate_up is NULL");
  const int es = elem_size(dtype);
  const int rw_es = rw_mode == SITU_RW_NONE ? 4 : elem_size(rw_dtype);
  if (!span_fits(tokens, gate_up_row_stride, 2 * inter, es) || !span_fits(tokens, grad_out_row_stride, inter, es) ||
      !span_fits(tokens, d_gate_up_row_stride, 2 * inter, es) ||
      (rw_mode == SITU_RW_ROW && !span_fits(tokens, rw_stride, 1, rw_es)) ||
      (want_drw && rw_mode == SITU_RW_ROW && !span_fits(tokens, d_rw_stride, 1, rw_es)))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  if (!aligned(gate_up, 16) || !aligned(grad_out, 16) || !aligned(d_gate_up, 16) ||
      (gate_up_row_stride * es) % 16 != 0 || (grad_out_row_stride * es) % 16 != 0 ||
      (d_gate_up_row_stride * es) % 16 != 0)
    return fail(SITU_ERR_MISALIGNED, "gate_up/grad_out/d_gate_up base or row pitch not 16-byte aligned");
  if (rw_mode != SITU_RW_NONE && !aligned(rw, rw_es)) return fail(SITU_ERR_MISALIGNED, "rw not aligned");
  if (want_drw && !aligned(d_rw, rw_es)) return fail(SITU_ERR_MISALIGNED, "d_rw not aligned");
  if (ws_needed > 0) {
    if (workspace == nullptr || workspace_bytes < ws_needed)
      return fail(SITU_ERR_INVALID_ARG, "workspace needs %zu bytes, got %zu", ws_needed,
                  workspace == nullptr ? (size_t)0 : workspace_bytes);
    if (!aligned(workspace, 16)) return fail(SITU_ERR_MISALIGNED, "workspace not 16-byte aligned");
  }

  // Aliasing: no output may overlap an input or another output.
  const Span s_gu = matrix_span(gate_up, tokens, gate_up_row_stride, 2 * inter, es);
  const Span s_go = matrix_span(grad_out, tokens, grad_out_row_stride, inter, es);
  const Span s_dgu = matrix_span(d_gate_up, tokens, d_gate_up_row_stride, 2 * inter, es);
  Span s_rw = {0, 0};
  if (rw_mode == SITU_RW_ROW) s_rw = matrix_span(rw, tokens, rw_stride, 1, rw_es);
  if (rw_mode == SITU_RW_SCALAR) s_rw = matrix_span(rw, 1, 1, 1, rw_es);
  if (overlap(s_dgu, s_gu) || overlap(s_dgu, s_go) || overlap(s_dgu, s_rw))
    return fail(SITU_ERR_INVALID_ARG, "d_gate_up overlaps an input");
  Span s_drw = {0, 0};
  if (want_drw) {
    s_drw = rw_mode == SITU_RW_ROW ? matrix_span(d_rw, tokens, d_rw_stride, 1, rw_es)
                                   : matrix_span(d_rw, 1, 1, 1, rw_es);
    if (overlap(s_drw, s_gu) || overlap(s_drw, s_go) || overlap(s_drw, s_rw) || overlap(s_drw, s_dgu))
      return fail(SITU_ERR_INVALID_ARG, "d_rw overlaps another tensor");
  }
  if (ws_needed > 0) {
    const Span s_ws = {reinterpret_cast<uintptr_t>(workspace), reinterpret_cast<uintptr_t>(workspace) + ws_needed};
    if (overlap(s_ws, s_gu) || overlap(s_ws, s_go) || overlap(s_ws, s_rw) || overlap(s_ws, s_dgu) ||
        overlap(s_ws, s_drw))
      return fail(SITU_ERR_INVALID_ARG, "workspace overlaps a tensor");
  }

  BwdArgs a;
  a.gate_up = static_cast<const char*>(gate_up);
  a.gu_pitch = gate_up_row_stride * es;
  a.grad_out = static_cast<const char*>(grad_out);
  a.go_pitch = grad_out_row_stride * es;
  a.d_gate_up = static_cast<char*>(d_gate_up);
  a.dgu_pitch = d_gate_up_row_stride * es;
  a.rw = {rw, rw_stride, static_cast<int>(rw_mode), (rw_mode != SITU_RW_NONE && rw_dtype == SITU_DTYPE_BF16) ? 1 : 0};
  a.d_rw = d_rw;
  a.d_rw_stride = d_rw_stride;
  a.partials = static_cast<float*>(workspace);
  a.want_drw = want_drw ? 1 : 0;
  a.tokens = tokens;
  a.half_bytes = static_cast<int>(inter * es);
  a.vpr = static_cast<int>(inter * es / kVecBytes);
  a.c = c;

  BwdKernel k = pick_bwd(dtype, gate, has_linear_beta != 0);
  const int threads = choose_threads(a.vpr);
  int grid = 0;
  st = launch_grid(reinterpret_cast<const void*>(k), threads, tokens, &grid);
  if (st != SITU_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  k<<<grid, threads, 0, s>>>(a);
  st = check_launch("situ_glu_bwd");
  if (st != SITU_OK) return st;
  if (want_drw && rw_mode == SITU_RW_SCALAR) {
    situ_glu_dw_scalar_finalize_kernel<<<1, kFinalizeThreads, 0, s>>>(a.partials, tokens, d_rw, a.rw.bf16);
    st = check_launch("situ_glu_bwd (scalar d_rw)");
  }
  return st;
}

const char* situ_glu_status_string(situ_status_t status) {
  switch (status) {
    case SITU_OK: return "SITU_OK";
    case SITU_ERR_INVALID_ARG: return "SITU_ERR_INVALID_ARG";
    case SITU_ERR_UNSUPPORTED: return "SITU_ERR_UNSUPPORTED";
    case SITU_ERR_MISALIGNED: return "SITU_ERR_MISALIGNED";
    case SITU_ERR_CUDA: return "SITU_ERR_CUDA";
  }
  return "SITU_ERR_UNKNOWN";
}

const char* situ_glu_last_error(void) { return tl_last_error; }

int situ_glu_abi_version(void) { return SITU_GLU_ABI_VERSION; }

int situ_glu_set_max_ctas(int max_ctas) {
  if (max_ctas < 0) return -1;
  return g_max_ctas.exchange(max_ctas);
}

}  // extern "C"
