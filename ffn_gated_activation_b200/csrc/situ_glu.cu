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

#include <cuda.h>  // CUtensorMap and its encoder's types (the encoder is fetched at run time)
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <initializer_list>
#include <type_traits>

#include "situ_glu.h"

namespace {

// ---------------------------------------------------------------------------
// Device helpers
// ---------------------------------------------------------------------------

constexpr float kLog2e = 1.4426950408889634f;  // log2(e)
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxThreads = 256;  // CTA size ceiling
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

// Hardware tanh (MUFU).  Its relative error (about 2^-11) is far below half a
// bf16 ulp (2^-9 relative), so it is used only where the result is rounded to
// bf16 and nothing is accumulated from it: the up branch of the bf16 forward.
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// max() that propagates NaN (a NaN input must give a NaN output).
__device__ __forceinline__ float max_nan(float a, float b) {
  float r;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
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

// 32-byte forms (sm_100): two adjacent 16-byte vectors in one instruction.
// The address must be 32-byte aligned.
struct U8 {
  uint4 a, b;
};

__device__ __forceinline__ U8 ld_stream32(const void* p) {
  U8 r;
  asm("ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r.a.x), "=r"(r.a.y), "=r"(r.a.z), "=r"(r.a.w), "=r"(r.b.x), "=r"(r.b.y), "=r"(r.b.z), "=r"(r.b.w)
      : "l"(p));
  return r;
}

__device__ __forceinline__ void st_stream32(void* p, const uint4& a, const uint4& b) {
  asm volatile("st.global.cs.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y),
               "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
               : "memory");
}

// Packed fp32 pairs: sm_100 executes one f32x2 add/mul/fma per issue slot.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 splat(float a) { return make_float2(a, a); }

__device__ __forceinline__ float2 ex2_neg2(float2 y) {  // (2^-y.x, 2^-y.y)
  return make_float2(ex2_approx(-y.x), ex2_approx(-y.y));
}
__device__ __forceinline__ float2 rcp2(float2 a) { return make_float2(rcp_approx(a.x), rcp_approx(a.y)); }

// A pair of input elements as fp32 bit patterns (bf16 widened exactly).
struct Bits2 {
  uint32_t lo, hi;
};

__device__ __forceinline__ float2 as_f2(Bits2 b) { return make_float2(__uint_as_float(b.lo), __uint_as_float(b.hi)); }
__device__ __forceinline__ float2 abs_f2(Bits2 b) {
  return make_float2(__uint_as_float(b.lo & 0x7fffffffu), __uint_as_float(b.hi & 0x7fffffffu));
}
// x with its sign bit flipped where the sign bit of `s` is set.
__device__ __forceinline__ float xor_sign(float x, uint32_t s) {
  return __uint_as_float(__float_as_uint(x) ^ (s & 0x80000000u));
}
__device__ __forceinline__ float2 xor_sign2(float2 x, Bits2 s) { return make_float2(xor_sign(x.x, s.lo), xor_sign(x.y, s.hi)); }
// s negative ? a : b, element-wise on the sign bit of s.
__device__ __forceinline__ float2 select_neg2(Bits2 s, float2 a, float2 b) {
  const uint32_t m0 = static_cast<uint32_t>(static_cast<int32_t>(s.lo) >> 31);
  const uint32_t m1 = static_cast<uint32_t>(static_cast<int32_t>(s.hi) >> 31);
  return make_float2(__uint_as_float((__float_as_uint(a.x) & m0) | (__float_as_uint(b.x) & ~m0)),
                     __uint_as_float((__float_as_uint(a.y) & m1) | (__float_as_uint(b.y) & ~m1)));
}

// Storage types.  A 16-byte vector holds 8 bf16 or 4 fp32 values, i.e. 4 or 2
// pairs.  Pair p of a vector is (element 2p, element 2p + 1).
struct Bf16 {
  static constexpr int kPairs = 4;
  __device__ __forceinline__ static Bits2 pair(const uint4& v, int p) {
    const uint32_t w = p == 0 ? v.x : p == 1 ? v.y : p == 2 ? v.z : v.w;
    return {w << 16, w & 0xffff0000u};
  }
  __device__ __forceinline__ static uint32_t pack(float2 f) {
    uint32_t r;  // cvt packs its first source into the high half
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(f.y), "f"(f.x));
    return r;
  }
  __device__ __forceinline__ static void put(uint4& v, int p, float2 f) {
    const uint32_t w = pack(f);
    if (p == 0) v.x = w; else if (p == 1) v.y = w; else if (p == 2) v.z = w; else v.w = w;
  }
};

struct F32 {
  static constexpr int kPairs = 2;
  __device__ __forceinline__ static Bits2 pair(const uint4& v, int p) {
    return p == 0 ? Bits2{v.x, v.y} : Bits2{v.z, v.w};
  }
  __device__ __forceinline__ static void put(uint4& v, int p, float2 f) {
    if (p == 0) {
      v.x = __float_as_uint(f.x);
      v.y = __float_as_uint(f.y);
    } else {
      v.z = __float_as_uint(f.x);
      v.w = __float_as_uint(f.y);
    }
  }
};

// 1 - 2^-y, given E = 2^-y from the MUFU.  Where |y| is small, 1 - E cancels;
// there the Taylor series of 1 - exp(-x) in x = y ln 2 is used, written in y:
//   sum_k (-1)^(k+1) (ln 2)^k y^k / k!.
// bf16 outputs: terms to y^4 for |x| < 1/16 (truncation below 2^-22 relative;
// 1 - E above it within about 2^-19).  fp32 outputs: terms to y^6 for
// |x| < 1/4 (truncation below 2^-24; 1 - E above it within about 2^-21).
// Valid for either sign of y.
template <typename S>
struct Series;

template <>
struct Series<Bf16> {
  static constexpr float kYmax = 0.0625f / kLn2;
  __device__ __forceinline__ static float2 eval(float2 y) {
    const float c1 = kLn2, c2 = -kLn2 * kLn2 / 2.0f, c3 = kLn2 * kLn2 * kLn2 / 6.0f,
                c4 = -kLn2 * kLn2 * kLn2 * kLn2 / 24.0f;
    float2 p = fma2(y, splat(c4), splat(c3));
    p = fma2(p, y, splat(c2));
    p = fma2(p, y, splat(c1));
    return mul2(p, y);
  }
};

template <>
struct Series<F32> {
  static constexpr float kYmax = 0.25f / kLn2;
  __device__ __forceinline__ static float2 eval(float2 y) {
    const float l = kLn2;
    const float c1 = l, c2 = -l * l / 2.0f, c3 = l * l * l / 6.0f, c4 = -l * l * l * l / 24.0f,
                c5 = l * l * l * l * l / 120.0f, c6 = -l * l * l * l * l * l / 720.0f;
    float2 p = fma2(y, splat(c6), splat(c5));
    p = fma2(p, y, splat(c4));
    p = fma2(p, y, splat(c3));
    p = fma2(p, y, splat(c2));
    p = fma2(p, y, splat(c1));
    return mul2(p, y);
  }
};

// The bf16 backward's up branch feeds T_u only as a relative factor (dG within
// 2^-8, d_w as a sum of terms with independent rounding), so terms to y^3 for
// |x| < 1/32 suffice there (truncation below 2^-19.6; 1 - E above it within
// about 2^-18).
struct SeriesBf16Up {
  static constexpr float kYmax = 0.03125f / kLn2;
  __device__ __forceinline__ static float2 eval(float2 y) {
    const float c1 = kLn2, c2 = -kLn2 * kLn2 / 2.0f, c3 = kLn2 * kLn2 * kLn2 / 6.0f;
    float2 p = fma2(y, splat(c3), splat(c2));
    p = fma2(p, y, splat(c1));
    return mul2(p, y);
  }
};

// Series used for the backward's up branch, per storage type.
template <typename S>
struct UpSeries {
  using type = Series<S>;
};
template <>
struct UpSeries<Bf16> {
  using type = SeriesBf16Up;
};

template <typename S, typename P = Series<S>>
__device__ __forceinline__ float2 one_minus_exp2_neg(float2 y, float2 E) {
  const float2 series = P::eval(y);
  const float2 direct = fma2(E, splat(-1.0f), splat(1.0f));
  return make_float2(fabsf(y.x) < P::kYmax ? series.x : direct.x, fabsf(y.y) < P::kYmax ? series.y : direct.y);
}

// How the two gate exponentials relate for the given beta.
enum GateMode : int {
  kGateGeneric = 0,  // two independent exponentials
  kGateSquare = 1,   // beta = 4: E_s = E_t^2
  kGateEqual = 2,    // beta = 2: E_s = E_t
  kGateRoot = 3,     // beta = 1: E_t = E_s^2
};

struct Coeffs {
  float beta;    // gate beta
  float lb;      // linear beta (1 without one)
  float inv_lb;  // 1 / linear beta
  float kt;      // 2 log2(e) / beta:    E_t = 2^-(|g| kt)
  float ku;      // 2 log2(e) / beta_L:  E_u = 2^-(|u| ku)
  float bb;      // beta * beta_L (beta without a linear beta)
};

// Exponentials of the gate: E_t = 2^-y with y = |g| kt (or g kt, signed form)
// and E_s = exp(-|g|) (exp(-g)).  `y` must already hold the scaled argument.
template <int GATE>
__device__ __forceinline__ void gate_exps(float2 y, float2& Et, float2& Es) {
  if (GATE == kGateSquare) {
    Et = ex2_neg2(y);
    Es = mul2(Et, Et);
  } else if (GATE == kGateEqual) {
    Et = ex2_neg2(y);
    Es = Et;
  } else if (GATE == kGateRoot) {  // kt = 2 log2(e): E_s = 2^-(y/2), E_t = E_s^2
    Es = ex2_neg2(mul2(y, splat(0.5f)));
    Et = mul2(Es, Es);
  } else {
    Et = ex2_neg2(y);
    Es = make_float2(0.0f, 0.0f);  // set by the caller from its own argument
  }
}

// ---- forward, bf16 storage ------------------------------------------------
// Signed form: with H = exp(-2g/beta) and Hs = exp(-g) (g of either sign),
//   tanh(g/beta) = (1 - H) / (1 + H),  sigmoid(g) = 1 / (1 + Hs),
//   T_g = beta (1 - H) / ((1 + H)(1 + Hs)),
// so neither a sign select nor |g| is needed.  The exponent argument is
// clamped at 2^126 (a NaN passes through); when (1 + H)(1 + Hs) overflows the
// reciprocal is 0 and T_g flushes to 0, which happens only where
// |T_g| < 4 exp(-59) -- below the bf16 output's absolute resolution of the
// tolerance.  The up branch uses the MUFU tanh (see tanh_approx).
template <int GATE, bool HAS_LB>
__device__ __forceinline__ float2 fwd_pair_bf16(Bits2 gb, Bits2 ub, float2 wbb, const Coeffs& c) {
  const float2 g = as_f2(gb);
  float2 y = mul2(g, splat(c.kt));
  y = make_float2(max_nan(y.x, -126.0f), max_nan(y.y, -126.0f));
  float2 H, Hs;
  gate_exps<GATE>(y, H, Hs);
  if (GATE == kGateGeneric) {
    float2 ys = mul2(g, splat(kLog2e));
    Hs = ex2_neg2(make_float2(max_nan(ys.x, -126.0f), max_nan(ys.y, -126.0f)));
  }
  const float2 em = one_minus_exp2_neg<Bf16>(y, H);
  const float2 den = mul2(add2(splat(1.0f), H), add2(splat(1.0f), Hs));
  float2 t;  // T_u / beta_L (or U)
  if (HAS_LB) {
    const float2 a = mul2(as_f2(ub), splat(c.inv_lb));
    t = make_float2(tanh_approx(a.x), tanh_approx(a.y));
  } else {
    t = as_f2(ub);
  }
  // em / den = T_g / beta lies in [-1, 1]: form it first so that a huge |1 - H|
  // meets its zero reciprocal before it can meet a large U.
  return mul2(mul2(em, rcp2(den)), mul2(t, wbb));
}

// ---- |g| form (fp32 forward and every backward) ---------------------------
// E_t = exp(-2|g|/beta) <= 1 and E_s = exp(-|g|) <= 1, so no intermediate can
// overflow; the sign of g enters through selects and sign flips.
struct GateAbs {
  float2 Et, Es, emt;  // emt = 1 - Et, accurate
};

template <int GATE, typename S>
__device__ __forceinline__ GateAbs gate_abs(Bits2 gb, const Coeffs& c) {
  const float2 ag = abs_f2(gb);
  const float2 y = mul2(ag, splat(c.kt));
  GateAbs r;
  gate_exps<GATE>(y, r.Et, r.Es);
  if (GATE == kGateGeneric) r.Es = ex2_neg2(mul2(ag, splat(kLog2e)));
  r.emt = one_minus_exp2_neg<S>(y, r.Et);
  return r;
}

template <typename S, typename P = Series<S>>
__device__ __forceinline__ float2 up_emu(Bits2 ub, const Coeffs& c, float2& Eu) {
  const float2 y = mul2(abs_f2(ub), splat(c.ku));
  Eu = ex2_neg2(y);
  return one_minus_exp2_neg<S, P>(y, Eu);
}

// fp32 forward of a pair.  Y = w beta beta_L s_g s_u (1 - E_t) sig (1 - E_u)
// / ((1 + E_t)(1 + E_s)(1 + E_u)), sig = 1 (g >= 0) or E_s (g < 0).
template <int GATE, bool HAS_LB, typename S>
__device__ __forceinline__ float2 fwd_pair_abs(Bits2 gb, Bits2 ub, float2 wbb, const Coeffs& c) {
  const GateAbs e = gate_abs<GATE, S>(gb, c);
  const float2 sig = select_neg2(gb, e.Es, splat(1.0f));
  float2 num = mul2(e.emt, sig);
  float2 den = mul2(add2(splat(1.0f), e.Et), add2(splat(1.0f), e.Es));
  if (HAS_LB) {
    float2 Eu;
    const float2 emu = up_emu<S>(ub, c, Eu);
    num = mul2(num, emu);
    den = mul2(den, add2(splat(1.0f), Eu));
    // sign of the product: s_g s_u
    const Bits2 s = {gb.lo ^ ub.lo, gb.hi ^ ub.hi};
    return xor_sign2(mul2(num, mul2(rcp2(den), wbb)), s);
  }
  num = mul2(num, abs_f2(ub));
  const Bits2 s = {gb.lo ^ ub.lo, gb.hi ^ ub.hi};
  return xor_sign2(mul2(num, mul2(rcp2(den), wbb)), s);
}

// Whether the backward of a pair takes the signed gate form: beta = 4, bf16
// dG and dU, and a caller whose every output derived from them tolerates the
// clamp below (CLAMPED): the native-output kernels and the per-column-weight
// backward, whose bf16 gradients carry an absolute tolerance far above the
// clamped values and whose weight gradients are sums.  Outputs that keep
// relative accuracy for tiny values -- block-scaled codes, whose scale
// follows the block, and per-element weight gradients -- take the |g| form
// (the block-scaled backward takes the signed form without the clamp where a
// warp vote shows it idle).  Measured on B200: 5 % less time for the bf16
// backward, 5-6 % for the per-column one.
template <int GATE, typename S, bool CLAMPED>
struct SignedBwd {
  static constexpr bool value = CLAMPED && GATE == kGateSquare && std::is_same<S, Bf16>::value;
};

// Backward of a pair.  With A = (1 + E_t)(1 + E_s), B = 1 + E_u (1 without a
// linear beta), sig as above and
//   tq  = (beta/4) tanh(g/beta) (1 + E_t)              (= (beta/4) s_g (1 - E_t))
//   T_g  = 4 tq sig / A  (tgA = tq sig A = T_g A^2 / 4)
//   T_g' = 4 [E_t sig (1 + E_s) + tq (1 + E_t) E_s] / A^2
//          (the sech^2(g/beta) sigmoid and beta tanh sigmoid (1 - sigmoid) terms)
//   T_u  = beta_L su / B,  su = s_u (1 - E_u),   T_u' = 4 E_u / B^2
// one reciprocal R = 1 / (A B)^2 serves every quotient.  The per-row factors
// are folded into two constants: k.x = 4 beta_L w (dG) and k.y = 16 w (dU);
// the d_w terms are accumulated without their factor 4 beta_L, which the
// caller applies once per row.  Returns dG, dU; adds go T_g T_u / (4 beta_L)
// to acc.
// The signed backward's clamp applied to packed bf16 gate values: g >= -27.75
// (a bf16 number; y = g kt >= -20.02 for beta = 4), NaN kept, one
// instruction per pair of elements.
__device__ __forceinline__ uint4 clamp_gate_bf16x8(uint4 v) {
  const uint32_t lo = 0xC1DEC1DEu;  // -27.75 in both halves
  asm("max.NaN.bf16x2 %0, %0, %4;\n\tmax.NaN.bf16x2 %1, %1, %4;\n\t"
      "max.NaN.bf16x2 %2, %2, %4;\n\tmax.NaN.bf16x2 %3, %3, %4;"
      : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
      : "r"(lo));
  return v;
}

template <int GATE, bool HAS_LB, typename S, bool CLAMPED = false, bool PRECLAMPED = false>
__device__ __forceinline__ void bwd_pair(Bits2 gb, Bits2 ub, float2 go, float2 kdg, float2 kdu, const Coeffs& c,
                                         float2& dg, float2& du, float2& acc) {
  float2 A, tgA, ng;
  if constexpr (SignedBwd<GATE, S, CLAMPED>::value) {
    // Signed form (beta = 4, bf16 outputs), as in the bf16 forward: with
    // H = exp(-g/2) and Hs = H^2 = exp(-g) for g of either sign,
    //   T_g  = 4 (1 - H) / A,                 A = (1 + H)(1 + Hs),
    //   T_g' = 4 [H (1 + Hs) + (1 - H)(1 + H) Hs] / A^2,
    // so no |g|, sign flip or select is needed.  The exponent argument is
    // clamped at 20 (g >= -27.7: H <= 2^20, A <= 2^60, (A B)^2 <= 2^122), where
    // |T_g| < 4e-12 and |T_g'| < 1e-11: far below a bf16 output's absolute
    // resolution of the tolerance.  PRECLAMPED: the caller clamped the packed
    // bf16 gate values at -27.75 instead (y >= -20.02, (A B)^2 <= 2^122.1).
    float2 y = mul2(as_f2(gb), splat(c.kt));
    if constexpr (!PRECLAMPED) y = make_float2(max_nan(y.x, -20.0f), max_nan(y.y, -20.0f));
    const float2 H = ex2_neg2(y), Hs = mul2(H, H);
    // 1 - H: below |x| = 1/32 from the series to x^3 (truncation under
    // 2^-19.6), above it 1 - H (MUFU error under 2^-17 relative there): both
    // far below what a bf16 output and a per-row sum of terms need.
    const float2 em = one_minus_exp2_neg<S, SeriesBf16Up>(y, H);
    const float2 opH = add2(splat(1.0f), H), opHs = add2(splat(1.0f), Hs);
    A = mul2(opH, opHs);
    tgA = mul2(em, A);                                // T_g A^2 / 4
    ng = fma2(H, opHs, mul2(mul2(em, opH), Hs));      // T_g' A^2 / 4
  } else {
    const GateAbs e = gate_abs<GATE, S>(gb, c);
    const float2 sig = select_neg2(gb, e.Es, splat(1.0f));
    const float2 opt = add2(splat(1.0f), e.Et), ops = add2(splat(1.0f), e.Es);
    A = mul2(opt, ops);
    float2 tq = xor_sign2(e.emt, gb);
    if (GATE != kGateSquare) tq = mul2(tq, splat(0.25f * c.beta));  // beta = 4: the factor is 1
    tgA = mul2(mul2(tq, sig), A);                                    // T_g A^2 / 4
    ng = fma2(mul2(e.Et, sig), ops, mul2(mul2(tq, opt), e.Es));      // T_g' A^2 / 4
  }
  if (HAS_LB) {
    float2 Eu;
    const float2 su = xor_sign2(up_emu<S, typename UpSeries<S>::type>(ub, c, Eu), ub);  // T_u B / beta_L
    const float2 B = add2(splat(1.0f), Eu);
    const float2 AB = mul2(A, B);
    const float2 gR = mul2(go, rcp2(mul2(AB, AB)));  // go / (A B)^2
    const float2 sB = mul2(su, B);
    const float2 gRt = mul2(gR, tgA);
    dg = mul2(mul2(gR, kdg), mul2(sB, ng));  // go w T_u T_g'
    du = mul2(gRt, mul2(Eu, kdu));           // go w T_g T_u'
    acc = fma2(gRt, sB, acc);                // go T_g T_u / (4 beta_L)
  } else {
    const float2 u = as_f2(ub);
    const float2 gR = mul2(go, rcp2(mul2(A, A)));  // go / A^2
    const float2 gRt = mul2(gR, tgA);
    dg = mul2(mul2(gR, kdg), mul2(u, ng));
    du = mul2(gRt, kdu);
    acc = fma2(gRt, u, acc);
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
// One CTA works on one row at a time and strides over rows.  Thread t handles
// the 16-byte vectors t, t + nt, t + 2 nt, ... of each half row, two at a time
// (both loads are issued before any arithmetic), so each thread keeps two
// vectors of every input in flight.

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
__device__ __forceinline__ uint4 fwd_vec(const uint4& gv, const uint4& uv, float2 wbb, const Coeffs& c) {
  uint4 o;
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) {
    float2 y;
    if constexpr (std::is_same<S, Bf16>::value)
      y = fwd_pair_bf16<GATE, HAS_LB>(S::pair(gv, p), S::pair(uv, p), wbb, c);
    else
      y = fwd_pair_abs<GATE, HAS_LB, S>(S::pair(gv, p), S::pair(uv, p), wbb, c);
    S::put(o, p, y);
  }
  return o;
}

// Whether a direct-load kernel loads the CTA's next row while it computes the
// current one (measured on B200: faster for every forward and the bf16
// backward, slower for the fp32 backward, whose extra registers cost more
// occupancy than the overlap gains).
template <typename S, bool BWD>
struct PipelineRows {
  static constexpr bool value = !BWD || std::is_same<S, Bf16>::value;
};
// Register budgets of the direct-load kernels (registers per thread); unset
// leaves the choice to the compiler.
#ifdef SITU_FWD_MAXNREG
#define SITU_FWD_BOUNDS __maxnreg__(SITU_FWD_MAXNREG)
#else
#define SITU_FWD_BOUNDS __launch_bounds__(kMaxThreads)
#endif
#ifdef SITU_BWD_MAXNREG
#define SITU_BWD_BOUNDS __maxnreg__(SITU_BWD_MAXNREG)
#else
#define SITU_BWD_BOUNDS __launch_bounds__(kMaxThreads)
#endif

template <typename S, int GATE, bool HAS_LB>
__global__ void SITU_FWD_BOUNDS situ_glu_fwd_kernel(const FwdArgs a) {
  const int nt = blockDim.x;
  if (PipelineRows<S, false>::value && a.vpr <= 2 * nt) {
    // Each thread owns vectors j and j + nt of every row it visits: load the
    // CTA's next row while computing the current one, so that loads stay in
    // flight during the arithmetic.
    const int j = threadIdx.x, j2 = j + nt;
    const bool one = j < a.vpr, two = j2 < a.vpr;
    int64_t row = blockIdx.x;
    if (row >= a.tokens) return;
    const uint4 z = make_uint4(0, 0, 0, 0);
    uint4 g0 = z, u0 = z, g1 = z, u1 = z;
    const char* gu = a.gate_up + row * a.gu_pitch;
    if (one) {
      g0 = ld_stream(gu + j * kVecBytes);
      u0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
    }
    if (two) {
      g1 = ld_stream(gu + j2 * kVecBytes);
      u1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
    }
    float w = load_rw(a.rw, row);
    for (;;) {
      const int64_t next = row + gridDim.x;
      const bool more = next < a.tokens;
      uint4 ng0, nu0, ng1, nu1;  // only the lanes' own vectors are loaded and used
      float nw = 0.0f;
      if (more) {
        const char* ngu = a.gate_up + next * a.gu_pitch;
        if (one) {
          ng0 = ld_stream(ngu + j * kVecBytes);
          nu0 = ld_stream(ngu + a.half_bytes + j * kVecBytes);
        }
        if (two) {
          ng1 = ld_stream(ngu + j2 * kVecBytes);
          nu1 = ld_stream(ngu + a.half_bytes + j2 * kVecBytes);
        }
        nw = load_rw(a.rw, next);
      }
      char* out = a.out + row * a.out_pitch;
      const float2 wbb = splat(w * a.c.bb);
      if (one) st_stream(out + j * kVecBytes, fwd_vec<S, GATE, HAS_LB>(g0, u0, wbb, a.c));
      if (two) st_stream(out + j2 * kVecBytes, fwd_vec<S, GATE, HAS_LB>(g1, u1, wbb, a.c));
      if (!more) break;
      row = next;
      g0 = ng0; u0 = nu0; g1 = ng1; u1 = nu1; w = nw;
    }
    return;
  }
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    const char* gu = a.gate_up + row * a.gu_pitch;
    char* out = a.out + row * a.out_pitch;
    const float2 wbb = splat(load_rw(a.rw, row) * a.c.bb);
    for (int j = threadIdx.x; j < a.vpr; j += 2 * nt) {
      const int j2 = j + nt;
      const bool two = j2 < a.vpr;
      const uint4 g0 = ld_stream(gu + j * kVecBytes);
      const uint4 u0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
      uint4 g1 = make_uint4(0, 0, 0, 0), u1 = g1;
      if (two) {
        g1 = ld_stream(gu + j2 * kVecBytes);
        u1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
      }
      st_stream(out + j * kVecBytes, fwd_vec<S, GATE, HAS_LB>(g0, u0, wbb, a.c));
      if (two) st_stream(out + j2 * kVecBytes, fwd_vec<S, GATE, HAS_LB>(g1, u1, wbb, a.c));
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

// Per-row constants of the backward: k.x = 4 beta_L w (dG); k.y = 16 w (dU:
// 4 from T_g, 4 from T_u' = 4 E_u / B^2), or 4 w without a linear beta
// (T_u' = 1); and the d_w scale 4 beta_L (beta_L = 1 without a linear beta).
template <bool HAS_LB>
__device__ __forceinline__ float2 bwd_row_consts(float w, const Coeffs& c) {
  return make_float2(4.0f * c.lb * w, (HAS_LB ? 16.0f : 4.0f) * w);
}
__device__ __forceinline__ float bwd_dw_scale(const Coeffs& c) { return 4.0f * c.lb; }

template <typename S, int GATE, bool HAS_LB>
__device__ __forceinline__ void bwd_vec(const uint4& gv, const uint4& uv, const uint4& gov, float2 k,
                                        const Coeffs& c, uint4& dgv, uint4& duv, float2& acc) {
  const float2 kdg = splat(k.x), kdu = splat(k.y);
  constexpr bool kPre = SignedBwd<GATE, S, true>::value;  // clamp the packed gate values, one instruction a pair
  const uint4 gc = kPre ? clamp_gate_bf16x8(gv) : gv;
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) {
    float2 dg, du;
    bwd_pair<GATE, HAS_LB, S, true, kPre>(S::pair(gc, p), S::pair(uv, p), as_f2(S::pair(gov, p)), kdg, kdu, c, dg,
                                          du, acc);
    S::put(dgv, p, dg);
    S::put(duv, p, du);
  }
}

template <typename S, int GATE, bool HAS_LB>
__global__ void SITU_BWD_BOUNDS situ_glu_bwd_kernel(const BwdArgs a) {
  __shared__ float red[2][kMaxThreads / 32];
  const int nt = blockDim.x;
  int parity = 0;
  if (PipelineRows<S, true>::value && a.vpr <= 2 * nt) {
    // As in the forward: the CTA's next row is loaded while this one computes.
    const int j = threadIdx.x, j2 = j + nt;
    const bool one = j < a.vpr, two = j2 < a.vpr;
    int64_t row = blockIdx.x;
    if (row >= a.tokens) return;
    const uint4 z = make_uint4(0, 0, 0, 0);
    uint4 g0 = z, u0 = z, o0 = z, g1 = z, u1 = z, o1 = z;
    {
      const char* gu = a.gate_up + row * a.gu_pitch;
      const char* go_row = a.grad_out + row * a.go_pitch;
      if (one) {
        g0 = ld_stream(gu + j * kVecBytes);
        u0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
        o0 = ld_stream(go_row + j * kVecBytes);
      }
      if (two) {
        g1 = ld_stream(gu + j2 * kVecBytes);
        u1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
        o1 = ld_stream(go_row + j2 * kVecBytes);
      }
    }
    float w = load_rw(a.rw, row);
    for (;;) {
      const int64_t next = row + gridDim.x;
      const bool more = next < a.tokens;
      uint4 ng0, nu0, no0, ng1, nu1, no1;  // only the lanes' own vectors are loaded and used
      float nw = 0.0f;
      if (more) {
        const char* gu = a.gate_up + next * a.gu_pitch;
        const char* go_row = a.grad_out + next * a.go_pitch;
        if (one) {
          ng0 = ld_stream(gu + j * kVecBytes);
          nu0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
          no0 = ld_stream(go_row + j * kVecBytes);
        }
        if (two) {
          ng1 = ld_stream(gu + j2 * kVecBytes);
          nu1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
          no1 = ld_stream(go_row + j2 * kVecBytes);
        }
        nw = load_rw(a.rw, next);
      }
      char* dgu = a.d_gate_up + row * a.dgu_pitch;
      const float2 k = bwd_row_consts<HAS_LB>(w, a.c);
      float2 acc = make_float2(0.0f, 0.0f);
      uint4 dg, du;
      if (one) {
        bwd_vec<S, GATE, HAS_LB>(g0, u0, o0, k, a.c, dg, du, acc);
        st_stream(dgu + j * kVecBytes, dg);
        st_stream(dgu + a.half_bytes + j * kVecBytes, du);
      }
      if (two) {
        bwd_vec<S, GATE, HAS_LB>(g1, u1, o1, k, a.c, dg, du, acc);
        st_stream(dgu + j2 * kVecBytes, dg);
        st_stream(dgu + a.half_bytes + j2 * kVecBytes, du);
      }
      if (a.want_drw) {  // uniform over the launch
        const float total = block_sum(acc.x + acc.y, red[parity]) * bwd_dw_scale(a.c);
        parity ^= 1;
        if (threadIdx.x == 0) {
          if (a.rw.mode == SITU_RW_SCALAR)
            a.partials[row] = total;
          else
            store_rw_grad(a.d_rw, row * a.d_rw_stride, a.rw.bf16, total);
        }
      }
      if (!more) break;
      row = next;
      g0 = ng0; u0 = nu0; o0 = no0; g1 = ng1; u1 = nu1; o1 = no1; w = nw;
    }
    return;
  }
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    const char* gu = a.gate_up + row * a.gu_pitch;
    const char* go_row = a.grad_out + row * a.go_pitch;
    char* dgu = a.d_gate_up + row * a.dgu_pitch;
    const float2 k = bwd_row_consts<HAS_LB>(load_rw(a.rw, row), a.c);
    float2 acc = make_float2(0.0f, 0.0f);
    for (int j = threadIdx.x; j < a.vpr; j += 2 * nt) {
      const int j2 = j + nt;
      const bool two = j2 < a.vpr;
      const uint4 g0 = ld_stream(gu + j * kVecBytes);
      const uint4 u0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
      const uint4 o0 = ld_stream(go_row + j * kVecBytes);
      uint4 g1 = make_uint4(0, 0, 0, 0), u1 = g1, o1 = g1;
      if (two) {
        g1 = ld_stream(gu + j2 * kVecBytes);
        u1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
        o1 = ld_stream(go_row + j2 * kVecBytes);
      }
      uint4 dg, du;
      bwd_vec<S, GATE, HAS_LB>(g0, u0, o0, k, a.c, dg, du, acc);
      st_stream(dgu + j * kVecBytes, dg);
      st_stream(dgu + a.half_bytes + j * kVecBytes, du);
      if (two) {  // zero inputs contribute exactly 0 to acc, but skip them anyway
        bwd_vec<S, GATE, HAS_LB>(g1, u1, o1, k, a.c, dg, du, acc);
        st_stream(dgu + j2 * kVecBytes, dg);
        st_stream(dgu + a.half_bytes + j2 * kVecBytes, du);
      }
    }
    if (a.want_drw) {  // uniform over the launch
      const float total = block_sum(acc.x + acc.y, red[parity]) * bwd_dw_scale(a.c);
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
// Element-wise routing weights: one per column ([I]) or per element ([T, I])
// ---------------------------------------------------------------------------
// The weight of element (r, i) enters the same pair arithmetic as a per-pair
// factor.  The [T, I] gradient is the term go T_g T_u itself; the [I] gradient
// sums it over rows.  The rows are cut into chunks of kColChunk (chunk k holds
// rows [k kColChunk, (k + 1) kColChunk)); a CTA takes chunks blockIdx.x,
// blockIdx.x + gridDim.x, ...; each thread adds the terms of its own columns
// in row order and writes the chunk's column sums to workspace row k; a second
// kernel adds the chunks in order.  Both orders are fixed by the shape alone,
// so the results do not depend on the grid.  Small chunks keep the CTAs evenly
// loaded; the partial sums cost 8 I bytes of traffic per chunk against the
// 10 I bytes (bf16) every row moves.
//
// As in the per-row kernels, a thread owns vectors j and j + blockDim.x of
// each row and loads the CTA's next row while it computes this one.  The
// column sums then live in registers; the looped form (rows wider than two
// vectors per thread) keeps them in shared memory.

constexpr int kColChunk = 16;
constexpr int kMaxColInter = 16384;  // column sums of the looped form live in shared memory

struct EwArgs {
  const char* gate_up;
  int64_t gu_pitch;  // bytes
  const char* grad_out;  // backward only
  int64_t go_pitch;
  char* out;  // forward: Y; backward: d_gate_up
  int64_t out_pitch;
  const char* rw;
  int64_t rw_pitch;  // bytes between rows of a [T, I] weight (0 for [I])
  char* d_rw;        // backward: gradient shaped like rw (NULL: not wanted)
  int64_t d_rw_pitch;
  float* partials;   // backward, [I] weights: [ceil(T / kColChunk)][inter]
  int rw_bf16;
  int64_t tokens;
  int half_bytes;
  int vpr;
  int inter;
  Coeffs c;
};

__device__ __forceinline__ uint2 ld_stream8(const void* p) {
  uint2 r;
  asm("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

__device__ __forceinline__ void st_stream8(void* p, const uint2& v) {
  asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t q) {
  return make_float2(__uint_as_float(q << 16), __uint_as_float(q & 0xffff0000u));
}

// The kPairs weight pairs of vector j (elements 2 kPairs j ...) from `w_row`:
// 8 or 16 bytes of bf16, 16 or 32 bytes of fp32.
template <typename S>
__device__ __forceinline__ void load_w_pairs(const char* w_row, int j, int bf16, float2 (&w)[S::kPairs]) {
  constexpr int kElems = 2 * S::kPairs;
  if (bf16) {
    const char* p = w_row + j * kElems * 2;
    if constexpr (kElems == 8) {
      const uint4 v = ld_stream(p);
      w[0] = bf16x2_to_f2(v.x); w[1] = bf16x2_to_f2(v.y); w[2] = bf16x2_to_f2(v.z); w[3] = bf16x2_to_f2(v.w);
    } else {
      const uint2 v = ld_stream8(p);
      w[0] = bf16x2_to_f2(v.x); w[1] = bf16x2_to_f2(v.y);
    }
  } else {
    const char* p = w_row + j * kElems * 4;
#pragma unroll
    for (int k = 0; k < S::kPairs / 2; ++k) {
      const uint4 v = ld_stream(p + 16 * k);
      w[2 * k] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
      w[2 * k + 1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
    }
  }
}

template <typename S>
__device__ __forceinline__ void store_w_pairs(char* d_row, int j, int bf16, const float2 (&d)[S::kPairs]) {
  constexpr int kElems = 2 * S::kPairs;
  if (bf16) {
    char* p = d_row + j * kElems * 2;
    if constexpr (kElems == 8)
      st_stream(p, make_uint4(Bf16::pack(d[0]), Bf16::pack(d[1]), Bf16::pack(d[2]), Bf16::pack(d[3])));
    else
      st_stream8(p, make_uint2(Bf16::pack(d[0]), Bf16::pack(d[1])));
  } else {
    char* p = d_row + j * kElems * 4;
#pragma unroll
    for (int k = 0; k < S::kPairs / 2; ++k)
      st_stream(p + 16 * k, make_uint4(__float_as_uint(d[2 * k].x), __float_as_uint(d[2 * k].y),
                                       __float_as_uint(d[2 * k + 1].x), __float_as_uint(d[2 * k + 1].y)));
  }
}

// One 16-byte vector of Y with per-element weights w.
template <typename S, int GATE, bool HAS_LB>
__device__ __forceinline__ uint4 ew_fwd_vec(const uint4& gv, const uint4& uv, const float2 (&w)[S::kPairs],
                                            const Coeffs& c) {
  uint4 o;
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) {
    const float2 wbb = mul2(w[p], splat(c.bb));
    float2 y;
    if constexpr (std::is_same<S, Bf16>::value)
      y = fwd_pair_bf16<GATE, HAS_LB>(S::pair(gv, p), S::pair(uv, p), wbb, c);
    else
      y = fwd_pair_abs<GATE, HAS_LB, S>(S::pair(gv, p), S::pair(uv, p), wbb, c);
    S::put(o, p, y);
  }
  return o;
}

// One 16-byte vector of dG and dU with per-element weights w; t receives the
// weight-gradient terms go T_g T_u.  CLAMPED: every weight gradient built from
// t is a column sum (per-column weights), so the clamped signed form serves;
// per-element weight gradients keep the |g| form.
template <typename S, int GATE, bool HAS_LB, bool CLAMPED>
__device__ __forceinline__ void ew_bwd_vec(const uint4& gv, const uint4& uv, const uint4& ov,
                                           const float2 (&w)[S::kPairs], const Coeffs& c, uint4& dgv, uint4& duv,
                                           float2 (&t)[S::kPairs]) {
  const float kdg = 4.0f * c.lb, kdu = HAS_LB ? 16.0f : 4.0f;
  const float dws = bwd_dw_scale(c);
  constexpr bool kPre = SignedBwd<GATE, S, CLAMPED>::value;  // clamp the packed gate values, one instruction a pair
  const uint4 gc = kPre ? clamp_gate_bf16x8(gv) : gv;
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) {
    float2 dg, du, acc = make_float2(0.0f, 0.0f);
    bwd_pair<GATE, HAS_LB, S, CLAMPED, kPre>(S::pair(gc, p), S::pair(uv, p), as_f2(S::pair(ov, p)),
                                             mul2(w[p], splat(kdg)), mul2(w[p], splat(kdu)), c, dg, du, acc);
    t[p] = mul2(acc, splat(dws));
    S::put(dgv, p, dg);
    S::put(duv, p, du);
  }
}

template <typename S>
__device__ __forceinline__ void add_pairs(float2 (&s)[S::kPairs], const float2 (&t)[S::kPairs]) {
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) s[p] = add2(s[p], t[p]);
}

template <typename S>
__device__ __forceinline__ void zero_pairs(float2 (&s)[S::kPairs]) {
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) s[p] = make_float2(0.0f, 0.0f);
}

// Column sums of vector j (kElems floats) to workspace row `chunk`.
template <typename S>
__device__ __forceinline__ void store_col_partials(float* partials, int64_t chunk, int inter, int j,
                                                   const float2 (&s)[S::kPairs]) {
  float4* p = reinterpret_cast<float4*>(partials + chunk * inter + j * 2 * S::kPairs);
#pragma unroll
  for (int k = 0; k < S::kPairs / 2; ++k) p[k] = make_float4(s[2 * k].x, s[2 * k].y, s[2 * k + 1].x, s[2 * k + 1].y);
}

template <typename S, int GATE, bool HAS_LB, bool FULL>
__global__ void __launch_bounds__(kMaxThreads) situ_glu_fwd_ew_kernel(const EwArgs a) {
  constexpr int kP = S::kPairs;
  const int nt = blockDim.x;
  if (a.vpr <= 2 * nt) {
    const int j = threadIdx.x, j2 = j + nt;
    const bool one = j < a.vpr, two = j2 < a.vpr;
    int64_t row = blockIdx.x;
    if (row >= a.tokens) return;
    const uint4 z = make_uint4(0, 0, 0, 0);
    uint4 g0 = z, u0 = z, g1 = z, u1 = z;
    float2 w0[kP], w1[kP];  // [I]: this thread's columns, loaded once; [T, I]: the current row's
    {
      const char* gu = a.gate_up + row * a.gu_pitch;
      const char* wr = a.rw + row * a.rw_pitch;
      if (one) {
        g0 = ld_stream(gu + j * kVecBytes);
        u0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
        load_w_pairs<S>(wr, j, a.rw_bf16, w0);
      }
      if (two) {
        g1 = ld_stream(gu + j2 * kVecBytes);
        u1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
        load_w_pairs<S>(wr, j2, a.rw_bf16, w1);
      }
    }
    for (;;) {
      const int64_t next = row + gridDim.x;
      const bool more = next < a.tokens;
      uint4 ng0, nu0, ng1, nu1;
      float2 nw0[kP], nw1[kP];
      if (more) {
        const char* gu = a.gate_up + next * a.gu_pitch;
        const char* wr = a.rw + next * a.rw_pitch;
        if (one) {
          ng0 = ld_stream(gu + j * kVecBytes);
          nu0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
          if (FULL) load_w_pairs<S>(wr, j, a.rw_bf16, nw0);
        }
        if (two) {
          ng1 = ld_stream(gu + j2 * kVecBytes);
          nu1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
          if (FULL) load_w_pairs<S>(wr, j2, a.rw_bf16, nw1);
        }
      }
      char* out = a.out + row * a.out_pitch;
      if (one) st_stream(out + j * kVecBytes, ew_fwd_vec<S, GATE, HAS_LB>(g0, u0, w0, a.c));
      if (two) st_stream(out + j2 * kVecBytes, ew_fwd_vec<S, GATE, HAS_LB>(g1, u1, w1, a.c));
      if (!more) break;
      row = next;
      g0 = ng0; u0 = nu0; g1 = ng1; u1 = nu1;
      if (FULL) {
#pragma unroll
        for (int p = 0; p < kP; ++p) { w0[p] = nw0[p]; w1[p] = nw1[p]; }
      }
    }
    return;
  }
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    const char* gu = a.gate_up + row * a.gu_pitch;
    char* out = a.out + row * a.out_pitch;
    const char* wr = a.rw + row * a.rw_pitch;
    for (int j = threadIdx.x; j < a.vpr; j += nt) {
      float2 w[kP];
      load_w_pairs<S>(wr, j, a.rw_bf16, w);
      st_stream(out + j * kVecBytes, ew_fwd_vec<S, GATE, HAS_LB>(ld_stream(gu + j * kVecBytes),
                                                                 ld_stream(gu + a.half_bytes + j * kVecBytes), w, a.c));
    }
  }
}

template <typename S, int GATE, bool HAS_LB, bool FULL>
__global__ void __launch_bounds__(kMaxThreads) situ_glu_bwd_ew_kernel(const EwArgs a) {
  extern __shared__ float col_sums[];  // looped form, [I] weights with a wanted gradient: [inter]
  constexpr int kP = S::kPairs, kElems = 2 * kP;
  constexpr int64_t kRows = FULL ? 1 : kColChunk;  // rows per chunk
  const int nt = blockDim.x;
  const bool want = a.d_rw != nullptr;
  const int64_t nchunks = (a.tokens + kRows - 1) / kRows;
  if (a.vpr <= 2 * nt) {
    const int j = threadIdx.x, j2 = j + nt;
    const bool one = j < a.vpr, two = j2 < a.vpr;
    int64_t ch = blockIdx.x;
    if (ch >= nchunks) return;
    int64_t row = ch * kRows, end = min(a.tokens, row + kRows);
    const uint4 z = make_uint4(0, 0, 0, 0);
    uint4 g0 = z, u0 = z, o0 = z, g1 = z, u1 = z, o1 = z;
    float2 w0[kP], w1[kP], s0[kP], s1[kP];
    zero_pairs<S>(s0);
    zero_pairs<S>(s1);
    {
      const char* gu = a.gate_up + row * a.gu_pitch;
      const char* gor = a.grad_out + row * a.go_pitch;
      const char* wr = a.rw + row * a.rw_pitch;
      if (one) {
        g0 = ld_stream(gu + j * kVecBytes);
        u0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
        o0 = ld_stream(gor + j * kVecBytes);
        load_w_pairs<S>(wr, j, a.rw_bf16, w0);
      }
      if (two) {
        g1 = ld_stream(gu + j2 * kVecBytes);
        u1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
        o1 = ld_stream(gor + j2 * kVecBytes);
        load_w_pairs<S>(wr, j2, a.rw_bf16, w1);
      }
    }
    for (;;) {
      int64_t next = row + 1, nch = ch, nend = end;
      if (next >= end) {  // the chunk is done: on to the CTA's next chunk
        nch = ch + gridDim.x;
        next = nch * kRows;
        nend = min(a.tokens, next + kRows);
      }
      const bool more = nch < nchunks;
      uint4 ng0, nu0, no0, ng1, nu1, no1;
      float2 nw0[kP], nw1[kP];
      if (more) {
        const char* gu = a.gate_up + next * a.gu_pitch;
        const char* gor = a.grad_out + next * a.go_pitch;
        const char* wr = a.rw + next * a.rw_pitch;
        if (one) {
          ng0 = ld_stream(gu + j * kVecBytes);
          nu0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
          no0 = ld_stream(gor + j * kVecBytes);
          if (FULL) load_w_pairs<S>(wr, j, a.rw_bf16, nw0);
        }
        if (two) {
          ng1 = ld_stream(gu + j2 * kVecBytes);
          nu1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
          no1 = ld_stream(gor + j2 * kVecBytes);
          if (FULL) load_w_pairs<S>(wr, j2, a.rw_bf16, nw1);
        }
      }
      char* dgu = a.out + row * a.out_pitch;
      char* drw = FULL && want ? a.d_rw + row * a.d_rw_pitch : nullptr;
      float2 t[kP];
      uint4 dg, du;
      if (one) {
        ew_bwd_vec<S, GATE, HAS_LB, !FULL>(g0, u0, o0, w0, a.c, dg, du, t);
        st_stream(dgu + j * kVecBytes, dg);
        st_stream(dgu + a.half_bytes + j * kVecBytes, du);
        if (want) {
          if (FULL) store_w_pairs<S>(drw, j, a.rw_bf16, t);
          else add_pairs<S>(s0, t);
        }
      }
      if (two) {
        ew_bwd_vec<S, GATE, HAS_LB, !FULL>(g1, u1, o1, w1, a.c, dg, du, t);
        st_stream(dgu + j2 * kVecBytes, dg);
        st_stream(dgu + a.half_bytes + j2 * kVecBytes, du);
        if (want) {
          if (FULL) store_w_pairs<S>(drw, j2, a.rw_bf16, t);
          else add_pairs<S>(s1, t);
        }
      }
      if (!FULL && want && nch != ch) {
        if (one) store_col_partials<S>(a.partials, ch, a.inter, j, s0);
        if (two) store_col_partials<S>(a.partials, ch, a.inter, j2, s1);
        zero_pairs<S>(s0);
        zero_pairs<S>(s1);
      }
      if (!more) break;
      row = next;
      ch = nch;
      end = nend;
      g0 = ng0; u0 = nu0; o0 = no0; g1 = ng1; u1 = nu1; o1 = no1;
      if (FULL) {
#pragma unroll
        for (int p = 0; p < kP; ++p) { w0[p] = nw0[p]; w1[p] = nw1[p]; }
      }
    }
    return;
  }
  // Looped form.  Thread t owns the columns of its vectors j = t, t + nt, ...:
  // it alone resets, adds to and exports them, so no barrier is needed.
  const bool colsum = !FULL && want;
  for (int64_t ch = blockIdx.x; ch < nchunks; ch += gridDim.x) {
    if (colsum)
      for (int j = threadIdx.x; j < a.vpr; j += nt)
        for (int e = 0; e < kElems; ++e) col_sums[j * kElems + e] = 0.0f;
    const int64_t r1 = min(a.tokens, (ch + 1) * kRows);
    for (int64_t row = ch * kRows; row < r1; ++row) {
      const char* gu = a.gate_up + row * a.gu_pitch;
      const char* gor = a.grad_out + row * a.go_pitch;
      char* dgu = a.out + row * a.out_pitch;
      const char* wr = a.rw + row * a.rw_pitch;
      for (int j = threadIdx.x; j < a.vpr; j += nt) {
        float2 w[kP], t[kP];
        load_w_pairs<S>(wr, j, a.rw_bf16, w);
        uint4 dg, du;
        ew_bwd_vec<S, GATE, HAS_LB, !FULL>(ld_stream(gu + j * kVecBytes), ld_stream(gu + a.half_bytes + j * kVecBytes),
                                    ld_stream(gor + j * kVecBytes), w, a.c, dg, du, t);
        st_stream(dgu + j * kVecBytes, dg);
        st_stream(dgu + a.half_bytes + j * kVecBytes, du);
        if (want) {
          if (FULL) {
            store_w_pairs<S>(a.d_rw + row * a.d_rw_pitch, j, a.rw_bf16, t);
          } else {
#pragma unroll
            for (int p = 0; p < kP; ++p) {
              col_sums[j * kElems + 2 * p] += t[p].x;
              col_sums[j * kElems + 2 * p + 1] += t[p].y;
            }
          }
        }
      }
    }
    if (colsum)
      for (int j = threadIdx.x; j < a.vpr; j += nt)
        for (int e = 0; e < kElems; ++e) a.partials[ch * a.inter + j * kElems + e] = col_sums[j * kElems + e];
  }
}

// Per-column gradient: add the chunks' partial sums.  A CTA takes 32 columns
// (one warp-wide, coalesced row of partials) and 32 chunk groups: group g adds
// chunks g, g + 32, ... in eight interleaved running sums (eight loads in
// flight per thread), and the groups are then added in group order.  The
// order depends on nchunks alone.
constexpr int kFinCols = 32, kFinGroups = 32, kFinLanes = 8;

__global__ void __launch_bounds__(kFinCols * kFinGroups)
    situ_glu_dw_columns_finalize_kernel(const float* partials, int64_t nchunks, int inter, void* d_rw, int bf16) {
  __shared__ float red[kFinGroups][kFinCols + 1];
  const int lane = threadIdx.x % kFinCols, grp = threadIdx.x / kFinCols;
  const int i = blockIdx.x * kFinCols + lane;
  float s = 0.0f;
  if (i < inter) {
    float acc[kFinLanes];
#pragma unroll
    for (int q = 0; q < kFinLanes; ++q) acc[q] = 0.0f;
    int64_t k = grp;
    for (; k + (kFinLanes - 1) * kFinGroups < nchunks; k += kFinLanes * kFinGroups) {
#pragma unroll
      for (int q = 0; q < kFinLanes; ++q) acc[q] += partials[(k + q * kFinGroups) * inter + i];
    }
    for (; k < nchunks; k += kFinGroups) acc[0] += partials[k * inter + i];
#pragma unroll
    for (int q = 0; q < kFinLanes; ++q) s += acc[q];
  }
  red[grp][lane] = s;
  __syncthreads();
  if (grp == 0 && i < inter) {
    float t = red[0][lane];
    for (int g = 1; g < kFinGroups; ++g) t += red[g][lane];
    store_rw_grad(d_rw, i, bf16, t);
  }
}

// ---------------------------------------------------------------------------
// Wide direct-load forward (the default whenever the layout allows)
// ---------------------------------------------------------------------------
// When a half row holds 64 k 16-byte vectors (k = 1..8) and every base and row
// pitch is 32-byte aligned, CTA thread t owns the 32 contiguous bytes at 32 t
// of each half row: one 256-bit load per input and one 256-bit store per
// output, no lane without work, and half the address arithmetic of the
// two-vector layout.  Rows are software-pipelined as in the kernels above.
// (The same layout measured slower for the backward, whose next-row loads it
// did not keep in flight; the backward keeps the two-vector layout.)

template <typename S, int GATE, bool HAS_LB>
__global__ void __launch_bounds__(kMaxThreads) situ_glu_fwd_wide_kernel(const FwdArgs a) {
  const int off = threadIdx.x * 32;
  int64_t row = blockIdx.x;
  if (row >= a.tokens) return;
  const char* gu = a.gate_up + row * a.gu_pitch + off;
  U8 g = ld_stream32(gu), u = ld_stream32(gu + a.half_bytes);
  float w = load_rw(a.rw, row);
  for (;;) {
    const int64_t next = row + gridDim.x;
    const bool more = next < a.tokens;
    U8 ng, nu;
    float nw = 0.0f;
    if (more) {
      const char* ngu = a.gate_up + next * a.gu_pitch + off;
      ng = ld_stream32(ngu);
      nu = ld_stream32(ngu + a.half_bytes);
      nw = load_rw(a.rw, next);
    }
    const float2 wbb = splat(w * a.c.bb);
    st_stream32(a.out + row * a.out_pitch + off, fwd_vec<S, GATE, HAS_LB>(g.a, u.a, wbb, a.c),
                fwd_vec<S, GATE, HAS_LB>(g.b, u.b, wbb, a.c));
    if (!more) break;
    row = next;
    g = ng;
    u = nu;
    w = nw;
  }
}

// ---------------------------------------------------------------------------
// MXFP8 outputs (OCP Microscaling Formats v1.0)
// ---------------------------------------------------------------------------
// Y (forward) or d_gate_up (backward) leave the kernel as FP8 E4M3 codes with
// one E8M0 scale per 32 consecutive elements of a row, the format of the
// MXFP8 recipe the SiTU-GLU integration was tested with (Megatron-LM PR #6673,
// "Test results").  A block is the 32 / kElems adjacent lanes that own its
// vectors (4 for bf16 inputs, 8 for fp32); its largest magnitude is combined
// with lane shuffles, so the fp32 values are quantised straight from
// registers.  Shared exponent e, stored as the byte e + 127:
//   SITU_MX_RULE_OCP:  floor(log2 amax) - 8 (the exponent of E4M3's largest
//                      normal), elements clamped to +-448;
//   SITU_MX_RULE_CEIL: the smallest e with amax <= 448 2^e (nothing clamps);
// both at least -127.  Both exponents come from the bits of amax, exactly.
// A block holding a NaN or an infinity gets scale byte 255 (NaN) and NaN codes.

constexpr int kMxBlock = 32;

struct MxOut {
  char* data;            // E4M3 codes, [tokens, cols]
  int64_t data_pitch;    // bytes
  uint8_t* scale;        // E8M0 bytes, [tokens, cols / 32]
  int64_t scale_pitch;   // bytes
  int rule;              // situ_mx_rule_t
};

__device__ __forceinline__ void st_stream_u32(void* p, uint32_t v) {
  asm volatile("st.global.cs.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Four E4M3 codes (nearest even, clamped to +-448, NaN to NaN) of a.x, a.y,
// b.x, b.y, in that byte order.  cvt...e4m3x2 puts its first source in the
// upper byte of the 16-bit result.
__device__ __forceinline__ uint32_t e4m3x4(float2 a, float2 b) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return r;
}

// Where a thread's vector j of a row goes: its codes at byte kElems j of the
// row, its block's scale byte at j / (32 / kElems) (written by the block's
// first lane).  Computed once per thread.
template <typename S>
struct MxSlot {
  int code_off;
  int scale_off;
  bool lead;
  __device__ __forceinline__ explicit MxSlot(int j) {
    constexpr int kElems = 2 * S::kPairs, kLanes = kMxBlock / kElems;
    code_off = j * kElems;
    scale_off = j / kLanes;
    lead = (j % kLanes) == 0;
  }
};

// Quantise the kPairs pairs y of one vector of a row.  Every lane of the warp
// calls this (the block maximum is shuffled); lanes with `active` set store
// their codes and the first lane of each block the scale byte -- or, with
// SCALE_ALL_LANES, every lane of the block the same byte, which drops a branch
// (measured faster in the backward, slower in the forward).  A block is
// active or inactive as a whole (rows are multiples of 32 elements).
template <typename S, bool ACTIVE_ALWAYS = false, bool SCALE_ALL_LANES = false>
__device__ __forceinline__ void mx_store_vec(const float2 (&y)[S::kPairs], bool active, char* data_row,
                                             uint8_t* scale_row, const MxSlot<S>& slot, int rule) {
  constexpr int kElems = 2 * S::kPairs;
  constexpr int kLanes = kMxBlock / kElems;
  float amax = 0.0f;
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) amax = max_nan(amax, max_nan(fabsf(y[p].x), fabsf(y[p].y)));
  if (!ACTIVE_ALWAYS && !active) amax = 0.0f;
#pragma unroll
  for (int o = 1; o < kLanes; o <<= 1) amax = max_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const uint32_t ab = __float_as_uint(amax);
  const int ef = static_cast<int>(ab >> 23);  // amax >= 0 (or NaN with the sign bit clear)
  // e + 127 = (ef - 127) - 8 + 127, plus one under the no-clamp rule when the
  // significand of amax exceeds 1.75 (448 = 1.75 2^8); zero and subnormal
  // blocks land on the smallest scale; ef = 255 (NaN, inf) gives the NaN scale.
  int sb = ef - 8 + ((rule == SITU_MX_RULE_CEIL && (ab & 0x7fffffu) > 0x600000u) ? 1 : 0);
  sb = sb < 0 ? 0 : sb;
  const bool nan_blk = ef >= 255;
  sb = nan_blk ? 255 : sb;
  // 2^-e as a normal float (biased exponent 254 - sb in [7, 254] for sb <= 247);
  // a NaN block scales by NaN, so that its codes come out NaN.
  const float inv = nan_blk ? __uint_as_float(0x7fc00000u) : __uint_as_float(static_cast<uint32_t>(254 - sb) << 23);
  uint32_t q[S::kPairs / 2];
#pragma unroll
  for (int k = 0; k < S::kPairs / 2; ++k) q[k] = e4m3x4(mul2(y[2 * k], splat(inv)), mul2(y[2 * k + 1], splat(inv)));
  if (!ACTIVE_ALWAYS && !active) return;
  char* p = data_row + slot.code_off;
  if constexpr (kElems == 8)
    st_stream8(p, make_uint2(q[0], q[1]));
  else
    st_stream_u32(p, q[0]);
  if (SCALE_ALL_LANES || slot.lead) scale_row[slot.scale_off] = static_cast<uint8_t>(sb);
}

// ---- NVFP4 (E2M1 codes, an E4M3 scale per 16 elements, a per-tensor scale)
// NVIDIA's NVFP4 format, the other block-scaled recipe the SiTU-GLU path was
// tested with (Megatron-LM PR #6673, "Test results").  With A the tensor's
// largest magnitude, S_enc = 448 * 6 / A (1 when A is 0 or not finite); block
// b of 16 elements stores s_b = E4M3(amax_b * S_enc / 6) and each element the
// E2M1 code of y * (S_enc / s_b) (nearest even, clamped to +-6); decoding is
// q * s_b / S_enc.  Codes are packed two per byte, element 2k in the low
// nibble.  A block holding NaN or infinity gets scale code 0x7F.

struct Nvfp4Out {
  char* data;            // packed E2M1 codes, [tokens, cols / 2] bytes
  int64_t data_pitch;    // bytes
  uint8_t* scale;        // E4M3 block scales, [tokens, cols / 16]
  int64_t scale_pitch;   // bytes
  const float* amax;     // device: the tensor's largest finite magnitude (read by the quantising pass)
  float* amax_out;       // the same word, written by the amax pass (host-side use)
};

// An NVFP4 output of the backward: where its codes go, and whether the
// caller gives the tensor maximum.
struct Nvfp4Bwd {
  Nvfp4Out out;
  int amax_given;
};

// Two E2M1 codes of (lo, hi) in one byte, lo in the low nibble (cvt packs its
// first source into the high nibble); four such bytes per register.
__device__ __forceinline__ uint32_t e2m1x8(const float2 (&v)[4]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0].x), "f"(v[0].y), "f"(v[1].x), "f"(v[1].y), "f"(v[2].x), "f"(v[2].y), "f"(v[3].x), "f"(v[3].y));
  return r;
}
__device__ __forceinline__ uint32_t e2m1x4(const float2 (&v)[2]) {
  uint16_t r;
  asm("{\n\t.reg .b8 b0, b1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "mov.b16 %0, {b0, b1};\n\t}"
      : "=h"(r)
      : "f"(v[0].x), "f"(v[0].y), "f"(v[1].x), "f"(v[1].y));
  return r;
}

__device__ __forceinline__ float nvfp4_tensor_scale(float amax) {
  return (amax > 0.0f && amax <= 3.402823466e38f) ? 2688.0f / amax : 1.0f;  // 448 * 6 / A
}

// Quantise the kPairs pairs y of vector j of a row into NVFP4.  Every lane of
// the warp calls this (the block maximum is shuffled over the 16 / kElems
// lanes of a block); lanes with `active` set store their codes and the first
// lane of each block (SCALE_ALL_LANES: every lane of it) its scale code.
template <typename S, bool ACTIVE_ALWAYS = false, bool SCALE_ALL_LANES = false>
__device__ __forceinline__ void nvfp4_store_vec(const float2 (&y)[S::kPairs], bool active, char* data_row,
                                                uint8_t* scale_row, int j, float s_enc) {
  constexpr int kElems = 2 * S::kPairs;
  constexpr int kLanes = 16 / kElems;
  float amax = 0.0f;
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) amax = max_nan(amax, max_nan(fabsf(y[p].x), fabsf(y[p].y)));
  if (!ACTIVE_ALWAYS && !active) amax = 0.0f;
#pragma unroll
  for (int o = 1; o < kLanes; o <<= 1) amax = max_nan(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const bool special = __float_as_uint(amax) >= 0x7f800000u;
  const uint8_t sc = special ? static_cast<uint8_t>(0x7f)
                             : static_cast<uint8_t>(__nv_cvt_float_to_fp8(amax * s_enc / 6.0f, __NV_SATFINITE, __NV_E4M3));
  const float sb = special ? 0.0f : __half2float(__half(__nv_cvt_fp8_to_halfraw(sc, __NV_E4M3)));
  // S_enc / s_b to 2 ulp (s_b is at most 448): an extra rounding of a few
  // 2^-24 that can only move an element sitting on an E2M1 midpoint
  const float r = sb > 0.0f ? __fdividef(s_enc, sb) : 0.0f;
  float2 q[S::kPairs];
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) q[p] = mul2(y[p], splat(r));
  if (!ACTIVE_ALWAYS && !active) return;
  if constexpr (S::kPairs == 4) {
    st_stream_u32(data_row + j * 4, e2m1x8(q));
  } else {
    const uint16_t v = static_cast<uint16_t>(e2m1x4(q));
    asm volatile("st.global.cs.u16 [%0], %1;" ::"l"(data_row + j * 2), "h"(v) : "memory");
  }
  if (SCALE_ALL_LANES || j % kLanes == 0) scale_row[j / kLanes] = sc;
}

// Register budgets of the block-scaled backward, as CTAs of 256 threads per
// SM.  MXFP8: three (at most 85 registers a thread), measured faster on B200
// than two, the issue-bound MXFP8 backward gaining more from the extra warps
// than it loses to the tighter budget.  The NVFP4 and amax-only passes: two
// (at most 128 registers), measured faster than three (which spills).
#ifndef SITU_BWD_MX_MIN_CTAS
#define SITU_BWD_MX_MIN_CTAS 3
#endif
#ifndef SITU_BWD_NV_MIN_CTAS
#define SITU_BWD_NV_MIN_CTAS 2
#endif
#ifndef SITU_BWD_AMAX_MIN_CTAS
#define SITU_BWD_AMAX_MIN_CTAS 2
#endif

// Output policies of the row pipeline below: MXFP8 codes, NVFP4 codes, or
// the tensor maximum only.  State is what a thread carries across its rows
// (the tensor scale, or its running maximum); finish() runs once per thread
// at the end, with every lane of the warp present.
struct MxQuant {
  using Out = MxOut;
  using State = int;
  static constexpr int kBwdMinCtas = SITU_BWD_MX_MIN_CTAS;  // CTAs of 256 threads per SM, backward
  __device__ __forceinline__ static State init(const Out&) { return 0; }
  template <typename S, bool ALL>
  __device__ __forceinline__ static void store(const float2 (&y)[S::kPairs], bool active, const Out& m, int64_t row,
                                               int j, State&) {
    mx_store_vec<S, ALL>(y, active, m.data + row * m.data_pitch, m.scale + row * m.scale_pitch, MxSlot<S>(j), m.rule);
  }
  // Backward: dG's codes and scales, then dU's half a row on.
  template <typename S, bool ALL>
  __device__ __forceinline__ static void store2(const float2 (&dg)[S::kPairs], const float2 (&du)[S::kPairs],
                                                bool active, const Out& m, int64_t row, int j, int inter, State&) {
    char* d = m.data + row * m.data_pitch;
    uint8_t* sc = m.scale + row * m.scale_pitch;
    const MxSlot<S> slot(j);
    mx_store_vec<S, ALL, true>(dg, active, d, sc, slot, m.rule);
    mx_store_vec<S, ALL, true>(du, active, d + inter, sc + inter / kMxBlock, slot, m.rule);
  }
  __device__ __forceinline__ static void finish(const Out&, const State&) {}
};
struct Nvfp4Quant {
  using Out = Nvfp4Out;
  using State = float;  // S_enc
  static constexpr int kBwdMinCtas = SITU_BWD_NV_MIN_CTAS;
  __device__ __forceinline__ static State init(const Out& m) { return nvfp4_tensor_scale(*m.amax); }
  template <typename S, bool ALL>
  __device__ __forceinline__ static void store(const float2 (&y)[S::kPairs], bool active, const Out& m, int64_t row,
                                               int j, State& s_enc) {
    nvfp4_store_vec<S, ALL>(y, active, m.data + row * m.data_pitch, m.scale + row * m.scale_pitch, j, s_enc);
  }
  template <typename S, bool ALL>
  __device__ __forceinline__ static void store2(const float2 (&dg)[S::kPairs], const float2 (&du)[S::kPairs],
                                                bool active, const Out& m, int64_t row, int j, int inter,
                                                State& s_enc) {
    char* d = m.data + row * m.data_pitch;
    uint8_t* sc = m.scale + row * m.scale_pitch;
    nvfp4_store_vec<S, ALL, true>(dg, active, d, sc, j, s_enc);
    nvfp4_store_vec<S, ALL, true>(du, active, d + inter / 2, sc + inter / 16, j, s_enc);
  }
  __device__ __forceinline__ static void finish(const Out&, const State&) {}
};
// The tensor's largest finite |Y| (NVFP4's tensor scale; NaN and infinite
// elements only mark their own blocks): per-thread maxima of the fp32
// results, a warp maximum, one integer atomicMax per warp on the float bits
// (non-negative floats order as integers), so the result is order-free.
struct AmaxOnly {
  using Out = unsigned int*;
  using State = float;
  static constexpr int kBwdMinCtas = SITU_BWD_AMAX_MIN_CTAS;
  __device__ __forceinline__ static State init(const Out&) { return 0.0f; }
  template <typename S, bool ALL>
  __device__ __forceinline__ static void store(const float2 (&y)[S::kPairs], bool, const Out&, int64_t, int,
                                               State& m) {
#pragma unroll
    for (int p = 0; p < S::kPairs; ++p) {  // inactive lanes hold zeros
      const float ax = fabsf(y[p].x), ay = fabsf(y[p].y);
      m = ax <= 3.402823466e38f ? fmaxf(m, ax) : m;  // false for NaN and infinity
      m = ay <= 3.402823466e38f ? fmaxf(m, ay) : m;
    }
  }
  template <typename S, bool ALL>
  __device__ __forceinline__ static void store2(const float2 (&dg)[S::kPairs], const float2 (&du)[S::kPairs],
                                                bool active, const Out& o, int64_t row, int j, int, State& m) {
    store<S, ALL>(dg, active, o, row, j, m);
    store<S, ALL>(du, active, o, row, j, m);
  }
  __device__ __forceinline__ static void finish(const Out& amax_bits, const State& m) {
    const unsigned int bits = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
    if ((threadIdx.x & 31) == 0 && bits != 0u) atomicMax(amax_bits, bits);
  }
};

template <typename S, int GATE, bool HAS_LB>
__device__ __forceinline__ void fwd_pairs(const uint4& gv, const uint4& uv, float2 wbb, const Coeffs& c,
                                          float2 (&y)[S::kPairs]) {
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) {
    if constexpr (std::is_same<S, Bf16>::value)
      y[p] = fwd_pair_bf16<GATE, HAS_LB>(S::pair(gv, p), S::pair(uv, p), wbb, c);
    else
      y[p] = fwd_pair_abs<GATE, HAS_LB, S>(S::pair(gv, p), S::pair(uv, p), wbb, c);
  }
}

// Whether any of 8 packed bf16 gate values lies below -27.75, the signed
// backward's clamp (NaN pairs count as below: they take the |g| form).
__device__ __forceinline__ bool gate_below_clamp_bf16x8(const uint4& v) {
  uint32_t m, cl;
  asm("{\n\t.reg .b32 t0, t1;\n\t"
      "min.bf16x2 t0, %2, %3;\n\t"
      "min.bf16x2 t1, %4, %5;\n\t"
      "min.bf16x2 %0, t0, t1;\n\t"
      "max.bf16x2 %1, %0, %6;\n\t}"
      : "=r"(m), "=r"(cl)
      : "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(0xC1DEC1DEu));
  return cl != m;
}

// dG and dU of one vector for the block-scaled outputs.  Their codes keep
// relative accuracy for tiny values, so the clamped signed form is out; but
// where no gate value of the warp's vectors lies below the clamp (`extreme`
// false, the caller's vote) the clamp changes nothing and the signed form
// runs without it.  Otherwise the |g| form, exact for every g.
template <typename S, int GATE, bool HAS_LB>
__device__ __forceinline__ void bwd_pairs(const uint4& gv, const uint4& uv, const uint4& gov, float2 k,
                                          const Coeffs& c, float2 (&dg)[S::kPairs], float2 (&du)[S::kPairs],
                                          float2& acc, bool extreme) {
  const float2 kdg = splat(k.x), kdu = splat(k.y);
  if constexpr (SignedBwd<GATE, S, true>::value) {
    if (!extreme) {
#pragma unroll
      for (int p = 0; p < S::kPairs; ++p)
        bwd_pair<GATE, HAS_LB, S, true, true>(S::pair(gv, p), S::pair(uv, p), as_f2(S::pair(gov, p)), kdg, kdu, c,
                                              dg[p], du[p], acc);
      return;
    }
  }
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p)
    bwd_pair<GATE, HAS_LB, S>(S::pair(gv, p), S::pair(uv, p), as_f2(S::pair(gov, p)), kdg, kdu, c, dg[p], du[p], acc);
}

template <typename S>
__device__ __forceinline__ void zero_y(float2 (&y)[S::kPairs]) {
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) y[p] = make_float2(0.0f, 0.0f);
}

// Rows of the two-vector layout; ALL: every lane owns two vectors (vpr = 2 nt),
// so no lane is ever inactive.  Q: the output format (MXFP8 or NVFP4).
template <typename S, int GATE, bool HAS_LB, bool ALL, class Q>
__device__ __forceinline__ void fwd_quant_rows(const FwdArgs& a, const typename Q::Out& m) {
  constexpr int kP = S::kPairs;
  const int nt = blockDim.x;
  const int j = threadIdx.x, j2 = j + nt;
  const bool one = ALL || j < a.vpr, two = ALL || j2 < a.vpr;
  typename Q::State st = Q::init(m);
  int64_t row = blockIdx.x;
  if (row >= a.tokens) return;  // the whole block
  const uint4 z = make_uint4(0, 0, 0, 0);
  uint4 g0 = z, u0 = z, g1 = z, u1 = z;
  {
    const char* gu = a.gate_up + row * a.gu_pitch;
    if (one) {
      g0 = ld_stream(gu + j * kVecBytes);
      u0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
    }
    if (two) {
      g1 = ld_stream(gu + j2 * kVecBytes);
      u1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
    }
  }
  float w = load_rw(a.rw, row);
  for (;;) {
    const int64_t next = row + gridDim.x;
    const bool more = next < a.tokens;
    uint4 ng0, nu0, ng1, nu1;
    float nw = 0.0f;
    if (more) {
      const char* ngu = a.gate_up + next * a.gu_pitch;
      if (one) {
        ng0 = ld_stream(ngu + j * kVecBytes);
        nu0 = ld_stream(ngu + a.half_bytes + j * kVecBytes);
      }
      if (two) {
        ng1 = ld_stream(ngu + j2 * kVecBytes);
        nu1 = ld_stream(ngu + a.half_bytes + j2 * kVecBytes);
      }
      nw = load_rw(a.rw, next);
    }
    const float2 wbb = splat(w * a.c.bb);
    float2 y[kP];
    if (ALL || one) fwd_pairs<S, GATE, HAS_LB>(g0, u0, wbb, a.c, y); else zero_y<S>(y);
    Q::template store<S, ALL>(y, one, m, row, j, st);
    if (ALL || two) fwd_pairs<S, GATE, HAS_LB>(g1, u1, wbb, a.c, y); else zero_y<S>(y);
    Q::template store<S, ALL>(y, two, m, row, j2, st);
    if (!more) break;
    row = next;
    g0 = ng0; u0 = nu0; g1 = ng1; u1 = nu1; w = nw;
  }
  Q::finish(m, st);
}

template <typename S, int GATE, bool HAS_LB, class Q>
__global__ void __launch_bounds__(kMaxThreads) situ_glu_fwd_quant_kernel(const FwdArgs a, const typename Q::Out m) {
  constexpr int kP = S::kPairs;
  const int nt = blockDim.x;
  if (a.vpr == 2 * nt) {
    fwd_quant_rows<S, GATE, HAS_LB, true, Q>(a, m);
    return;
  }
  if (a.vpr < 2 * nt) {
    fwd_quant_rows<S, GATE, HAS_LB, false, Q>(a, m);
    return;
  }
  typename Q::State st = Q::init(m);
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    const char* gu = a.gate_up + row * a.gu_pitch;
    const float2 wbb = splat(load_rw(a.rw, row) * a.c.bb);
    for (int jb = 0; jb < a.vpr; jb += nt) {  // uniform trip count: every lane reaches the shuffles
      const int j = jb + threadIdx.x;
      const bool act = j < a.vpr;
      float2 y[kP];
      if (act)
        fwd_pairs<S, GATE, HAS_LB>(ld_stream(gu + j * kVecBytes), ld_stream(gu + a.half_bytes + j * kVecBytes), wbb,
                                   a.c, y);
      else
        zero_y<S>(y);
      Q::template store<S, false>(y, act, m, row, j, st);
    }
  }
  Q::finish(m, st);
}

// Backward with a block-scaled d_gate_up (MXFP8 or NVFP4; dG's codes and
// scales, then dU's), or the tensor maximum of d_gate_up only (the NVFP4
// amax pass); the routing-weight gradient as in the per-row kernel.
template <typename S, int GATE, bool HAS_LB>
__device__ __forceinline__ void bwd_quant_finish_row(const BwdArgs& a, int64_t row, float2 acc, float* red) {
  if (a.want_drw) {  // uniform over the launch
    const float total = block_sum(acc.x + acc.y, red) * bwd_dw_scale(a.c);
    if (threadIdx.x == 0) {
      if (a.rw.mode == SITU_RW_SCALAR)
        a.partials[row] = total;
      else
        store_rw_grad(a.d_rw, row * a.d_rw_stride, a.rw.bf16, total);
    }
  }
}

// One vector's dG and dU, handed to the output policy.
template <typename S, int GATE, bool HAS_LB, bool ALL, class Q>
__device__ __forceinline__ void bwd_quant_vec(const uint4& g, const uint4& u, const uint4& o, bool act, float2 k,
                                              const Coeffs& c, const typename Q::Out& m, int64_t row, int j,
                                              int inter, typename Q::State& st, float2& acc) {
  constexpr int kP = S::kPairs;
  float2 dg[kP], du[kP];
  // Every lane of the warp is here (inactive lanes hold zero vectors).
  const bool extreme = !SignedBwd<GATE, S, true>::value || __any_sync(0xffffffffu, gate_below_clamp_bf16x8(g));
  if (ALL || act) {
    bwd_pairs<S, GATE, HAS_LB>(g, u, o, k, c, dg, du, acc, extreme);
  } else {
    zero_y<S>(dg);
    zero_y<S>(du);
  }
  Q::template store2<S, ALL>(dg, du, act, m, row, j, inter, st);
}

template <typename S, int GATE, bool HAS_LB, bool ALL, class Q>
__device__ __forceinline__ void bwd_quant_rows(const BwdArgs& a, const typename Q::Out& m,
                                               float (*red)[kMaxThreads / 32]) {
  constexpr int kP = S::kPairs;
  const int nt = blockDim.x;
  const int inter = a.half_bytes / kVecBytes * (2 * kP);  // elements per half row
  const int j = threadIdx.x, j2 = j + nt;
  const bool one = ALL || j < a.vpr, two = ALL || j2 < a.vpr;
  typename Q::State st = Q::init(m);
  int parity = 0;
  int64_t row = blockIdx.x;
  if (row >= a.tokens) return;  // the whole block
  const uint4 z = make_uint4(0, 0, 0, 0);
  uint4 g0 = z, u0 = z, o0 = z, g1 = z, u1 = z, o1 = z;
  {
    const char* gu = a.gate_up + row * a.gu_pitch;
    const char* go_row = a.grad_out + row * a.go_pitch;
    if (one) {
      g0 = ld_stream(gu + j * kVecBytes);
      u0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
      o0 = ld_stream(go_row + j * kVecBytes);
    }
    if (two) {
      g1 = ld_stream(gu + j2 * kVecBytes);
      u1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
      o1 = ld_stream(go_row + j2 * kVecBytes);
    }
  }
  float w = load_rw(a.rw, row);
  for (;;) {
    const int64_t next = row + gridDim.x;
    const bool more = next < a.tokens;
    uint4 ng0, nu0, no0, ng1, nu1, no1;
    float nw = 0.0f;
    if (more) {
      const char* gu = a.gate_up + next * a.gu_pitch;
      const char* go_row = a.grad_out + next * a.go_pitch;
      if (one) {
        ng0 = ld_stream(gu + j * kVecBytes);
        nu0 = ld_stream(gu + a.half_bytes + j * kVecBytes);
        no0 = ld_stream(go_row + j * kVecBytes);
      }
      if (two) {
        ng1 = ld_stream(gu + j2 * kVecBytes);
        nu1 = ld_stream(gu + a.half_bytes + j2 * kVecBytes);
        no1 = ld_stream(go_row + j2 * kVecBytes);
      }
      nw = load_rw(a.rw, next);
    }
    const float2 k = bwd_row_consts<HAS_LB>(w, a.c);
    float2 acc = make_float2(0.0f, 0.0f);
    bwd_quant_vec<S, GATE, HAS_LB, ALL, Q>(g0, u0, o0, one, k, a.c, m, row, j, inter, st, acc);
    bwd_quant_vec<S, GATE, HAS_LB, ALL, Q>(g1, u1, o1, two, k, a.c, m, row, j2, inter, st, acc);
    bwd_quant_finish_row<S, GATE, HAS_LB>(a, row, acc, red[parity]);
    parity ^= 1;
    if (!more) break;
    row = next;
    g0 = ng0; u0 = nu0; o0 = no0; g1 = ng1; u1 = nu1; o1 = no1; w = nw;
  }
  Q::finish(m, st);
}


template <typename S, int GATE, bool HAS_LB, class Q>
__global__ void __launch_bounds__(kMaxThreads, Q::kBwdMinCtas)
    situ_glu_bwd_quant_kernel(const BwdArgs a, const typename Q::Out m) {
  __shared__ float red[2][kMaxThreads / 32];
  const int nt = blockDim.x;
  if (PipelineRows<S, true>::value && a.vpr == 2 * nt) {
    bwd_quant_rows<S, GATE, HAS_LB, true, Q>(a, m, red);
    return;
  }
  if (PipelineRows<S, true>::value && a.vpr < 2 * nt) {
    bwd_quant_rows<S, GATE, HAS_LB, false, Q>(a, m, red);
    return;
  }
  const int inter = a.half_bytes / kVecBytes * (2 * S::kPairs);
  typename Q::State st = Q::init(m);
  int parity = 0;
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    const char* gu = a.gate_up + row * a.gu_pitch;
    const char* go_row = a.grad_out + row * a.go_pitch;
    const float2 k = bwd_row_consts<HAS_LB>(load_rw(a.rw, row), a.c);
    float2 acc = make_float2(0.0f, 0.0f);
    for (int jb = 0; jb < a.vpr; jb += nt) {  // uniform trip count: every lane reaches the shuffles
      const int j = jb + threadIdx.x;
      const bool act = j < a.vpr;
      const uint4 z = make_uint4(0, 0, 0, 0);
      bwd_quant_vec<S, GATE, HAS_LB, false, Q>(act ? ld_stream(gu + j * kVecBytes) : z,
                                               act ? ld_stream(gu + a.half_bytes + j * kVecBytes) : z,
                                               act ? ld_stream(go_row + j * kVecBytes) : z, act, k, a.c, m, row, j,
                                               inter, st, acc);
    }
    bwd_quant_finish_row<S, GATE, HAS_LB>(a, row, acc, red[parity]);
    parity ^= 1;
  }
  Q::finish(m, st);
}

// ---------------------------------------------------------------------------
// TMA-staged kernels (load path 1)
// ---------------------------------------------------------------------------
// Warp 0 of each CTA is a producer: one lane streams chunks of rows from HBM
// into a ring of shared-memory stages with 1-D bulk copies (cp.async.bulk,
// completion counted in bytes on the stage's "full" mbarrier).  The other
// warps are consumers: they wait on "full", read their 16-byte vectors from
// shared memory, compute in registers, store the outputs straight to global
// memory, and release the stage on its "empty" mbarrier.  The bytes in flight
// are set by the ring, not by registers, so the consumers keep every register
// for arithmetic.  A CTA visits rows blockIdx.x, blockIdx.x + gridDim.x, ...
// and, within a row, its chunks in order; producer and consumers derive the
// same sequence, so no work queue is needed.
//
// Every wait is bounded (kWaitLimitNs of %globaltimer).  A wait that expires
// sets g_device_status; a consumer then stops waiting and computing but keeps
// the control flow (so the consumer-only named barrier cannot strand anyone),
// and the producer waits, again bounded, for the copies it issued before it
// returns.

constexpr int kMaxStages = 8;
constexpr int kMaxConsumers = 256;
#ifndef SITU_RING_BYTES
#define SITU_RING_BYTES (32 * 1024)
#endif
constexpr int kRingBytes = SITU_RING_BYTES;  // shared-memory ring per CTA
constexpr int kHeaderBytes = 256;      // mbarriers + reduction slots
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kStatusWaitExpired = 1;

__device__ int g_device_status = 0;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for the phase of parity `parity` to complete; false once `limit_ns`
// (the kernels': kWaitLimitNs) has passed.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* b, uint32_t parity, unsigned long long limit_ns) {
  if (mbar_try_wait(b, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  while (!mbar_try_wait(b, parity))
    if (global_timer_ns() - t0 > limit_ns) return false;
  return true;
}
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity) {
  return mbar_wait_for(b, parity, kWaitLimitNs);
}

// One thread waiting on an mbarrier that nothing completes (situ_glu_wait_probe):
// the expiry path every staged kernel takes when a copy never lands.
__global__ void situ_wait_probe_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
    if (!mbar_wait_for(&bar, 0, limit_ns)) atomicExch(&g_device_status, kStatusWaitExpired);
  }
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Thread-block clusters: this CTA's rank, its cluster's index and count
// (1-D grids), and cluster-scope addressing and synchronisation.
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_index() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// The shared::cluster address of the same shared-memory location in CTA `rank`.
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint4 lds16(const unsigned char* p) { return *reinterpret_cast<const uint4*>(p); }
__device__ __forceinline__ void consumer_bar(int n) { asm volatile("bar.sync 1, %0;" ::"r"(n) : "memory"); }

struct StreamArgs {
  const char* gate_up;
  int64_t gu_pitch;  // bytes
  const char* grad_out;  // backward only
  int64_t go_pitch;
  char* out;  // forward: Y; backward: d_gate_up
  int64_t out_pitch;
  RwArgs rw;
  void* d_rw;
  int64_t d_rw_stride;
  float* partials;
  int want_drw;
  int64_t tokens;
  int half_bytes;   // inter * element size
  int vpr;          // 16-byte vectors per half row
  int chunk_v;      // vectors per half row per chunk (the last chunk may be shorter)
  int nchunks;      // chunks per row
  int stages;       // ring stages
  int stage_bytes;  // bytes per stage (inputs x chunk_v x 16, rounded to 128)
  Coeffs c;
};

template <typename S, int GATE, bool HAS_LB, bool BWD>
__device__ __forceinline__ void tma_stream_body(const StreamArgs& a) {
  extern __shared__ __align__(128) unsigned char smem[];
  constexpr int kInputs = BWD ? 3 : 2;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  float* red = reinterpret_cast<float*>(empty + kMaxStages);  // [2][kMaxConsumers / 32]
  unsigned char* ring = smem + kHeaderBytes;
  const int nc = blockDim.x - 32;
  const int chunk_bytes = a.chunk_v * kVecBytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], nc / 32);
    }
    mbar_fence_init();
  }
  __syncthreads();

  if (threadIdx.x < 32) {  // ---- producer warp: one lane issues the copies
    if (threadIdx.x != 0) return;
    int64_t k = 0;
    bool ok = true;
    for (int64_t row = blockIdx.x; ok && row < a.tokens; row += gridDim.x) {
      const char* gu = a.gate_up + row * a.gu_pitch;
      const char* go = BWD ? a.grad_out + row * a.go_pitch : nullptr;
      for (int ch = 0; ch < a.nchunks; ++ch, ++k) {
        const int s = static_cast<int>(k % a.stages);
        const int64_t use = k / a.stages;
        if (use > 0 && !mbar_wait(&empty[s], static_cast<uint32_t>((use - 1) & 1))) {
          ok = false;
          break;
        }
        const int v0 = ch * a.chunk_v;
        const uint32_t bytes = static_cast<uint32_t>(min(a.chunk_v, a.vpr - v0)) * kVecBytes;
        unsigned char* st = ring + s * a.stage_bytes;
        mbar_arrive_expect_tx(&full[s], bytes * kInputs);
        bulk_load(st, gu + v0 * kVecBytes, bytes, &full[s]);
        bulk_load(st + chunk_bytes, gu + a.half_bytes + v0 * kVecBytes, bytes, &full[s]);
        if (BWD) bulk_load(st + 2 * chunk_bytes, go + v0 * kVecBytes, bytes, &full[s]);
      }
    }
    if (!ok) {  // drain: the last copy issued into each stage must land before the CTA exits
      atomicExch(&g_device_status, kStatusWaitExpired);
      for (int s = 0; s < a.stages && s < k; ++s) {
        const int64_t last_use = (k - 1 - s) / a.stages;
        mbar_wait(&full[s], static_cast<uint32_t>(last_use & 1));
      }
    }
    return;
  }

  // ---- consumer warps
  const int ctid = threadIdx.x - 32;
  const int lane = threadIdx.x & 31;
  int64_t k = 0;
  int parity = 0;
  bool ok = true;
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    const float w = load_rw(a.rw, row);
    const float2 wbb = splat(w * a.c.bb);
    const float2 kc = bwd_row_consts<HAS_LB>(w, a.c);
    char* out = a.out + row * a.out_pitch;
    float2 acc = make_float2(0.0f, 0.0f);
    for (int ch = 0; ch < a.nchunks; ++ch, ++k) {
      const int s = static_cast<int>(k % a.stages);
      const int64_t use = k / a.stages;
      if (ok && !mbar_wait(&full[s], static_cast<uint32_t>(use & 1))) {
        ok = false;
        atomicExch(&g_device_status, kStatusWaitExpired);
      }
      if (!ok) continue;
      const unsigned char* st = ring + s * a.stage_bytes;
      const int v0 = ch * a.chunk_v;
      const int nv = min(a.chunk_v, a.vpr - v0);
      for (int v = ctid; v < nv; v += 2 * nc) {
        const int v2 = v + nc;
        const bool two = v2 < nv;
        const uint4 g0 = lds16(st + v * kVecBytes);
        const uint4 u0 = lds16(st + chunk_bytes + v * kVecBytes);
        uint4 g1 = make_uint4(0, 0, 0, 0), u1 = g1;
        if (two) {
          g1 = lds16(st + v2 * kVecBytes);
          u1 = lds16(st + chunk_bytes + v2 * kVecBytes);
        }
        char* o0 = out + (v0 + v) * kVecBytes;
        char* o1 = out + (v0 + v2) * kVecBytes;
        if constexpr (BWD) {
          const uint4 q0 = lds16(st + 2 * chunk_bytes + v * kVecBytes);
          const uint4 q1 = two ? lds16(st + 2 * chunk_bytes + v2 * kVecBytes) : make_uint4(0, 0, 0, 0);
          uint4 dg, du;
          bwd_vec<S, GATE, HAS_LB>(g0, u0, q0, kc, a.c, dg, du, acc);
          st_stream(o0, dg);
          st_stream(o0 + a.half_bytes, du);
          if (two) {
            bwd_vec<S, GATE, HAS_LB>(g1, u1, q1, kc, a.c, dg, du, acc);
            st_stream(o1, dg);
            st_stream(o1 + a.half_bytes, du);
          }
        } else {
          st_stream(o0, fwd_vec<S, GATE, HAS_LB>(g0, u0, wbb, a.c));
          if (two) st_stream(o1, fwd_vec<S, GATE, HAS_LB>(g1, u1, wbb, a.c));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (BWD && a.want_drw) {  // fixed-order sum over the consumer threads
      float v = acc.x + acc.y;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      float* slot = red + parity * (kMaxConsumers / 32);
      if (lane == 0) slot[ctid >> 5] = v;
      consumer_bar(nc);
      if (ctid < 32) {
        float t = ctid < nc / 32 ? slot[ctid] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
        t *= bwd_dw_scale(a.c);
        if (ctid == 0 && ok) {
          if (a.rw.mode == SITU_RW_SCALAR)
            a.partials[row] = t;
          else
            store_rw_grad(a.d_rw, row * a.d_rw_stride, a.rw.bf16, t);
        }
      }
      parity ^= 1;
    }
  }
}

template <typename S, int GATE, bool HAS_LB>
__global__ void __launch_bounds__(kMaxConsumers + 32) situ_glu_fwd_tma_kernel(const StreamArgs a) {
  tma_stream_body<S, GATE, HAS_LB, false>(a);
}

template <typename S, int GATE, bool HAS_LB>
__global__ void __launch_bounds__(kMaxConsumers + 32) situ_glu_bwd_tma_kernel(const StreamArgs a) {
  tma_stream_body<S, GATE, HAS_LB, true>(a);
}

// ---------------------------------------------------------------------------
// Attention-residual mixing core
// ---------------------------------------------------------------------------
// NeMo AutoModel kimi_k3.situ `_attn_res_core` / `_apply_attn_res`: for token
// row t with sources b (the stored block sums, then the current prefix sum),
//   logit[b] = sum_h values[b, h] / sqrt(mean_h values[b]^2 + eps) * norm_w[h] * proj_w[h]
//   out[h]   = sum_b softmax(logit)[b] values[b, h]
// in fp32.  The RMSNorm scale is constant over h, so each logit is
// rsqrt(ss_b / H + eps) * dd_b with two sums per source, ss_b = sum_h x^2 and
// dd_b = sum_h x c_h, c = norm_w * proj_w (kept in shared memory).  One CTA
// works on one row at a time: pass 1 streams the row's sources once for the
// 2 S sums (per-thread partials, warp shuffles, then the warps in order: a
// fixed order, so results do not depend on the grid); every thread then forms
// the softmax; pass 2 reads the sources again -- from L2, where pass 1 left
// them -- and writes the weighted sum.  HBM sees each value once.

constexpr int kArMaxSources = 16;
constexpr int kArThreads = 256;

struct ArArgs {
  const char* blocks;        // stored sums: row pitch / source pitch in bytes
  int64_t block_row_pitch;
  int64_t block_pitch;
  const char* prefix;        // current sum (the last source) or NULL
  int64_t prefix_row_pitch;
  int nblocks;
  int sources;
  int64_t tokens;
  int hidden;
  int vpr;                   // 16-byte vectors of one source row
  const void* norm_w;
  int norm_bf16;
  const void* proj_w;
  int proj_bf16;
  float eps;
  float inv_hidden;
  char* out;
  int64_t out_pitch;         // bytes
  int out_bf16;
};

__device__ __forceinline__ float ar_weight(const void* w, int bf16, int h) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(w)[h]) : reinterpret_cast<const float*>(w)[h];
}

template <typename S>
__device__ __forceinline__ const char* ar_source(const ArArgs& a, int64_t row, int b) {
  return b < a.nblocks ? a.blocks + row * a.block_row_pitch + b * a.block_pitch : a.prefix + row * a.prefix_row_pitch;
}

template <typename S>
__global__ void __launch_bounds__(kArThreads) situ_attn_res_kernel(const ArArgs a) {
  constexpr int kElems = 2 * S::kPairs;
  extern __shared__ float c_sh[];                       // [hidden]: norm_w * proj_w
  __shared__ float red[kArThreads / 32][2 * kArMaxSources];
  __shared__ float prob_sh[kArMaxSources];
  const int nt = blockDim.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int h = threadIdx.x; h < a.hidden; h += nt) c_sh[h] = ar_weight(a.norm_w, a.norm_bf16, h) * ar_weight(a.proj_w, a.proj_bf16, h);
  __syncthreads();
  for (int64_t row = blockIdx.x; row < a.tokens; row += gridDim.x) {
    float ss[kArMaxSources], dd[kArMaxSources];
#pragma unroll
    for (int b = 0; b < kArMaxSources; ++b) {
      ss[b] = 0.0f;
      dd[b] = 0.0f;
      if (b < a.sources) {
        const char* src = ar_source<S>(a, row, b);
        for (int j = threadIdx.x; j < a.vpr; j += nt) {
          const uint4 v = ld_stream(src + j * kVecBytes);
#pragma unroll
          for (int p = 0; p < S::kPairs; ++p) {
            const float2 x = as_f2(S::pair(v, p));
            const float2 c = make_float2(c_sh[j * kElems + 2 * p], c_sh[j * kElems + 2 * p + 1]);
            ss[b] = fmaf(x.x, x.x, fmaf(x.y, x.y, ss[b]));
            dd[b] = fmaf(x.x, c.x, fmaf(x.y, c.y, dd[b]));
          }
        }
      }
    }
    // CTA sums of the 2 S partials: warp shuffles, then the warps in order.
#pragma unroll
    for (int b = 0; b < kArMaxSources; ++b) {
      if (b < a.sources) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          ss[b] += __shfl_xor_sync(0xffffffffu, ss[b], o);
          dd[b] += __shfl_xor_sync(0xffffffffu, dd[b], o);
        }
        if (lane == 0) {
          red[warp][2 * b] = ss[b];
          red[warp][2 * b + 1] = dd[b];
        }
      }
    }
    __syncthreads();
    if (threadIdx.x < a.sources) {
      const int b = threadIdx.x;
      float s2 = 0.0f, d2 = 0.0f;
      for (int w = 0; w < (nt >> 5); ++w) {
        s2 += red[w][2 * b];
        d2 += red[w][2 * b + 1];
      }
      prob_sh[b] = d2 * rsqrtf(s2 * a.inv_hidden + a.eps);  // the logit, for now
    }
    __syncthreads();
    float p[kArMaxSources];
    float mx = prob_sh[0];
#pragma unroll
    for (int b = 1; b < kArMaxSources; ++b)
      if (b < a.sources) mx = fmaxf(mx, prob_sh[b]);
    float z = 0.0f;
#pragma unroll
    for (int b = 0; b < kArMaxSources; ++b) {
      p[b] = b < a.sources ? __expf(prob_sh[b] - mx) : 0.0f;
      z += p[b];
    }
    const float rz = 1.0f / z;
#pragma unroll
    for (int b = 0; b < kArMaxSources; ++b) p[b] *= rz;
    // pass 2: out = sum_b p_b values[b]
    char* orow = a.out + row * a.out_pitch;
    for (int j = threadIdx.x; j < a.vpr; j += nt) {
      float2 acc[S::kPairs];
#pragma unroll
      for (int q = 0; q < S::kPairs; ++q) acc[q] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int b = 0; b < kArMaxSources; ++b) {
        if (b < a.sources) {
          const uint4 v = *reinterpret_cast<const uint4*>(ar_source<S>(a, row, b) + j * kVecBytes);
#pragma unroll
          for (int q = 0; q < S::kPairs; ++q) acc[q] = fma2(splat(p[b]), as_f2(S::pair(v, q)), acc[q]);
        }
      }
      if (a.out_bf16) {
        uint32_t w[S::kPairs];
#pragma unroll
        for (int q = 0; q < S::kPairs; ++q) w[q] = Bf16::pack(acc[q]);
        if constexpr (S::kPairs == 4)
          st_stream(orow + j * 16, make_uint4(w[0], w[1], w[2], w[3]));
        else
          st_stream8(orow + j * 8, make_uint2(w[0], w[1]));
      } else {
#pragma unroll
        for (int q = 0; q < S::kPairs / 2; ++q)
          st_stream(orow + j * kElems * 4 + q * 16, make_uint4(__float_as_uint(acc[2 * q].x), __float_as_uint(acc[2 * q].y),
                                                              __float_as_uint(acc[2 * q + 1].x),
                                                              __float_as_uint(acc[2 * q + 1].y)));
      }
    }
    __syncthreads();  // red and prob_sh are rewritten by the next row
  }
}

// Staged form (the default when a source row is at most 1024 16-byte
// vectors, there are at most kArStagedSources sources, and the row fits in
// shared memory): one CTA per SM; thread j owns column vectors j,
// j + nt, ... (V of them, nt threads) of every source.  Bulk copies bring the
// CTA's next token row -- the stored sums as one run when they lie back to
// back, else one run per source, and the current sum -- into shared memory
// while the current row is computed from registers, so each value crosses
// HBM once and the copy of the next row overlaps the reductions, the softmax
// and the weighted sum of this one.  The mbarrier wait is bounded; an expired
// wait sets the device status word and the CTA stops after letting its own
// copy land.
constexpr int kArStagedSources = 9;
constexpr int kArStagedThreads = 896;  // vectors per row at V = 1 (hidden 7168 in bf16)

// The warp's per-source partial sums of one token row for the attention-
// residual core: red_w[2b] = sum of x_b^2 and red_w[2b + 1] = sum of x_b * c
// over the warp's column vectors (x[v]: the thread's v-th vector of each
// source, zero past `sources` or past the row; c[v]: norm_w * proj_w for its
// elements).
template <typename S, int V>
__device__ __forceinline__ void ar_warp_sums(const uint4 (&x)[V][kArStagedSources], const float2 (&c)[V][S::kPairs],
                                             int sources, int lane, float* red_w) {
  // Per-source sums of squares and projections (packed pairs).  Sources
  // 0-7 (16 slots: 2b the sum of squares, 2b + 1 the projection) are
  // reduced over the warp in one halving pass: at each level a lane keeps
  // half of its slots and adds its partner's copy of that half (8 + 4 + 2
  // + 1 exchanges, then one more add across lane pairs, instead of 5 per
  // slot); source 8 takes plain shuffles.  Every addition order is fixed.
  auto sums = [&](int b, float& ss, float& dd) {
    float2 ss2 = make_float2(0.0f, 0.0f), dd2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int v = 0; v < V; ++v) {
#pragma unroll
      for (int p = 0; p < S::kPairs; ++p) {
        const float2 xv = as_f2(S::pair(x[v][b], p));
        ss2 = fma2(xv, xv, ss2);
        dd2 = fma2(xv, c[v][p], dd2);
      }
    }
    ss = ss2.x + ss2.y;
    dd = dd2.x + dd2.y;
  };
  {
    float v[16];
#pragma unroll
    for (int b = 0; b < 8; ++b) {
      v[2 * b] = 0.0f;
      v[2 * b + 1] = 0.0f;
      if (b < sources) sums(b, v[2 * b], v[2 * b + 1]);
    }
#pragma unroll
    for (int o = 16, n = 8; n > 0; o >>= 1, n >>= 1) {
      const bool upper = (lane & o) != 0;  // keep slots [n, 2n), send [0, n)
#pragma unroll
      for (int k = 0; k < n; ++k) {
        const float send = upper ? v[k] : v[n + k];
        const float keep = upper ? v[n + k] : v[k];
        v[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    // Lanes 2s and 2s + 1 now hold the warp's sum of slot s (the halves
    // kept, level by level, spell out bits 4..1 of the lane).
    const int slot = lane >> 1;
    if ((lane & 1) == 0 && slot < 2 * sources && slot < 16) red_w[slot] = v[0];
  }
  if (sources > 8) {  // uniform
    float ss = 0.0f, dd = 0.0f;
    sums(8, ss, dd);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ss += __shfl_xor_sync(0xffffffffu, ss, o);
      dd += __shfl_xor_sync(0xffffffffu, dd, o);
    }
    if (lane == 0) {
      red_w[16] = ss;
      red_w[17] = dd;
    }
  }
}

// norm_w * proj_w for the elements of column vector jv (zero if !col).
template <typename S>
__device__ __forceinline__ void ar_weights(const ArArgs& a, bool col, int jv, float2 (&c)[S::kPairs]) {
  constexpr int kElems = 2 * S::kPairs;
#pragma unroll
  for (int p = 0; p < S::kPairs; ++p) {
    const int h = jv * kElems + 2 * p;
    c[p] = col ? make_float2(ar_weight(a.norm_w, a.norm_bf16, h) * ar_weight(a.proj_w, a.proj_bf16, h),
                             ar_weight(a.norm_w, a.norm_bf16, h + 1) * ar_weight(a.proj_w, a.proj_bf16, h + 1))
               : make_float2(0.0f, 0.0f);
  }
}

// The weighted sum of one column vector jv of a token row, sources in order,
// rounded once to the output dtype and stored.
template <typename S>
__device__ __forceinline__ void ar_combine_store(const ArArgs& a, const uint4 (&x)[kArStagedSources],
                                                 const float (&p)[kArStagedSources], int64_t row, int jv) {
  constexpr int kElems = 2 * S::kPairs;
  float2 acc[S::kPairs];
#pragma unroll
  for (int q = 0; q < S::kPairs; ++q) acc[q] = make_float2(0.0f, 0.0f);
#pragma unroll
  for (int b = 0; b < kArStagedSources; ++b) {
    if (b < a.sources) {
#pragma unroll
      for (int q = 0; q < S::kPairs; ++q) acc[q] = fma2(splat(p[b]), as_f2(S::pair(x[b], q)), acc[q]);
    }
  }
  char* orow = a.out + row * a.out_pitch;
  if (a.out_bf16) {
    uint32_t w[S::kPairs];
#pragma unroll
    for (int q = 0; q < S::kPairs; ++q) w[q] = Bf16::pack(acc[q]);
    if constexpr (S::kPairs == 4)
      st_stream(orow + jv * 16, make_uint4(w[0], w[1], w[2], w[3]));
    else
      st_stream8(orow + jv * 8, make_uint2(w[0], w[1]));
  } else {
#pragma unroll
    for (int q = 0; q < S::kPairs / 2; ++q)
      st_stream(orow + jv * kElems * 4 + q * 16,
                make_uint4(__float_as_uint(acc[2 * q].x), __float_as_uint(acc[2 * q].y),
                           __float_as_uint(acc[2 * q + 1].x), __float_as_uint(acc[2 * q + 1].y)));
  }
}

// NT: the most threads a launch may have.  Two vectors a thread take 448
// threads for rows of up to 896 vectors and 512 beyond (up to 1024: hidden
// 8192 in bf16, 4096 in fp32); the 448-thread bound keeps the register
// allocation that measured 2 % faster at hidden 7168.
template <typename S, int V, int NT>
__global__ void __launch_bounds__(NT, 1) situ_attn_res_staged_kernel(const ArArgs a) {
  extern __shared__ __align__(16) unsigned char ar_stage[];  // [sources][row bytes]
  __shared__ float red[NT / 32][2 * kArStagedSources];
  __shared__ float logit_sh[kArStagedSources];
  __shared__ float prob_sh[kArStagedSources];
  __shared__ __align__(8) uint64_t bar;
  const int j = threadIdx.x, warp = j >> 5, lane = j & 31, nwarps = blockDim.x >> 5, nt = blockDim.x;
  bool col[V];  // thread j owns column vectors j, j + nt, ...
#pragma unroll
  for (int v = 0; v < V; ++v) col[v] = j + v * nt < a.vpr;
  const uint32_t row_bytes = static_cast<uint32_t>(a.vpr) * kVecBytes;
  float2 c[V][S::kPairs];  // norm_w * proj_w for this thread's elements, as pairs
#pragma unroll
  for (int v = 0; v < V; ++v) ar_weights<S>(a, col[v], j + v * nt, c[v]);
  int64_t row = blockIdx.x;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  // Stored sums laid out back to back ([T, B, H] with a source pitch of one
  // row) travel as one bulk copy, the current sum as another: fewer, larger
  // copies per row measured 5 % faster than one copy per source.
  const bool merged = a.block_pitch == static_cast<int64_t>(row_bytes) && a.nblocks > 1;
  auto issue = [&](int64_t r) {  // thread 0: copy token row r into the stage
    mbar_arrive_expect_tx(&bar, row_bytes * static_cast<uint32_t>(a.sources));
    if (merged) {
      bulk_load(ar_stage, ar_source<S>(a, r, 0), row_bytes * static_cast<uint32_t>(a.nblocks), &bar);
      for (int b = a.nblocks; b < a.sources; ++b)
        bulk_load(ar_stage + b * row_bytes, ar_source<S>(a, r, b), row_bytes, &bar);
    } else {
      for (int b = 0; b < a.sources; ++b)
        bulk_load(ar_stage + b * row_bytes, ar_source<S>(a, r, b), row_bytes, &bar);
    }
  };
  if (threadIdx.x == 0 && row < a.tokens) issue(row);
  uint32_t phase = 0;
  bool in_flight = row < a.tokens;
  while (row < a.tokens) {
    const bool ok = mbar_wait(&bar, phase);
    if (__syncthreads_or(!ok)) {
      if (threadIdx.x == 0) atomicExch(&g_device_status, kStatusWaitExpired);
      break;
    }
    in_flight = false;
    phase ^= 1u;
    uint4 x[V][kArStagedSources];
#pragma unroll
    for (int v = 0; v < V; ++v)
#pragma unroll
      for (int b = 0; b < kArStagedSources; ++b)
        x[v][b] = (col[v] && b < a.sources) ? lds16(ar_stage + b * row_bytes + (j + v * nt) * kVecBytes)
                                            : make_uint4(0, 0, 0, 0);
    __syncthreads();  // the stage is free: start the next row's copy
    const int64_t next = row + gridDim.x;
    if (threadIdx.x == 0 && next < a.tokens) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // our reads before the copy's writes
      issue(next);
    }
    in_flight = next < a.tokens;
    ar_warp_sums<S, V>(x, c, a.sources, lane, red[warp]);
    __syncthreads();
    // The logits: the warps take the sources in turn, each summing one
    // source's two partial sums over the warps with a fixed shuffle tree.
    for (int b = warp; b < a.sources; b += nwarps) {  // warp w: sources w, w + nwarps, ...; one shuffle tree each
      float s2 = lane < nwarps ? red[lane][2 * b] : 0.0f;
      float d2 = lane < nwarps ? red[lane][2 * b + 1] : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        s2 += __shfl_xor_sync(0xffffffffu, s2, o);
        d2 += __shfl_xor_sync(0xffffffffu, d2, o);
      }
      if (lane == 0) logit_sh[b] = d2 * rsqrtf(s2 * a.inv_hidden + a.eps);
    }
    __syncthreads();
    // Warp 0 turns the logits into probabilities once and the other threads
    // read them: measured 10 % faster than every thread computing the softmax.
    if (warp == 0) {
      const float lg = lane < a.sources ? logit_sh[lane] : -INFINITY;
      float mxw = lg;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mxw = fmaxf(mxw, __shfl_xor_sync(0xffffffffu, mxw, o));
      const float e = lane < a.sources ? __expf(lg - mxw) : 0.0f;
      float zw = e;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) zw += __shfl_xor_sync(0xffffffffu, zw, o);
      if (lane < a.sources) prob_sh[lane] = e * (1.0f / zw);
    }
    __syncthreads();
    float p[kArStagedSources];
#pragma unroll
    for (int b = 0; b < kArStagedSources; ++b) p[b] = b < a.sources ? prob_sh[b] : 0.0f;
#pragma unroll
    for (int v = 0; v < V; ++v)
      if (col[v]) ar_combine_store<S>(a, x[v], p, row, j + v * nt);
    row = next;
  }
  // An expired wait leaves a copy possibly in flight: let it land (bounded)
  // before the CTA's shared memory is released.
  if (in_flight && threadIdx.x == 0) {
    const unsigned long long t0 = global_timer_ns();
    while (!mbar_try_wait(&bar, phase) && global_timer_ns() - t0 < kWaitLimitNs) {
    }
  }
}


#include "situ_fused_gemm.cuh"

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

// Bytes a routing-weight tensor (or its gradient) spans in a given mode.
Span weight_span(const void* p, situ_rw_mode_t mode, int64_t tokens, int64_t stride, int64_t inter, int es) {
  switch (mode) {
    case SITU_RW_ROW: return matrix_span(p, tokens, stride, 1, es);
    case SITU_RW_SCALAR: return matrix_span(p, 1, 1, 1, es);
    case SITU_RW_COL: return matrix_span(p, 1, inter, inter, es);
    case SITU_RW_FULL: return matrix_span(p, tokens, stride, inter, es);
    default: return {0, 0};
  }
}

// rows * pitch + width fits in int64 bytes.
bool span_fits(int64_t rows, int64_t pitch, int64_t width, int es) {
  if (width > INT64_MAX / es) return false;  // one row alone
  const int64_t limit = INT64_MAX / es - width;
  return rows <= 1 || (pitch <= limit / (rows - 1));
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int64_t kMaxInter = int64_t(1) << 28;

// Bytes of element-wise weights that go with one 16-byte vector of gate_up
// (the kernels load them in one piece), at most 16: the alignment that
// per-column and per-element weights and their gradient rows need.
int ew_align(situ_dtype_t dtype, situ_dtype_t rw_dtype) {
  const int a = kVecBytes / elem_size(dtype) * elem_size(rw_dtype);
  return a < 16 ? a : 16;
}

// Per-call constants of the element arithmetic and the gate's exponent form.
void fill_coeffs(double beta, int has_lb, double lb, Coeffs* c, int* gate_mode) {
  const double kLog2eD = 1.4426950408889634;
  c->beta = static_cast<float>(beta);
  c->kt = static_cast<float>(2.0 * kLog2eD / beta);
  c->lb = has_lb ? static_cast<float>(lb) : 1.0f;
  c->inv_lb = has_lb ? static_cast<float>(1.0 / lb) : 1.0f;
  c->ku = has_lb ? static_cast<float>(2.0 * kLog2eD / lb) : 0.0f;
  c->bb = static_cast<float>(has_lb ? beta * lb : beta);
  *gate_mode = beta == 4.0 ? kGateSquare : beta == 2.0 ? kGateEqual : beta == 1.0 ? kGateRoot : kGateGeneric;
}

// Checks common to fwd and bwd.  Fills coefficients and the gate mode.
situ_status_t check_common(situ_dtype_t dtype, int64_t tokens, int64_t inter, int64_t gu_stride,
                           const void* rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                           int64_t rw_stride, double beta, int has_lb, double lb, Coeffs* c,
                           int* gate_mode) {
  if (!valid_dtype(dtype)) return fail(SITU_ERR_INVALID_ARG, "dtype %d is not a situ_dtype_t", (int)dtype);
  if (rw_mode != SITU_RW_ROW && rw_mode != SITU_RW_SCALAR && rw_mode != SITU_RW_NONE && rw_mode != SITU_RW_COL &&
      rw_mode != SITU_RW_FULL)
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
  if (rw_mode == SITU_RW_FULL && rw_stride < inter) return fail(SITU_ERR_INVALID_ARG, "rw_stride < inter (full weights)");
  if (rw_mode == SITU_RW_COL && inter > kMaxColInter)
    return fail(SITU_ERR_UNSUPPORTED, "per-column weights support inter <= %d", kMaxColInter);
  const int es = elem_size(dtype);
  if ((rw_mode == SITU_RW_COL || rw_mode == SITU_RW_FULL) && tokens > 0) {
    const int a = ew_align(dtype, rw_dtype);
    if (!aligned(rw, a)) return fail(SITU_ERR_MISALIGNED, "element-wise weights must be %d-byte aligned", a);
    if (rw_mode == SITU_RW_FULL && (rw_stride * elem_size(rw_dtype)) % a != 0)
      return fail(SITU_ERR_MISALIGNED, "row pitch of full weights is not a multiple of %d bytes", a);
  }
  if ((inter * es) % kVecBytes != 0)
    return fail(SITU_ERR_MISALIGNED, "inter * element size (%lld bytes) is not a multiple of 16",
                (long long)(inter * es));

  fill_coeffs(beta, has_lb, lb, c, gate_mode);
  return SITU_OK;
}

// Threads per CTA: enough that each thread handles two 16-byte vectors of a
// half row (one pass of the kernel's two-vector body), at most kMaxThreads.
int choose_threads(int vpr) {
  const int passes = (vpr + 2 * kMaxThreads - 1) / (2 * kMaxThreads);
  const int nt = (vpr + 2 * passes - 1) / (2 * passes);
  return (nt + 31) / 32 * 32;
}

situ_status_t launch_grid(const void* kernel, int threads, int smem, int64_t tokens, int* grid) {
  int sms = 0;
  situ_status_t st = device_sm_count(&sms);
  if (st != SITU_OK) return st;
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, smem);
  if (err != cudaSuccess || per_sm <= 0)
    return fail(SITU_ERR_CUDA, "occupancy query: %s", cudaGetErrorString(err));
  int64_t g = static_cast<int64_t>(sms) * per_sm;
  const int cap = g_max_ctas.load(std::memory_order_relaxed);
  if (cap > 0 && g > cap) g = cap;
  if (g > tokens) g = tokens;
  *grid = static_cast<int>(g);
  return SITU_OK;
}

situ_status_t check_launch(const char* what);

std::atomic<int> g_load_path{0};  // 0: direct vector loads (default), 1: TMA ring

// Ring geometry of the TMA-staged kernels for a half row of `vpr` vectors and
// `inputs` streamed inputs (2 forward, 3 backward).
struct Geometry {
  int chunk_v, nchunks, consumers, stage_bytes, stages, smem;
};

Geometry stream_geometry(int vpr, int inputs) {
  Geometry g;
  const int balanced = (vpr + 2 * kMaxConsumers - 1) / (2 * kMaxConsumers);
  g.chunk_v = (vpr + balanced - 1) / balanced;        // <= 2 * kMaxConsumers
  g.nchunks = (vpr + g.chunk_v - 1) / g.chunk_v;      // every chunk holds >= 1 vector
  g.consumers = ((g.chunk_v + 1) / 2 + 31) / 32 * 32;
  g.stage_bytes = (g.chunk_v * kVecBytes * inputs + 127) / 128 * 128;
  g.stages = kRingBytes / g.stage_bytes;
  if (g.stages > kMaxStages) g.stages = kMaxStages;
  if (g.stages < 2) g.stages = 2;
  g.smem = kHeaderBytes + g.stages * g.stage_bytes;
  return g;
}

// Opt a kernel in to more than 48 KB of dynamic shared memory, once per
// (device, kernel, size).
situ_status_t ensure_smem(const void* kernel, int bytes) {
  struct Entry {
    int dev;
    const void* kernel;
    int bytes;
  };
  static std::mutex mu;
  static Entry seen[256];
  static int n_seen = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaGetDevice failed");
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < n_seen; ++i)
    if (seen[i].dev == dev && seen[i].kernel == kernel && seen[i].bytes >= bytes) return SITU_OK;
  cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(err));
  if (n_seen < 256) seen[n_seen++] = {dev, kernel, bytes};
  return SITU_OK;
}

using StreamKernel = void (*)(StreamArgs);

template <typename S, int GATE, bool LB, bool BWD>
StreamKernel stream_kernel() {
  if constexpr (BWD)
    return situ_glu_bwd_tma_kernel<S, GATE, LB>;
  else
    return situ_glu_fwd_tma_kernel<S, GATE, LB>;
}

template <typename S, bool LB, bool BWD>
StreamKernel pick_stream_gate(int gate) {
  switch (gate) {
    case kGateSquare: return stream_kernel<S, kGateSquare, LB, BWD>();
    case kGateEqual: return stream_kernel<S, kGateEqual, LB, BWD>();
    case kGateRoot: return stream_kernel<S, kGateRoot, LB, BWD>();
    default: return stream_kernel<S, kGateGeneric, LB, BWD>();
  }
}

template <bool BWD>
StreamKernel pick_stream(situ_dtype_t dtype, int gate, bool lb) {
  if (dtype == SITU_DTYPE_BF16)
    return lb ? pick_stream_gate<Bf16, true, BWD>(gate) : pick_stream_gate<Bf16, false, BWD>(gate);
  return lb ? pick_stream_gate<F32, true, BWD>(gate) : pick_stream_gate<F32, false, BWD>(gate);
}

// Launch the TMA-staged kernel for the arguments in `a`.
template <bool BWD>
situ_status_t launch_stream(StreamArgs& a, situ_dtype_t dtype, int gate, bool lb, cudaStream_t stream) {
  const Geometry g = stream_geometry(a.vpr, BWD ? 3 : 2);
  a.chunk_v = g.chunk_v;
  a.nchunks = g.nchunks;
  a.stages = g.stages;
  a.stage_bytes = g.stage_bytes;
  StreamKernel k = pick_stream<BWD>(dtype, gate, lb);
  situ_status_t st = ensure_smem(reinterpret_cast<const void*>(k), g.smem);
  if (st != SITU_OK) return st;
  const int threads = g.consumers + 32;
  int grid = 0;
  st = launch_grid(reinterpret_cast<const void*>(k), threads, g.smem, a.tokens, &grid);
  if (st != SITU_OK) return st;
  k<<<grid, threads, g.smem, stream>>>(a);
  return check_launch(BWD ? "situ_glu_bwd" : "situ_glu_fwd");
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

using EwKernel = void (*)(EwArgs);

template <typename S, int GATE, bool LB, bool BWD>
EwKernel ew_kernel(bool full) {
  if constexpr (BWD)
    return full ? situ_glu_bwd_ew_kernel<S, GATE, LB, true> : situ_glu_bwd_ew_kernel<S, GATE, LB, false>;
  else
    return full ? situ_glu_fwd_ew_kernel<S, GATE, LB, true> : situ_glu_fwd_ew_kernel<S, GATE, LB, false>;
}

template <typename S, bool LB, bool BWD>
EwKernel pick_ew_gate(int gate, bool full) {
  switch (gate) {
    case kGateSquare: return ew_kernel<S, kGateSquare, LB, BWD>(full);
    case kGateEqual: return ew_kernel<S, kGateEqual, LB, BWD>(full);
    case kGateRoot: return ew_kernel<S, kGateRoot, LB, BWD>(full);
    default: return ew_kernel<S, kGateGeneric, LB, BWD>(full);
  }
}

template <bool BWD>
EwKernel pick_ew(situ_dtype_t dtype, int gate, bool lb, bool full) {
  if (dtype == SITU_DTYPE_BF16)
    return lb ? pick_ew_gate<Bf16, true, BWD>(gate, full) : pick_ew_gate<Bf16, false, BWD>(gate, full);
  return lb ? pick_ew_gate<F32, true, BWD>(gate, full) : pick_ew_gate<F32, false, BWD>(gate, full);
}

template <typename S, bool LB>
FwdKernel pick_fwd_wide_gate(int gate) {
  switch (gate) {
    case kGateSquare: return situ_glu_fwd_wide_kernel<S, kGateSquare, LB>;
    case kGateEqual: return situ_glu_fwd_wide_kernel<S, kGateEqual, LB>;
    case kGateRoot: return situ_glu_fwd_wide_kernel<S, kGateRoot, LB>;
    default: return situ_glu_fwd_wide_kernel<S, kGateGeneric, LB>;
  }
}

FwdKernel pick_fwd_wide(situ_dtype_t dtype, int gate, bool lb) {
  if (dtype == SITU_DTYPE_BF16)
    return lb ? pick_fwd_wide_gate<Bf16, true>(gate) : pick_fwd_wide_gate<Bf16, false>(gate);
  return lb ? pick_fwd_wide_gate<F32, true>(gate) : pick_fwd_wide_gate<F32, false>(gate);
}

// The wide layout applies when a half row is 64 k vectors (k = 1..8: one
// 32-byte chunk per thread, at most kMaxThreads threads) and every listed
// base address and row pitch (bytes) is a multiple of 32.
bool wide_layout(int vpr, std::initializer_list<const void*> bases, std::initializer_list<int64_t> pitches) {
  if (vpr % 64 != 0 || vpr / 2 > kMaxThreads) return false;
  for (const void* b : bases)
    if (!aligned(b, 32)) return false;
  for (int64_t p : pitches)
    if (p % 32 != 0) return false;
  return true;
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

// Kernel of a block-scaled (or amax-only) pass for the dtype, gate form and
// linear-beta flag: the forward's or the backward's row loop with policy Q.
template <typename S, bool LB, class Q, bool BWD>
auto pick_quant_gate(int gate) {
  if constexpr (BWD) {
    switch (gate) {
      case kGateSquare: return situ_glu_bwd_quant_kernel<S, kGateSquare, LB, Q>;
      case kGateEqual: return situ_glu_bwd_quant_kernel<S, kGateEqual, LB, Q>;
      case kGateRoot: return situ_glu_bwd_quant_kernel<S, kGateRoot, LB, Q>;
      default: return situ_glu_bwd_quant_kernel<S, kGateGeneric, LB, Q>;
    }
  } else {
    switch (gate) {
      case kGateSquare: return situ_glu_fwd_quant_kernel<S, kGateSquare, LB, Q>;
      case kGateEqual: return situ_glu_fwd_quant_kernel<S, kGateEqual, LB, Q>;
      case kGateRoot: return situ_glu_fwd_quant_kernel<S, kGateRoot, LB, Q>;
      default: return situ_glu_fwd_quant_kernel<S, kGateGeneric, LB, Q>;
    }
  }
}
template <class Q, bool BWD>
auto pick_quant(situ_dtype_t dtype, int gate, bool lb) {
  if (dtype == SITU_DTYPE_BF16)
    return lb ? pick_quant_gate<Bf16, true, Q, BWD>(gate) : pick_quant_gate<Bf16, false, Q, BWD>(gate);
  return lb ? pick_quant_gate<F32, true, Q, BWD>(gate) : pick_quant_gate<F32, false, Q, BWD>(gate);
}

// Argument checks of an MXFP8 output of `cols` columns per row.
situ_status_t check_mx_args(const MxOut& m, int64_t inter, int64_t cols, situ_rw_mode_t rw_mode) {
  if (m.rule != SITU_MX_RULE_OCP && m.rule != SITU_MX_RULE_CEIL)
    return fail(SITU_ERR_INVALID_ARG, "rule %d is not a situ_mx_rule_t", m.rule);
  if (inter % kMxBlock != 0)
    return fail(SITU_ERR_INVALID_ARG, "MXFP8 outputs need inter a multiple of %d, got %lld", kMxBlock,
                (long long)inter);
  if (rw_mode == SITU_RW_COL || rw_mode == SITU_RW_FULL)
    return fail(SITU_ERR_UNSUPPORTED, "MXFP8 outputs take per-row, broadcast or no routing weights");
  if (m.data_pitch < cols) return fail(SITU_ERR_INVALID_ARG, "MXFP8 data row pitch < %lld bytes", (long long)cols);
  if (m.scale_pitch < cols / kMxBlock)
    return fail(SITU_ERR_INVALID_ARG, "MXFP8 scale row pitch < %lld bytes", (long long)(cols / kMxBlock));
  return SITU_OK;
}

// Pointer, extent and alignment checks of an MXFP8 output (tokens > 0).
situ_status_t check_mx_buffers(const MxOut& m, int64_t tokens, int64_t cols) {
  if (m.data == nullptr || m.scale == nullptr) return fail(SITU_ERR_INVALID_ARG, "MXFP8 data or scale is NULL");
  if (!span_fits(tokens, m.data_pitch, cols, 1) || !span_fits(tokens, m.scale_pitch, cols / kMxBlock, 1))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  if (!aligned(m.data, 16) || m.data_pitch % 16 != 0)
    return fail(SITU_ERR_MISALIGNED, "MXFP8 data base or row pitch not 16-byte aligned");
  const Span sd = matrix_span(m.data, tokens, m.data_pitch, cols, 1);
  const Span ss = matrix_span(m.scale, tokens, m.scale_pitch, cols / kMxBlock, 1);
  if (overlap(sd, ss)) return fail(SITU_ERR_INVALID_ARG, "MXFP8 data overlaps its scales");
  return SITU_OK;
}

// Argument checks of an NVFP4 output of `cols` columns per row.
situ_status_t check_nv_args(const Nvfp4Bwd& n, int64_t inter, int64_t cols, situ_rw_mode_t rw_mode) {
  if (inter % 16 != 0)
    return fail(SITU_ERR_INVALID_ARG, "NVFP4 outputs need inter a multiple of 16, got %lld", (long long)inter);
  if (rw_mode == SITU_RW_COL || rw_mode == SITU_RW_FULL)
    return fail(SITU_ERR_UNSUPPORTED, "NVFP4 outputs take per-row, broadcast or no routing weights");
  if (n.amax_given < 0 || n.amax_given > 2) return fail(SITU_ERR_INVALID_ARG, "amax_given must be 0, 1 or 2");
  if (n.amax_given != 2 && (n.out.data_pitch < cols / 2 || n.out.scale_pitch < cols / 16))
    return fail(SITU_ERR_INVALID_ARG, "NVFP4 data or scale row pitch shorter than a row");
  if (n.out.amax_out == nullptr) return fail(SITU_ERR_INVALID_ARG, "amax is NULL");
  if (!aligned(n.out.amax_out, 4)) return fail(SITU_ERR_MISALIGNED, "amax not 4-byte aligned");
  return SITU_OK;
}

// Pointer, extent and alignment checks of an NVFP4 output (tokens > 0).
situ_status_t check_nv_buffers(const Nvfp4Bwd& n, int64_t tokens, int64_t cols) {
  if (n.out.data == nullptr || n.out.scale == nullptr)
    return fail(SITU_ERR_INVALID_ARG, "NVFP4 data or scale is NULL");
  if (!span_fits(tokens, n.out.data_pitch, cols / 2, 1) || !span_fits(tokens, n.out.scale_pitch, cols / 16, 1))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  // a thread stores the codes of one 16-byte input vector: 4 bytes (bf16) or 2 (fp32)
  if (!aligned(n.out.data, 4) || n.out.data_pitch % 4 != 0)
    return fail(SITU_ERR_MISALIGNED, "NVFP4 data base or row pitch not 4-byte aligned");
  const Span sd = matrix_span(n.out.data, tokens, n.out.data_pitch, cols / 2, 1);
  const Span ss = matrix_span(n.out.scale, tokens, n.out.scale_pitch, cols / 16, 1);
  if (overlap(sd, ss)) return fail(SITU_ERR_INVALID_ARG, "NVFP4 data overlaps its scales");
  return SITU_OK;
}

// The forward with a native (mx == NULL) or an MXFP8 output.
situ_status_t fwd_entry(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                        int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                        int64_t rw_stride, double beta, int has_linear_beta, double linear_beta, void* out,
                        int64_t out_row_stride, const MxOut* mx, void* stream) {
  tl_last_error[0] = '\0';
  Coeffs c;
  int gate = kGateGeneric;
  situ_status_t st = check_common(dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                  rw_stride, beta, has_linear_beta, linear_beta, &c, &gate);
  if (st != SITU_OK) return st;
  if (mx != nullptr) {
    st = check_mx_args(*mx, inter, inter, rw_mode);
    if (st != SITU_OK) return st;
  } else if (out_row_stride < inter) {
    return fail(SITU_ERR_INVALID_ARG, "out_row_stride < inter");
  }
  if (tokens == 0) return SITU_OK;
  if (gate_up == nullptr || (mx == nullptr && out == nullptr))
    return fail(SITU_ERR_INVALID_ARG, "gate_up or out is NULL");
  const int es = elem_size(dtype);
  if (!span_fits(tokens, gate_up_row_stride, 2 * inter, es) ||
      (mx == nullptr && !span_fits(tokens, out_row_stride, inter, es)) ||
      (rw_mode == SITU_RW_ROW && !span_fits(tokens, rw_stride, 1, elem_size(rw_dtype))) ||
      (rw_mode == SITU_RW_FULL && !span_fits(tokens, rw_stride, inter, elem_size(rw_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  if (mx != nullptr) {
    st = check_mx_buffers(*mx, tokens, inter);
    if (st != SITU_OK) return st;
  }
  if (!aligned(gate_up, 16) || (gate_up_row_stride * es) % 16 != 0 ||
      (mx == nullptr && (!aligned(out, 16) || (out_row_stride * es) % 16 != 0)))
    return fail(SITU_ERR_MISALIGNED, "gate_up/out base or row pitch not 16-byte aligned");
  if (rw_mode != SITU_RW_NONE && !aligned(rw, elem_size(rw_dtype)))
    return fail(SITU_ERR_MISALIGNED, "rw not aligned to its element size");
  const Span s_gu = matrix_span(gate_up, tokens, gate_up_row_stride, 2 * inter, es);
  const Span s_rw = weight_span(rw, rw_mode, tokens, rw_stride, inter, elem_size(rw_dtype));
  const Span s_out = mx ? matrix_span(mx->data, tokens, mx->data_pitch, inter, 1)
                        : matrix_span(out, tokens, out_row_stride, inter, es);
  if (overlap(s_out, s_gu)) return fail(SITU_ERR_INVALID_ARG, "out overlaps gate_up");
  if (overlap(s_out, s_rw)) return fail(SITU_ERR_INVALID_ARG, "out overlaps rw");
  if (mx != nullptr) {
    const Span s_sc = matrix_span(mx->scale, tokens, mx->scale_pitch, inter / kMxBlock, 1);
    if (overlap(s_sc, s_gu) || overlap(s_sc, s_rw)) return fail(SITU_ERR_INVALID_ARG, "MXFP8 scales overlap an input");
  }

  if (rw_mode == SITU_RW_COL || rw_mode == SITU_RW_FULL) {
    EwArgs e{};
    e.gate_up = static_cast<const char*>(gate_up);
    e.gu_pitch = gate_up_row_stride * es;
    e.out = static_cast<char*>(out);
    e.out_pitch = out_row_stride * es;
    e.rw = static_cast<const char*>(rw);
    e.rw_pitch = rw_mode == SITU_RW_FULL ? rw_stride * elem_size(rw_dtype) : 0;
    e.rw_bf16 = rw_dtype == SITU_DTYPE_BF16 ? 1 : 0;
    e.tokens = tokens;
    e.half_bytes = static_cast<int>(inter * es);
    e.vpr = static_cast<int>(inter * es / kVecBytes);
    e.inter = static_cast<int>(inter);
    e.c = c;
    EwKernel k = pick_ew<false>(dtype, gate, has_linear_beta != 0, rw_mode == SITU_RW_FULL);
    const int threads = choose_threads(e.vpr);
    int grid = 0;
    st = launch_grid(reinterpret_cast<const void*>(k), threads, 0, tokens, &grid);
    if (st != SITU_OK) return st;
    k<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(e);
    return check_launch("situ_glu_fwd");
  }

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

  if (mx != nullptr) {
    auto k = pick_quant<MxQuant, false>(dtype, gate, has_linear_beta != 0);
    const int threads = choose_threads(a.vpr);
    int grid = 0;
    st = launch_grid(reinterpret_cast<const void*>(k), threads, 0, tokens, &grid);
    if (st != SITU_OK) return st;
    k<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(a, *mx);
    return check_launch("situ_glu_fwd_mxfp8");
  }
  if (g_load_path.load(std::memory_order_relaxed) == 1) {
    StreamArgs sa{};
    sa.gate_up = a.gate_up;
    sa.gu_pitch = a.gu_pitch;
    sa.out = a.out;
    sa.out_pitch = a.out_pitch;
    sa.rw = a.rw;
    sa.tokens = tokens;
    sa.half_bytes = a.half_bytes;
    sa.vpr = a.vpr;
    sa.c = c;
    return launch_stream<false>(sa, dtype, gate, has_linear_beta != 0, static_cast<cudaStream_t>(stream));
  }
  const bool wide = wide_layout(a.vpr, {gate_up, out}, {a.gu_pitch, a.out_pitch});
  FwdKernel k = wide ? pick_fwd_wide(dtype, gate, has_linear_beta != 0) : pick_fwd(dtype, gate, has_linear_beta != 0);
  const int threads = wide ? a.vpr / 2 : choose_threads(a.vpr);
  int grid = 0;
  st = launch_grid(reinterpret_cast<const void*>(k), threads, 0, tokens, &grid);
  if (st != SITU_OK) return st;
  k<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return check_launch("situ_glu_fwd");
}

// ---- FC1 grouped GEMM + SiTU-GLU: tensor maps and launch ----------------------

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 tensor map of a row-major [rows, >= inner] matrix read in boxes of
// 64 x 128 with the 128-byte swizzle the UMMA descriptors expect.
situ_status_t bf16_tile_map(CUtensorMap* m, const void* base, int64_t inner, int64_t rows, int64_t pitch_elems) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return fail(SITU_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(pitch_elems) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(fc1::kBK), static_cast<cuuint32_t>(fc1::kBM)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SITU_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  return SITU_OK;
}

using FusedGemmKernel = void (*)(const CUtensorMap, const CUtensorMap, const fc1::Args);

template <class Epi, bool LB, bool PAIR>
FusedGemmKernel pick_fused_gate(int gate) {
  if constexpr (PAIR) {
    switch (gate) {
      case kGateSquare: return fc1::situ_fused_gemm_2sm_kernel<Epi, kGateSquare, LB>;
      case kGateEqual: return fc1::situ_fused_gemm_2sm_kernel<Epi, kGateEqual, LB>;
      case kGateRoot: return fc1::situ_fused_gemm_2sm_kernel<Epi, kGateRoot, LB>;
      default: return fc1::situ_fused_gemm_2sm_kernel<Epi, kGateGeneric, LB>;
    }
  } else {
    switch (gate) {
      case kGateSquare: return fc1::situ_fused_gemm_kernel<Epi, kGateSquare, LB>;
      case kGateEqual: return fc1::situ_fused_gemm_kernel<Epi, kGateEqual, LB>;
      case kGateRoot: return fc1::situ_fused_gemm_kernel<Epi, kGateRoot, LB>;
      default: return fc1::situ_fused_gemm_kernel<Epi, kGateGeneric, LB>;
    }
  }
}

// The one-SM and two-SM kernels of a fused GEMM.
struct FusedKernels {
  FusedGemmKernel one, pair;
};

template <class Epi>
FusedKernels pick_fused(int gate, bool lb) {
  if (lb) return {pick_fused_gate<Epi, true, false>(gate), pick_fused_gate<Epi, true, true>(gate)};
  return {pick_fused_gate<Epi, false, false>(gate), pick_fused_gate<Epi, false, true>(gate)};
}

// Launch of a fused grouped GEMM, persistent over the output tiles.  The
// two-SM form (clusters of two CTAs, tcgen05 cta_group::2) runs whenever the
// device can keep at least one such cluster resident, as many clusters as fit
// at once; it measured 1.5 % (FC1) and 4 % (FC2) faster than the one-SM form
// on B200.  Otherwise one CTA per SM runs the one-SM kernel.
situ_status_t launch_fused(const FusedKernels& ks, const CUtensorMap& ma, const CUtensorMap& mb,
                           const fc1::Args& a, int64_t experts, cudaStream_t s, const char* what) {
  const int tables = static_cast<int>(experts) * (8 + 8 + 4) + 8;
  int sms = 0;
  situ_status_t st = device_sm_count(&sms);
  if (st != SITU_OK) return st;
  int grid = sms;
  const int cap = g_max_ctas.load(std::memory_order_relaxed);
  if (cap > 0 && grid > cap) grid = cap;
  if (grid >= 2) {
    const int smem = fc1::kStages2 * fc1::kStageBytes2 + 1024 + fc1::kHeaderBytes2 + tables;
    cudaError_t err = cudaFuncSetAttribute(reinterpret_cast<const void*>(ks.pair),
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(err));
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(fc1::kThreads, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    err = cudaOccupancyMaxActiveClusters(&clusters, reinterpret_cast<const void*>(ks.pair), &cfg);
    if (err != cudaSuccess) {
      (void)cudaGetLastError();  // the query's error is not sticky: fall back to the one-SM form
      clusters = 0;
    }
    if (clusters > 0) {
      if (2 * clusters > grid) clusters = grid / 2;
      cfg.gridDim = dim3(2 * clusters, 1, 1);
      err = cudaLaunchKernelEx(&cfg, ks.pair, ma, mb, a);
      if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "%s launch: %s", what, cudaGetErrorString(err));
      return check_launch(what);
    }
  }
  const int smem = fc1::kStages * fc1::kStageBytes + 1024 + fc1::kHeaderBytes + tables;
  cudaError_t err = cudaFuncSetAttribute(reinterpret_cast<const void*>(ks.one),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(err));
  ks.one<<<grid, fc1::kThreads, smem, s>>>(ma, mb, a);
  return check_launch(what);
}

// Per-row d_w of the fused FC2 data gradient: the row's column-tile partials
// in tile order, for the rows [offsets[0], offsets[experts]) (clamped).
__global__ void __launch_bounds__(256) situ_fc2_dw_finalize_kernel(const float* partials, int n_tiles,
                                                                   const int64_t* offsets, int experts,
                                                                   int64_t tokens, void* d_rw, int64_t d_rw_stride,
                                                                   int bf16) {
  int64_t lo = offsets[0], hi = offsets[experts];
  lo = lo < 0 ? 0 : (lo > tokens ? tokens : lo);
  hi = hi < lo ? lo : (hi > tokens ? tokens : hi);
  for (int64_t r = lo + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < hi;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float sum = 0.0f;
    for (int k = 0; k < n_tiles; ++k) sum += partials[r * n_tiles + k];
    store_rw_grad(d_rw, r * d_rw_stride, bf16, sum);
  }
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
  return fwd_entry(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                   has_linear_beta, linear_beta, out, out_row_stride, nullptr, stream);
}

situ_status_t situ_glu_fwd_mxfp8(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                                 int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype,
                                 situ_rw_mode_t rw_mode, int64_t rw_stride, double beta, int has_linear_beta,
                                 double linear_beta, void* y_data, int64_t y_data_row_stride, void* y_scale,
                                 int64_t y_scale_row_stride, situ_mx_rule_t rule, void* stream) {
  const MxOut m{static_cast<char*>(y_data), y_data_row_stride, static_cast<uint8_t*>(y_scale), y_scale_row_stride,
                static_cast<int>(rule)};
  return fwd_entry(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                   has_linear_beta, linear_beta, nullptr, 0, &m, stream);
}

size_t situ_glu_bwd_workspace_bytes(int64_t tokens, int64_t inter, situ_rw_mode_t rw_mode, int want_drw) {
  if (tokens <= 0 || inter <= 0 || !want_drw) return 0;
  uint64_t bytes = 0;
  if (rw_mode == SITU_RW_SCALAR) bytes = static_cast<uint64_t>(tokens) * sizeof(float);
  if (rw_mode == SITU_RW_COL)
    bytes = static_cast<uint64_t>((tokens + kColChunk - 1) / kColChunk) * static_cast<uint64_t>(inter) * sizeof(float);
  return static_cast<size_t>((bytes + 255) / 256 * 256);
}

}  // extern "C"

namespace {

// The backward with a native (mx == NULL) or an MXFP8 d_gate_up.
situ_status_t bwd_entry(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                        int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode,
                        int64_t rw_stride, double beta, int has_linear_beta, double linear_beta,
                        const void* grad_out, int64_t grad_out_row_stride, void* d_gate_up,
                        int64_t d_gate_up_row_stride, void* d_rw, int64_t d_rw_stride, void* workspace,
                        size_t workspace_bytes, const MxOut* mx, const Nvfp4Bwd* nv, void* stream) {
  tl_last_error[0] = '\0';
  Coeffs c;
  int gate = kGateGeneric;
  situ_status_t st = check_common(dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode,
                                  rw_stride, beta, has_linear_beta, linear_beta, &c, &gate);
  if (st != SITU_OK) return st;
  if (grad_out_row_stride < inter) return fail(SITU_ERR_INVALID_ARG, "grad_out_row_stride < inter");
  if (mx != nullptr) {
    st = check_mx_args(*mx, inter, 2 * inter, rw_mode);
    if (st != SITU_OK) return st;
  } else if (nv != nullptr) {
    st = check_nv_args(*nv, inter, 2 * inter, rw_mode);
    if (st != SITU_OK) return st;
  } else if (d_gate_up_row_stride < 2 * inter) {
    return fail(SITU_ERR_INVALID_ARG, "d_gate_up_row_stride < 2 * inter");
  }
  if (rw_mode == SITU_RW_NONE && d_rw != nullptr)
    return fail(SITU_ERR_INVALID_ARG, "d_rw must be NULL for SITU_RW_NONE");
  if (nv != nullptr && nv->amax_given == 2 && d_rw != nullptr)
    return fail(SITU_ERR_INVALID_ARG, "d_rw must be NULL when only the tensor maximum is computed");
  const bool want_drw = d_rw != nullptr;
  if (want_drw && rw_mode == SITU_RW_ROW && d_rw_stride < 1) return fail(SITU_ERR_INVALID_ARG, "d_rw_stride < 1");
  if (want_drw && rw_mode == SITU_RW_FULL && d_rw_stride < inter)
    return fail(SITU_ERR_INVALID_ARG, "d_rw_stride < inter (full weights)");
  const size_t ws_needed = situ_glu_bwd_workspace_bytes(tokens, inter, rw_mode, want_drw ? 1 : 0);
  if (tokens == 0) {
    // The gradient of a broadcast weight over zero rows is zero, and so is the
    // maximum of an empty NVFP4 gradient; nothing else is written.
    if (nv != nullptr && nv->amax_given != 1) {
      cudaError_t err = cudaMemsetAsync(nv->out.amax_out, 0, sizeof(float), static_cast<cudaStream_t>(stream));
      if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    }
    if (want_drw && (rw_mode == SITU_RW_SCALAR || rw_mode == SITU_RW_COL)) {
      if (!aligned(d_rw, elem_size(rw_dtype))) return fail(SITU_ERR_MISALIGNED, "d_rw not aligned");
      const size_t n = rw_mode == SITU_RW_COL ? static_cast<size_t>(inter) : 1;
      cudaError_t err = cudaMemsetAsync(d_rw, 0, n * elem_size(rw_dtype), static_cast<cudaStream_t>(stream));
      if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    }
    return SITU_OK;
  }
  const bool native = mx == nullptr && nv == nullptr;
  if (gate_up == nullptr || grad_out == nullptr || (native && d_gate_up == nullptr))
    return fail(SITU_ERR_INVALID_ARG, "gate_up, grad_out or d_gate_up is NULL");
  const int es = elem_size(dtype);
  const int rw_es = rw_mode == SITU_RW_NONE ? 4 : elem_size(rw_dtype);
  if (mx != nullptr) {
    st = check_mx_buffers(*mx, tokens, 2 * inter);
    if (st != SITU_OK) return st;
  }
  if (nv != nullptr && nv->amax_given != 2) {
    st = check_nv_buffers(*nv, tokens, 2 * inter);
    if (st != SITU_OK) return st;
  }
  if (!span_fits(tokens, gate_up_row_stride, 2 * inter, es) || !span_fits(tokens, grad_out_row_stride, inter, es) ||
      (native && !span_fits(tokens, d_gate_up_row_stride, 2 * inter, es)) ||
      (rw_mode == SITU_RW_ROW && !span_fits(tokens, rw_stride, 1, rw_es)) ||
      (want_drw && rw_mode == SITU_RW_ROW && !span_fits(tokens, d_rw_stride, 1, rw_es)) ||
      (rw_mode == SITU_RW_FULL && !span_fits(tokens, rw_stride, inter, rw_es)) ||
      (want_drw && rw_mode == SITU_RW_FULL && !span_fits(tokens, d_rw_stride, inter, rw_es)))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  if (!aligned(gate_up, 16) || !aligned(grad_out, 16) || (gate_up_row_stride * es) % 16 != 0 ||
      (grad_out_row_stride * es) % 16 != 0 ||
      (native && (!aligned(d_gate_up, 16) || (d_gate_up_row_stride * es) % 16 != 0)))
    return fail(SITU_ERR_MISALIGNED, "gate_up/grad_out/d_gate_up base or row pitch not 16-byte aligned");
  if (rw_mode != SITU_RW_NONE && !aligned(rw, rw_es)) return fail(SITU_ERR_MISALIGNED, "rw not aligned");
  if (want_drw && !aligned(d_rw, rw_es)) return fail(SITU_ERR_MISALIGNED, "d_rw not aligned");
  if (want_drw && rw_mode == SITU_RW_FULL &&
      (!aligned(d_rw, ew_align(dtype, rw_dtype)) || (d_rw_stride * rw_es) % ew_align(dtype, rw_dtype) != 0))
    return fail(SITU_ERR_MISALIGNED, "per-element weight gradient base or row pitch not %d-byte aligned",
                ew_align(dtype, rw_dtype));
  if (ws_needed > 0) {
    if (workspace == nullptr || workspace_bytes < ws_needed)
      return fail(SITU_ERR_INVALID_ARG, "workspace needs %zu bytes, got %zu", ws_needed,
                  workspace == nullptr ? (size_t)0 : workspace_bytes);
    if (!aligned(workspace, 16)) return fail(SITU_ERR_MISALIGNED, "workspace not 16-byte aligned");
  }

  // Aliasing: no output may overlap an input or another output.
  const Span s_gu = matrix_span(gate_up, tokens, gate_up_row_stride, 2 * inter, es);
  const Span s_go = matrix_span(grad_out, tokens, grad_out_row_stride, inter, es);
  const Span s_dgu = mx   ? matrix_span(mx->data, tokens, mx->data_pitch, 2 * inter, 1)
                    : nv ? (nv->amax_given == 2 ? Span{0, 0}
                                                : matrix_span(nv->out.data, tokens, nv->out.data_pitch, inter, 1))
                         : matrix_span(d_gate_up, tokens, d_gate_up_row_stride, 2 * inter, es);
  const Span s_rw = weight_span(rw, rw_mode, tokens, rw_stride, inter, rw_es);
  if (overlap(s_dgu, s_gu) || overlap(s_dgu, s_go) || overlap(s_dgu, s_rw))
    return fail(SITU_ERR_INVALID_ARG, "d_gate_up overlaps an input");
  const Span s_sc = mx   ? matrix_span(mx->scale, tokens, mx->scale_pitch, 2 * inter / kMxBlock, 1)
                    : nv ? (nv->amax_given == 2
                                ? Span{0, 0}
                                : matrix_span(nv->out.scale, tokens, nv->out.scale_pitch, 2 * inter / 16, 1))
                         : Span{0, 0};
  if (!native && (overlap(s_sc, s_gu) || overlap(s_sc, s_go) || overlap(s_sc, s_rw)))
    return fail(SITU_ERR_INVALID_ARG, "block scales overlap an input");
  const Span s_am = nv ? Span{reinterpret_cast<uintptr_t>(nv->out.amax_out),
                              reinterpret_cast<uintptr_t>(nv->out.amax_out) + sizeof(float)}
                       : Span{0, 0};
  if (nv != nullptr && (overlap(s_am, s_gu) || overlap(s_am, s_go) || overlap(s_am, s_rw) ||
                        overlap(s_am, s_dgu) || overlap(s_am, s_sc)))
    return fail(SITU_ERR_INVALID_ARG, "amax overlaps another tensor");
  Span s_drw = {0, 0};
  if (want_drw) {
    s_drw = weight_span(d_rw, rw_mode, tokens, d_rw_stride, inter, rw_es);
    if (overlap(s_drw, s_gu) || overlap(s_drw, s_go) || overlap(s_drw, s_rw) || overlap(s_drw, s_dgu) ||
        overlap(s_drw, s_sc) || overlap(s_drw, s_am))
      return fail(SITU_ERR_INVALID_ARG, "d_rw overlaps another tensor");
  }
  if (ws_needed > 0) {
    const Span s_ws = {reinterpret_cast<uintptr_t>(workspace), reinterpret_cast<uintptr_t>(workspace) + ws_needed};
    if (overlap(s_ws, s_gu) || overlap(s_ws, s_go) || overlap(s_ws, s_rw) || overlap(s_ws, s_dgu) ||
        overlap(s_ws, s_drw) || overlap(s_ws, s_sc) || overlap(s_ws, s_am))
      return fail(SITU_ERR_INVALID_ARG, "workspace overlaps a tensor");
  }

  if (rw_mode == SITU_RW_COL || rw_mode == SITU_RW_FULL) {
    EwArgs e{};
    e.gate_up = static_cast<const char*>(gate_up);
    e.gu_pitch = gate_up_row_stride * es;
    e.grad_out = static_cast<const char*>(grad_out);
    e.go_pitch = grad_out_row_stride * es;
    e.out = static_cast<char*>(d_gate_up);
    e.out_pitch = d_gate_up_row_stride * es;
    e.rw = static_cast<const char*>(rw);
    e.rw_pitch = rw_mode == SITU_RW_FULL ? rw_stride * rw_es : 0;
    e.d_rw = static_cast<char*>(d_rw);
    e.d_rw_pitch = rw_mode == SITU_RW_FULL ? d_rw_stride * rw_es : 0;
    e.partials = static_cast<float*>(workspace);
    e.rw_bf16 = rw_dtype == SITU_DTYPE_BF16 ? 1 : 0;
    e.tokens = tokens;
    e.half_bytes = static_cast<int>(inter * es);
    e.vpr = static_cast<int>(inter * es / kVecBytes);
    e.inter = static_cast<int>(inter);
    e.c = c;
    const bool full = rw_mode == SITU_RW_FULL;
    EwKernel k = pick_ew<true>(dtype, gate, has_linear_beta != 0, full);
    const int threads = choose_threads(e.vpr);
    // Shared memory only for the column sums of the looped form.
    const int smem = (!full && want_drw && e.vpr > 2 * threads) ? static_cast<int>(inter * sizeof(float)) : 0;
    const int64_t nchunks = full ? tokens : (tokens + kColChunk - 1) / kColChunk;
    if (smem > 48 * 1024) {  // opt in beyond the default dynamic shared-memory limit
      st = ensure_smem(reinterpret_cast<const void*>(k), smem);
      if (st != SITU_OK) return st;
    }
    int grid = 0;
    st = launch_grid(reinterpret_cast<const void*>(k), threads, smem, nchunks, &grid);
    if (st != SITU_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    k<<<grid, threads, smem, s>>>(e);
    st = check_launch("situ_glu_bwd");
    if (st != SITU_OK || rw_mode != SITU_RW_COL || !want_drw) return st;
    const int fin_grid = static_cast<int>((inter + kFinCols - 1) / kFinCols);
    situ_glu_dw_columns_finalize_kernel<<<fin_grid, kFinCols * kFinGroups, 0, s>>>(e.partials, nchunks, e.inter,
                                                                                  d_rw, e.rw_bf16);
    return check_launch("situ_glu_bwd (per-column d_rw)");
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

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (mx != nullptr) {
    auto k = pick_quant<MxQuant, true>(dtype, gate, has_linear_beta != 0);
    const int threads = choose_threads(a.vpr);
    int grid = 0;
    st = launch_grid(reinterpret_cast<const void*>(k), threads, 0, tokens, &grid);
    if (st != SITU_OK) return st;
    k<<<grid, threads, 0, s>>>(a, *mx);
    st = check_launch("situ_glu_bwd_mxfp8");
  } else if (nv != nullptr) {
    const int threads = choose_threads(a.vpr);
    if (nv->amax_given != 1) {  // the tensor maximum of d_gate_up first: a pass without stores or d_w
      cudaError_t err = cudaMemsetAsync(nv->out.amax_out, 0, sizeof(float), s);
      if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
      auto ka = pick_quant<AmaxOnly, true>(dtype, gate, has_linear_beta != 0);
      BwdArgs am = a;
      am.want_drw = 0;
      int grid = 0;
      st = launch_grid(reinterpret_cast<const void*>(ka), threads, 0, tokens, &grid);
      if (st != SITU_OK) return st;
      ka<<<grid, threads, 0, s>>>(am, reinterpret_cast<unsigned int*>(nv->out.amax_out));
      st = check_launch("situ_glu_bwd_nvfp4 (amax)");
      if (st != SITU_OK || nv->amax_given == 2) return st;
    }
    auto k = pick_quant<Nvfp4Quant, true>(dtype, gate, has_linear_beta != 0);
    int grid = 0;
    st = launch_grid(reinterpret_cast<const void*>(k), threads, 0, tokens, &grid);
    if (st != SITU_OK) return st;
    k<<<grid, threads, 0, s>>>(a, nv->out);
    st = check_launch("situ_glu_bwd_nvfp4");
  } else if (g_load_path.load(std::memory_order_relaxed) == 1) {
    StreamArgs sa{};
    sa.gate_up = a.gate_up;
    sa.gu_pitch = a.gu_pitch;
    sa.grad_out = a.grad_out;
    sa.go_pitch = a.go_pitch;
    sa.out = a.d_gate_up;
    sa.out_pitch = a.dgu_pitch;
    sa.rw = a.rw;
    sa.d_rw = a.d_rw;
    sa.d_rw_stride = a.d_rw_stride;
    sa.partials = a.partials;
    sa.want_drw = a.want_drw;
    sa.tokens = tokens;
    sa.half_bytes = a.half_bytes;
    sa.vpr = a.vpr;
    sa.c = c;
    st = launch_stream<true>(sa, dtype, gate, has_linear_beta != 0, s);
  } else {
    BwdKernel k = pick_bwd(dtype, gate, has_linear_beta != 0);
    const int threads = choose_threads(a.vpr);
    int grid = 0;
    st = launch_grid(reinterpret_cast<const void*>(k), threads, 0, tokens, &grid);
    if (st != SITU_OK) return st;
    k<<<grid, threads, 0, s>>>(a);
    st = check_launch("situ_glu_bwd");
  }
  if (st != SITU_OK) return st;
  if (want_drw && rw_mode == SITU_RW_SCALAR) {
    situ_glu_dw_scalar_finalize_kernel<<<1, kFinalizeThreads, 0, s>>>(a.partials, tokens, d_rw, a.rw.bf16);
    st = check_launch("situ_glu_bwd (scalar d_rw)");
  }
  return st;
}

}  // namespace

extern "C" {

situ_status_t situ_glu_bwd(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                           int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype,
                           situ_rw_mode_t rw_mode, int64_t rw_stride, double beta, int has_linear_beta,
                           double linear_beta, const void* grad_out, int64_t grad_out_row_stride,
                           void* d_gate_up, int64_t d_gate_up_row_stride, void* d_rw, int64_t d_rw_stride,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_entry(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                   has_linear_beta, linear_beta, grad_out, grad_out_row_stride, d_gate_up, d_gate_up_row_stride,
                   d_rw, d_rw_stride, workspace, workspace_bytes, nullptr, nullptr, stream);
}

situ_status_t situ_glu_bwd_mxfp8(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                                 int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype,
                                 situ_rw_mode_t rw_mode, int64_t rw_stride, double beta, int has_linear_beta,
                                 double linear_beta, const void* grad_out, int64_t grad_out_row_stride,
                                 void* d_gate_up_data, int64_t d_gate_up_data_row_stride, void* d_gate_up_scale,
                                 int64_t d_gate_up_scale_row_stride, situ_mx_rule_t rule, void* d_rw,
                                 int64_t d_rw_stride, void* workspace, size_t workspace_bytes, void* stream) {
  const MxOut m{static_cast<char*>(d_gate_up_data), d_gate_up_data_row_stride,
                static_cast<uint8_t*>(d_gate_up_scale), d_gate_up_scale_row_stride, static_cast<int>(rule)};
  return bwd_entry(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                   has_linear_beta, linear_beta, grad_out, grad_out_row_stride, nullptr, 0, d_rw, d_rw_stride,
                   workspace, workspace_bytes, &m, nullptr, stream);
}

situ_status_t situ_glu_bwd_nvfp4(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                                 int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype,
                                 situ_rw_mode_t rw_mode, int64_t rw_stride, double beta, int has_linear_beta,
                                 double linear_beta, const void* grad_out, int64_t grad_out_row_stride,
                                 void* d_gate_up_data, int64_t d_gate_up_data_row_stride, void* d_gate_up_scale,
                                 int64_t d_gate_up_scale_row_stride, float* amax, int amax_given, void* d_rw,
                                 int64_t d_rw_stride, void* workspace, size_t workspace_bytes, void* stream) {
  const Nvfp4Bwd nv{{static_cast<char*>(d_gate_up_data), d_gate_up_data_row_stride,
                     static_cast<uint8_t*>(d_gate_up_scale), d_gate_up_scale_row_stride, amax, amax},
                    amax_given};
  return bwd_entry(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                   has_linear_beta, linear_beta, grad_out, grad_out_row_stride, nullptr, 0, d_rw, d_rw_stride,
                   workspace, workspace_bytes, nullptr, &nv, stream);
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

int situ_glu_set_load_path(int path) {
  if (path != 0 && path != 1) return -1;
  return g_load_path.exchange(path);
}

int situ_glu_device_status(int clear) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return -1;
  if (clear && v != 0) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero) != cudaSuccess) return -1;
  }
  return v;
}

situ_status_t situ_glu_wait_probe(int64_t limit_ns, void* stream) {
  if (limit_ns < 1 || limit_ns > 10000000000LL)
    return fail(SITU_ERR_INVALID_ARG, "limit_ns %lld outside [1, 1e10]", (long long)limit_ns);
  situ_wait_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned long long>(limit_ns));
  return check_launch("situ_glu_wait_probe");
}

int situ_glu_set_max_ctas(int max_ctas) {
  if (max_ctas < 0) return -1;
  return g_max_ctas.exchange(max_ctas);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free backward
// ---------------------------------------------------------------------------
// Some callers cannot allocate device memory at the point where they run the
// backward: engines that reserve all of HBM up front and hand their kernels
// only the buffers they planned, or plain C callers with no CUDA allocator of
// their own.  situ_glu_bwd needs caller-owned scratch in two modes when the
// weight gradient is wanted (a routing weight broadcast to every row: one
// fp32 partial per row; a per-column weight: one fp32 partial per column per
// 16-row chunk).  The entry point below takes that scratch from a fixed array
// that lives in this library instead, so its caller passes only inputs and
// outputs.  The cached address is valid until the device is reset.

namespace {

constexpr int64_t kNoAllocMaxTokens = 262144;  // rows the fixed scratch can hold (1 MiB)

}  // namespace

// The fixed scratch: one copy on every GPU that loads this library, held
// until the process exits.  In host code this name is only a stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxTokens];

namespace {

std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and cached.
situ_status_t noalloc_scratch(void** addr) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(err));
  if (dev < 0 || dev >= kMaxDevices) return fail(SITU_ERR_UNSUPPORTED, "device %d beyond %d", dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess || p == nullptr)
      return fail(SITU_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(err));
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return SITU_OK;
}

}  // namespace

extern "C" situ_status_t situ_glu_bwd_no_alloc(const void* gate_up, situ_dtype_t dtype, int64_t tokens,
                                               int64_t inter, int64_t gate_up_row_stride, const void* rw,
                                               situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode, int64_t rw_stride,
                                               double beta, int has_linear_beta, double linear_beta,
                                               const void* grad_out, int64_t grad_out_row_stride, void* d_gate_up,
                                               int64_t d_gate_up_row_stride, void* d_rw, int64_t d_rw_stride,
                                               void* stream) {
  tl_last_error[0] = '\0';
  const size_t need = situ_glu_bwd_workspace_bytes(tokens, inter, rw_mode, d_rw != nullptr ? 1 : 0);
  void* ws = nullptr;
  if (need > 0) {
    if (need > sizeof(g_noalloc_scratch))
      return fail(SITU_ERR_UNSUPPORTED,
                  "situ_glu_bwd_no_alloc: %lld rows need %zu bytes of scratch; its fixed scratch holds %zu bytes "
                  "(%lld rows with a broadcast weight)",
                  (long long)tokens, need, sizeof(g_noalloc_scratch), (long long)kNoAllocMaxTokens);
    const situ_status_t st = noalloc_scratch(&ws);
    if (st != SITU_OK) return st;
  }
  // Every step runs in situ_glu_bwd; the per-row partials it writes to the
  // scratch are all written before the finishing kernel reads them, so no
  // part of the array has to start at zero.
  return situ_glu_bwd(gate_up, dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                      has_linear_beta, linear_beta, grad_out, grad_out_row_stride, d_gate_up, d_gate_up_row_stride,
                      d_rw, d_rw_stride, ws, need > 0 ? sizeof(g_noalloc_scratch) : 0, stream);
}


// ---------------------------------------------------------------------------
// FC1 grouped GEMM + SiTU-GLU forward
// ---------------------------------------------------------------------------

extern "C" situ_status_t situ_glu_fc1_fwd(const void* x, int64_t tokens, int64_t hidden, int64_t x_row_stride,
                                          const void* w1, int64_t experts, int64_t inter, int64_t w1_row_stride,
                                          const int64_t* offsets, const void* rw, situ_dtype_t rw_dtype,
                                          situ_rw_mode_t rw_mode, int64_t rw_stride, double beta,
                                          int has_linear_beta, double linear_beta, void* y, int64_t y_row_stride,
                                          void* stream) {
  tl_last_error[0] = '\0';
  if (!finite_positive(beta)) return fail(SITU_ERR_INVALID_ARG, "beta must be finite and > 0");
  if (has_linear_beta != 0 && has_linear_beta != 1)
    return fail(SITU_ERR_INVALID_ARG, "has_linear_beta must be 0 or 1");
  if (has_linear_beta && !finite_positive(linear_beta))
    return fail(SITU_ERR_INVALID_ARG, "linear_beta must be finite and > 0");
  if (rw_mode != SITU_RW_ROW && rw_mode != SITU_RW_SCALAR && rw_mode != SITU_RW_NONE)
    return fail(rw_mode == SITU_RW_COL || rw_mode == SITU_RW_FULL ? SITU_ERR_UNSUPPORTED : SITU_ERR_INVALID_ARG,
                "situ_glu_fc1_fwd takes per-row, broadcast or no routing weights");
  if (rw_mode != SITU_RW_NONE && !valid_dtype(rw_dtype))
    return fail(SITU_ERR_INVALID_ARG, "rw_dtype %d is not a situ_dtype_t", (int)rw_dtype);
  if (tokens < 0) return fail(SITU_ERR_INVALID_ARG, "tokens = %lld < 0", (long long)tokens);
  if (hidden < fc1::kBK || hidden % fc1::kBK != 0)
    return fail(SITU_ERR_UNSUPPORTED, "hidden must be a positive multiple of %d, got %lld", fc1::kBK,
                (long long)hidden);
  if (inter < fc1::kBN || inter % fc1::kBN != 0)
    return fail(SITU_ERR_UNSUPPORTED, "inter must be a positive multiple of %d, got %lld", fc1::kBN,
                (long long)inter);
  if (experts < 1 || experts > fc1::kMaxExperts)
    return fail(SITU_ERR_UNSUPPORTED, "experts must be in [1, %d], got %lld", fc1::kMaxExperts, (long long)experts);
  if (tokens > INT32_MAX || experts * 2 * inter > INT32_MAX || hidden > INT32_MAX)
    return fail(SITU_ERR_UNSUPPORTED, "sizes exceed the 32-bit tensor-map coordinates");
  if (x_row_stride < hidden || w1_row_stride < hidden || y_row_stride < inter)
    return fail(SITU_ERR_INVALID_ARG, "a row stride is shorter than its row");
  if (rw_mode == SITU_RW_ROW && rw_stride < 0) return fail(SITU_ERR_INVALID_ARG, "rw_stride < 0");
  if (tokens == 0) return SITU_OK;
  if (x == nullptr || w1 == nullptr || offsets == nullptr || y == nullptr ||
      (rw_mode != SITU_RW_NONE && rw == nullptr))
    return fail(SITU_ERR_INVALID_ARG, "x, w1, offsets, y or rw is NULL");
  if (rw_mode == SITU_RW_NONE && rw != nullptr) return fail(SITU_ERR_INVALID_ARG, "rw must be NULL for SITU_RW_NONE");
  if (!span_fits(tokens, x_row_stride, hidden, 2) || !span_fits(experts * 2 * inter, w1_row_stride, hidden, 2) ||
      !span_fits(tokens, y_row_stride, inter, 2) ||
      (rw_mode == SITU_RW_ROW && !span_fits(tokens, rw_stride, 1, elem_size(rw_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  if (!aligned(x, 16) || !aligned(w1, 16) || !aligned(y, 16) || (x_row_stride * 2) % 16 != 0 ||
      (w1_row_stride * 2) % 16 != 0 || (y_row_stride * 2) % 16 != 0 || !aligned(offsets, 8) ||
      (rw_mode != SITU_RW_NONE && !aligned(rw, elem_size(rw_dtype))))
    return fail(SITU_ERR_MISALIGNED, "x, w1, y (16 bytes), offsets (8) or rw base or row pitch misaligned");
  const Span s_y = matrix_span(y, tokens, y_row_stride, inter, 2);
  const Span s_off = {reinterpret_cast<uintptr_t>(offsets),
                      reinterpret_cast<uintptr_t>(offsets) + static_cast<uintptr_t>(experts + 1) * 8};
  if (overlap(s_y, matrix_span(x, tokens, x_row_stride, hidden, 2)) ||
      overlap(s_y, matrix_span(w1, experts * 2 * inter, w1_row_stride, hidden, 2)) || overlap(s_y, s_off) ||
      overlap(s_y, weight_span(rw, rw_mode, tokens, rw_stride, inter, elem_size(rw_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "y overlaps an input");

  fc1::Args a{};
  a.offsets = offsets;
  a.experts = static_cast<int>(experts);
  a.tokens = tokens;
  a.hidden = static_cast<int>(hidden);
  a.inter = static_cast<int>(inter);
  a.rw = {rw, rw_stride, static_cast<int>(rw_mode), (rw_mode != SITU_RW_NONE && rw_dtype == SITU_DTYPE_BF16) ? 1 : 0};
  a.y = static_cast<char*>(y);
  a.y_pitch = y_row_stride * 2;
  int gate = kGateGeneric;
  fill_coeffs(beta, has_linear_beta, linear_beta, &a.c, &gate);

  CUtensorMap mx, mw;
  situ_status_t st = bf16_tile_map(&mx, x, hidden, tokens, x_row_stride);
  if (st != SITU_OK) return st;
  st = bf16_tile_map(&mw, w1, hidden, experts * 2 * inter, w1_row_stride);
  if (st != SITU_OK) return st;

  return launch_fused(pick_fused<fc1::Fc1Epilogue>(gate, has_linear_beta != 0), mx, mw, a, experts,
                      static_cast<cudaStream_t>(stream), "situ_glu_fc1_fwd");
}

// ---------------------------------------------------------------------------
// FC2 data gradient + SiTU-GLU backward
// ---------------------------------------------------------------------------

extern "C" size_t situ_glu_fc2_dgrad_workspace_bytes(int64_t tokens, int64_t inter, int want_drw) {
  if (tokens <= 0 || inter <= 0 || !want_drw) return 0;
  const uint64_t bytes = static_cast<uint64_t>(tokens) * static_cast<uint64_t>(inter / fc1::kUmmaN) * sizeof(float);
  return static_cast<size_t>((bytes + 255) / 256 * 256);
}

extern "C" situ_status_t situ_glu_fc2_dgrad_bwd(const void* dout, int64_t tokens, int64_t hidden,
                                                int64_t dout_row_stride, const void* w2t, int64_t experts,
                                                int64_t inter, int64_t w2t_row_stride, const int64_t* offsets,
                                                const void* gate_up, int64_t gate_up_row_stride, const void* rw,
                                                situ_dtype_t rw_dtype, situ_rw_mode_t rw_mode, int64_t rw_stride,
                                                double beta, int has_linear_beta, double linear_beta,
                                                void* d_gate_up, int64_t d_gate_up_row_stride, void* d_rw,
                                                int64_t d_rw_stride, void* workspace, size_t workspace_bytes,
                                                void* stream) {
  tl_last_error[0] = '\0';
  if (!finite_positive(beta)) return fail(SITU_ERR_INVALID_ARG, "beta must be finite and > 0");
  if (has_linear_beta != 0 && has_linear_beta != 1)
    return fail(SITU_ERR_INVALID_ARG, "has_linear_beta must be 0 or 1");
  if (has_linear_beta && !finite_positive(linear_beta))
    return fail(SITU_ERR_INVALID_ARG, "linear_beta must be finite and > 0");
  if (rw_mode != SITU_RW_ROW && rw_mode != SITU_RW_NONE)
    return fail(rw_mode == SITU_RW_SCALAR || rw_mode == SITU_RW_COL || rw_mode == SITU_RW_FULL ? SITU_ERR_UNSUPPORTED
                                                                                                : SITU_ERR_INVALID_ARG,
                "situ_glu_fc2_dgrad_bwd takes per-row or no routing weights");
  if (rw_mode != SITU_RW_NONE && !valid_dtype(rw_dtype))
    return fail(SITU_ERR_INVALID_ARG, "rw_dtype %d is not a situ_dtype_t", (int)rw_dtype);
  if (rw_mode == SITU_RW_NONE && (rw != nullptr || d_rw != nullptr))
    return fail(SITU_ERR_INVALID_ARG, "rw and d_rw must be NULL for SITU_RW_NONE");
  if (tokens < 0) return fail(SITU_ERR_INVALID_ARG, "tokens = %lld < 0", (long long)tokens);
  if (hidden < fc1::kBK || hidden % fc1::kBK != 0)
    return fail(SITU_ERR_UNSUPPORTED, "hidden must be a positive multiple of %d, got %lld", fc1::kBK,
                (long long)hidden);
  if (inter < fc1::kUmmaN || inter % fc1::kUmmaN != 0)
    return fail(SITU_ERR_UNSUPPORTED, "inter must be a positive multiple of %d, got %lld", fc1::kUmmaN,
                (long long)inter);
  if (experts < 1 || experts > fc1::kMaxExperts)
    return fail(SITU_ERR_UNSUPPORTED, "experts must be in [1, %d], got %lld", fc1::kMaxExperts, (long long)experts);
  if (tokens > INT32_MAX || experts * inter > INT32_MAX || hidden > INT32_MAX)
    return fail(SITU_ERR_UNSUPPORTED, "sizes exceed the 32-bit tensor-map coordinates");
  if (dout_row_stride < hidden || w2t_row_stride < hidden || gate_up_row_stride < 2 * inter ||
      d_gate_up_row_stride < 2 * inter)
    return fail(SITU_ERR_INVALID_ARG, "a row stride is shorter than its row");
  if (rw_mode == SITU_RW_ROW && (rw_stride < 0 || (d_rw != nullptr && d_rw_stride < 1)))
    return fail(SITU_ERR_INVALID_ARG, "rw_stride < 0 or d_rw_stride < 1");
  const bool want_drw = d_rw != nullptr;
  const size_t ws_needed = situ_glu_fc2_dgrad_workspace_bytes(tokens, inter, want_drw ? 1 : 0);
  if (tokens == 0) return SITU_OK;
  if (dout == nullptr || w2t == nullptr || offsets == nullptr || gate_up == nullptr || d_gate_up == nullptr ||
      (rw_mode == SITU_RW_ROW && rw == nullptr))
    return fail(SITU_ERR_INVALID_ARG, "dout, w2t, offsets, gate_up, d_gate_up or rw is NULL");
  if (!span_fits(tokens, dout_row_stride, hidden, 2) || !span_fits(experts * inter, w2t_row_stride, hidden, 2) ||
      !span_fits(tokens, gate_up_row_stride, 2 * inter, 2) || !span_fits(tokens, d_gate_up_row_stride, 2 * inter, 2) ||
      (rw_mode == SITU_RW_ROW && !span_fits(tokens, rw_stride, 1, elem_size(rw_dtype))) ||
      (want_drw && !span_fits(tokens, d_rw_stride, 1, elem_size(rw_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  if (!aligned(dout, 16) || !aligned(w2t, 16) || !aligned(gate_up, 16) || !aligned(d_gate_up, 16) ||
      (dout_row_stride * 2) % 16 != 0 || (w2t_row_stride * 2) % 16 != 0 || (gate_up_row_stride * 2) % 16 != 0 ||
      (d_gate_up_row_stride * 2) % 16 != 0 || !aligned(offsets, 8) ||
      (rw_mode == SITU_RW_ROW && !aligned(rw, elem_size(rw_dtype))) ||
      (want_drw && !aligned(d_rw, elem_size(rw_dtype))))
    return fail(SITU_ERR_MISALIGNED, "a base address or row pitch is misaligned");
  if (ws_needed > 0 && (workspace == nullptr || workspace_bytes < ws_needed || !aligned(workspace, 16)))
    return fail(SITU_ERR_INVALID_ARG, "workspace needs %zu bytes (16-byte aligned), got %zu", ws_needed,
                workspace == nullptr ? (size_t)0 : workspace_bytes);
  const Span s_dgu = matrix_span(d_gate_up, tokens, d_gate_up_row_stride, 2 * inter, 2);
  const Span s_ws = {reinterpret_cast<uintptr_t>(workspace), reinterpret_cast<uintptr_t>(workspace) + ws_needed};
  const Span s_off = {reinterpret_cast<uintptr_t>(offsets),
                      reinterpret_cast<uintptr_t>(offsets) + static_cast<uintptr_t>(experts + 1) * 8};
  const Span ins[] = {matrix_span(dout, tokens, dout_row_stride, hidden, 2),
                      matrix_span(w2t, experts * inter, w2t_row_stride, hidden, 2),
                      matrix_span(gate_up, tokens, gate_up_row_stride, 2 * inter, 2), s_off,
                      weight_span(rw, rw_mode, tokens, rw_stride, inter, elem_size(rw_dtype))};
  const Span s_drw = want_drw ? weight_span(d_rw, SITU_RW_ROW, tokens, d_rw_stride, inter, elem_size(rw_dtype))
                              : Span{0, 0};
  for (const Span& in : ins)
    if (overlap(s_dgu, in) || overlap(s_drw, in) || (ws_needed && overlap(s_ws, in)))
      return fail(SITU_ERR_INVALID_ARG, "an output or the workspace overlaps an input");
  if (overlap(s_dgu, s_drw) || (ws_needed && (overlap(s_ws, s_dgu) || overlap(s_ws, s_drw))))
    return fail(SITU_ERR_INVALID_ARG, "outputs or the workspace overlap each other");

  fc1::Args a{};
  a.offsets = offsets;
  a.experts = static_cast<int>(experts);
  a.tokens = tokens;
  a.hidden = static_cast<int>(hidden);
  a.inter = static_cast<int>(inter);
  a.rw = {rw, rw_stride, static_cast<int>(rw_mode), (rw_mode != SITU_RW_NONE && rw_dtype == SITU_DTYPE_BF16) ? 1 : 0};
  a.y = static_cast<char*>(d_gate_up);
  a.y_pitch = d_gate_up_row_stride * 2;
  a.gate_up = static_cast<const char*>(gate_up);
  a.gu_pitch = gate_up_row_stride * 2;
  a.partials = want_drw ? static_cast<float*>(workspace) : nullptr;
  int gate = kGateGeneric;
  fill_coeffs(beta, has_linear_beta, linear_beta, &a.c, &gate);

  CUtensorMap ma, mb;
  situ_status_t st = bf16_tile_map(&ma, dout, hidden, tokens, dout_row_stride);
  if (st != SITU_OK) return st;
  st = bf16_tile_map(&mb, w2t, hidden, experts * inter, w2t_row_stride);
  if (st != SITU_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_fused(pick_fused<fc1::Fc2Epilogue>(gate, has_linear_beta != 0), ma, mb, a, experts, s,
                    "situ_glu_fc2_dgrad_bwd");
  if (st != SITU_OK || !want_drw) return st;
  int sms = 0;
  st = device_sm_count(&sms);
  if (st != SITU_OK) return st;
  situ_fc2_dw_finalize_kernel<<<sms, 256, 0, s>>>(a.partials, static_cast<int>(inter / fc1::kUmmaN), offsets,
                                                  static_cast<int>(experts), tokens, d_rw, d_rw_stride,
                                                  a.rw.bf16);
  return check_launch("situ_glu_fc2_dgrad_bwd (d_rw)");
}


// ---------------------------------------------------------------------------
// Attention-residual mixing core
// ---------------------------------------------------------------------------

extern "C" situ_status_t situ_attn_res_fwd(const void* blocks, int64_t nblocks, int64_t block_row_stride,
                                           int64_t block_stride, const void* prefix, int64_t prefix_row_stride,
                                           situ_dtype_t dtype, int64_t tokens, int64_t hidden,
                                           const void* norm_weight, situ_dtype_t norm_dtype,
                                           const void* proj_weight, situ_dtype_t proj_dtype, double variance_epsilon,
                                           void* out, situ_dtype_t out_dtype, int64_t out_row_stride,
                                           void* stream) {
  tl_last_error[0] = '\0';
  if (!valid_dtype(dtype) || !valid_dtype(norm_dtype) || !valid_dtype(proj_dtype) || !valid_dtype(out_dtype))
    return fail(SITU_ERR_INVALID_ARG, "a dtype is not a situ_dtype_t");
  if (nblocks < 0) return fail(SITU_ERR_INVALID_ARG, "nblocks < 0");
  const int64_t sources = nblocks + (prefix != nullptr ? 1 : 0);
  if (sources < 1 || sources > kArMaxSources)
    return fail(SITU_ERR_UNSUPPORTED, "sources (blocks plus the prefix sum) must be in [1, %d], got %lld",
                kArMaxSources, (long long)sources);
  if (tokens < 0) return fail(SITU_ERR_INVALID_ARG, "tokens = %lld < 0", (long long)tokens);
  if (hidden <= 0) return fail(SITU_ERR_INVALID_ARG, "hidden = %lld <= 0", (long long)hidden);
  if (hidden > 32768) return fail(SITU_ERR_UNSUPPORTED, "hidden = %lld exceeds 32768", (long long)hidden);
  if (!std::isfinite(variance_epsilon) || variance_epsilon < 0.0)
    return fail(SITU_ERR_INVALID_ARG, "variance_epsilon must be finite and >= 0");
  if ((nblocks > 0 && (block_row_stride < hidden || block_stride < hidden)) ||
      (prefix != nullptr && prefix_row_stride < hidden) || out_row_stride < hidden)
    return fail(SITU_ERR_INVALID_ARG, "a stride is shorter than a row");
  const int es = elem_size(dtype), oes = elem_size(out_dtype);
  if ((hidden * es) % 16 != 0)
    return fail(SITU_ERR_MISALIGNED, "hidden * element size (%lld bytes) is not a multiple of 16",
                (long long)(hidden * es));
  if (tokens == 0) return SITU_OK;
  if ((nblocks > 0 && blocks == nullptr) || norm_weight == nullptr || proj_weight == nullptr || out == nullptr)
    return fail(SITU_ERR_INVALID_ARG, "blocks, norm_weight, proj_weight or out is NULL");
  // a token's sources span (nblocks - 1) block strides plus one row; the
  // tokens then add (tokens - 1) row strides to that
  if ((nblocks > 0 && (!span_fits(nblocks, block_stride, hidden, es) ||
                       !span_fits(tokens, block_row_stride, (nblocks - 1) * block_stride + hidden, es))) ||
      (prefix != nullptr && !span_fits(tokens, prefix_row_stride, hidden, es)) ||
      !span_fits(tokens, out_row_stride, hidden, oes))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  if ((nblocks > 0 && (!aligned(blocks, 16) || (block_row_stride * es) % 16 != 0 || (block_stride * es) % 16 != 0)) ||
      (prefix != nullptr && (!aligned(prefix, 16) || (prefix_row_stride * es) % 16 != 0)) || !aligned(out, 16) ||
      (out_row_stride * oes) % 16 != 0 || !aligned(norm_weight, elem_size(norm_dtype)) ||
      !aligned(proj_weight, elem_size(proj_dtype)))
    return fail(SITU_ERR_MISALIGNED, "a base address or row pitch is misaligned");
  const Span s_out = matrix_span(out, tokens, out_row_stride, hidden, oes);
  if ((nblocks > 0 && overlap(s_out, matrix_span(blocks, tokens, block_row_stride, (nblocks - 1) * block_stride + hidden,
                                                  es))) ||
      (prefix != nullptr && overlap(s_out, matrix_span(prefix, tokens, prefix_row_stride, hidden, es))) ||
      overlap(s_out, matrix_span(norm_weight, 1, hidden, hidden, elem_size(norm_dtype))) ||
      overlap(s_out, matrix_span(proj_weight, 1, hidden, hidden, elem_size(proj_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "out overlaps an input");

  ArArgs a{};
  a.blocks = static_cast<const char*>(blocks);
  a.block_row_pitch = block_row_stride * es;
  a.block_pitch = block_stride * es;
  a.prefix = static_cast<const char*>(prefix);
  a.prefix_row_pitch = prefix_row_stride * es;
  a.nblocks = static_cast<int>(nblocks);
  a.sources = static_cast<int>(sources);
  a.tokens = tokens;
  a.hidden = static_cast<int>(hidden);
  a.vpr = static_cast<int>(hidden * es / kVecBytes);
  a.norm_w = norm_weight;
  a.norm_bf16 = norm_dtype == SITU_DTYPE_BF16;
  a.proj_w = proj_weight;
  a.proj_bf16 = proj_dtype == SITU_DTYPE_BF16;
  a.eps = static_cast<float>(variance_epsilon);
  a.inv_hidden = static_cast<float>(1.0 / static_cast<double>(hidden));
  a.out = static_cast<char*>(out);
  a.out_pitch = out_row_stride * oes;
  a.out_bf16 = out_dtype == SITU_DTYPE_BF16;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t stage_bytes = sources * hidden * es;
  if (a.vpr <= 1024 && sources <= kArStagedSources && stage_bytes <= 180 * 1024) {
    auto staged = [&](auto kb, auto kf, int vecs) -> situ_status_t {
      const void* ks = dtype == SITU_DTYPE_BF16 ? reinterpret_cast<const void*>(kb) : reinterpret_cast<const void*>(kf);
      const int threads = ((a.vpr + vecs - 1) / vecs + 31) / 32 * 32;
      const int smem = static_cast<int>(stage_bytes);
      if (smem > 48 * 1024) {
        situ_status_t st = ensure_smem(ks, smem);
        if (st != SITU_OK) return st;
      }
      int grid = 0;
      situ_status_t st = launch_grid(ks, threads, smem, tokens, &grid);
      if (st != SITU_OK) return st;
      if (dtype == SITU_DTYPE_BF16)
        kb<<<grid, threads, smem, s>>>(a);
      else
        kf<<<grid, threads, smem, s>>>(a);
      return check_launch("situ_attn_res_fwd");
    };
    // Two column vectors per thread once a row has at least 128: 5 % faster
    // than one at hidden 7168 (the per-row reductions and the softmax
    // broadcast are paid once per two vectors); four were 7 % slower (seven
    // warps per SM leave the row's dependent steps exposed).
    if (a.vpr > 2 * 448)
      return staged(situ_attn_res_staged_kernel<Bf16, 2, 512>, situ_attn_res_staged_kernel<F32, 2, 512>, 2);
    if (a.vpr >= 128)
      return staged(situ_attn_res_staged_kernel<Bf16, 2, 448>, situ_attn_res_staged_kernel<F32, 2, 448>, 2);
    return staged(situ_attn_res_staged_kernel<Bf16, 1, kArStagedThreads>,
                  situ_attn_res_staged_kernel<F32, 1, kArStagedThreads>, 1);
  }
  const void* k = dtype == SITU_DTYPE_BF16 ? reinterpret_cast<const void*>(situ_attn_res_kernel<Bf16>)
                                           : reinterpret_cast<const void*>(situ_attn_res_kernel<F32>);
  const int threads = a.vpr >= kArThreads ? kArThreads : (a.vpr + 31) / 32 * 32;
  const int smem = static_cast<int>(hidden * sizeof(float));
  if (smem > 48 * 1024) {
    situ_status_t st = ensure_smem(k, smem);
    if (st != SITU_OK) return st;
  }
  int grid = 0;
  situ_status_t st = launch_grid(k, threads, smem, tokens, &grid);
  if (st != SITU_OK) return st;
  if (dtype == SITU_DTYPE_BF16)
    situ_attn_res_kernel<Bf16><<<grid, threads, smem, s>>>(a);
  else
    situ_attn_res_kernel<F32><<<grid, threads, smem, s>>>(a);
  return check_launch("situ_attn_res_fwd");
}


// ---------------------------------------------------------------------------
// NVFP4 forward
// ---------------------------------------------------------------------------

extern "C" situ_status_t situ_glu_fwd_nvfp4(const void* gate_up, situ_dtype_t dtype, int64_t tokens, int64_t inter,
                                            int64_t gate_up_row_stride, const void* rw, situ_dtype_t rw_dtype,
                                            situ_rw_mode_t rw_mode, int64_t rw_stride, double beta,
                                            int has_linear_beta, double linear_beta, void* y_data,
                                            int64_t y_data_row_stride, void* y_scale, int64_t y_scale_row_stride,
                                            float* amax, int amax_given, void* stream) {
  tl_last_error[0] = '\0';
  Coeffs c;
  int gate = kGateGeneric;
  situ_status_t st = check_common(dtype, tokens, inter, gate_up_row_stride, rw, rw_dtype, rw_mode, rw_stride, beta,
                                  has_linear_beta, linear_beta, &c, &gate);
  if (st != SITU_OK) return st;
  if (inter % 16 != 0)
    return fail(SITU_ERR_INVALID_ARG, "NVFP4 outputs need inter a multiple of 16, got %lld", (long long)inter);
  if (rw_mode == SITU_RW_COL || rw_mode == SITU_RW_FULL)
    return fail(SITU_ERR_UNSUPPORTED, "NVFP4 outputs take per-row, broadcast or no routing weights");
  if (amax_given < 0 || amax_given > 2) return fail(SITU_ERR_INVALID_ARG, "amax_given must be 0, 1 or 2");
  const bool amax_only = amax_given == 2;  // the tensor maximum alone: no codes, no scales
  if (!amax_only && (y_data_row_stride < inter / 2 || y_scale_row_stride < inter / 16))
    return fail(SITU_ERR_INVALID_ARG, "NVFP4 data or scale row pitch shorter than a row");
  if (amax == nullptr) return fail(SITU_ERR_INVALID_ARG, "amax is NULL");
  if (!aligned(amax, 4)) return fail(SITU_ERR_MISALIGNED, "amax not 4-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (tokens == 0) {
    if (amax_given != 1) {
      cudaError_t err = cudaMemsetAsync(amax, 0, sizeof(float), s);
      if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    }
    return SITU_OK;
  }
  if (gate_up == nullptr || (!amax_only && (y_data == nullptr || y_scale == nullptr)))
    return fail(SITU_ERR_INVALID_ARG, "gate_up, y_data or y_scale is NULL");
  const int es = elem_size(dtype);
  if (!span_fits(tokens, gate_up_row_stride, 2 * inter, es) ||
      (!amax_only && (!span_fits(tokens, y_data_row_stride, inter / 2, 1) ||
                      !span_fits(tokens, y_scale_row_stride, inter / 16, 1))) ||
      (rw_mode == SITU_RW_ROW && !span_fits(tokens, rw_stride, 1, elem_size(rw_dtype))))
    return fail(SITU_ERR_INVALID_ARG, "tensor extent overflows int64");
  // a thread stores the codes of one 16-byte input vector: 4 bytes (bf16) or 2 (fp32)
  if (!aligned(gate_up, 16) || (gate_up_row_stride * es) % 16 != 0 ||
      (!amax_only && (!aligned(y_data, 4) || y_data_row_stride % 4 != 0)) ||
      (rw_mode != SITU_RW_NONE && !aligned(rw, elem_size(rw_dtype))))
    return fail(SITU_ERR_MISALIGNED,
                "gate_up base or row pitch not 16-byte aligned, y_data base or row pitch not 4-byte aligned, or rw "
                "misaligned");
  const Span s_gu = matrix_span(gate_up, tokens, gate_up_row_stride, 2 * inter, es);
  const Span s_rw = weight_span(rw, rw_mode, tokens, rw_stride, inter, elem_size(rw_dtype));
  const Span s_d = amax_only ? Span{0, 0} : matrix_span(y_data, tokens, y_data_row_stride, inter / 2, 1);
  const Span s_s = amax_only ? Span{0, 0} : matrix_span(y_scale, tokens, y_scale_row_stride, inter / 16, 1);
  const Span s_a = {reinterpret_cast<uintptr_t>(amax), reinterpret_cast<uintptr_t>(amax) + 4};
  const Span outs[] = {s_d, s_s, s_a};
  for (int i = 0; i < 3; ++i) {
    if (overlap(outs[i], s_gu) || overlap(outs[i], s_rw)) return fail(SITU_ERR_INVALID_ARG, "an output overlaps an input");
    for (int k = i + 1; k < 3; ++k)
      if (overlap(outs[i], outs[k])) return fail(SITU_ERR_INVALID_ARG, "outputs overlap each other");
  }
  FwdArgs a;
  a.gate_up = static_cast<const char*>(gate_up);
  a.gu_pitch = gate_up_row_stride * es;
  a.out = nullptr;
  a.out_pitch = 0;
  a.rw = {rw, rw_stride, static_cast<int>(rw_mode), (rw_mode != SITU_RW_NONE && rw_dtype == SITU_DTYPE_BF16) ? 1 : 0};
  a.tokens = tokens;
  a.half_bytes = static_cast<int>(inter * es);
  a.vpr = static_cast<int>(inter * es / kVecBytes);
  a.c = c;
  const int threads = choose_threads(a.vpr);
  if (amax_given != 1) {
    cudaError_t err = cudaMemsetAsync(amax, 0, sizeof(float), s);
    if (err != cudaSuccess) return fail(SITU_ERR_CUDA, "cudaMemsetAsync: %s", cudaGetErrorString(err));
    auto ka = pick_quant<AmaxOnly, false>(dtype, gate, has_linear_beta != 0);
    int grid = 0;
    st = launch_grid(reinterpret_cast<const void*>(ka), threads, 0, tokens, &grid);
    if (st != SITU_OK) return st;
    ka<<<grid, threads, 0, s>>>(a, reinterpret_cast<unsigned int*>(amax));
    st = check_launch("situ_glu_fwd_nvfp4 (amax)");
    if (st != SITU_OK || amax_only) return st;
  }
  const Nvfp4Out m{static_cast<char*>(y_data), y_data_row_stride, static_cast<uint8_t*>(y_scale), y_scale_row_stride,
                   amax, amax};
  auto k = pick_quant<Nvfp4Quant, false>(dtype, gate, has_linear_beta != 0);
  int grid = 0;
  st = launch_grid(reinterpret_cast<const void*>(k), threads, 0, tokens, &grid);
  if (st != SITU_OK) return st;
  k<<<grid, threads, 0, s>>>(a, m);
  return check_launch("situ_glu_fwd_nvfp4");
}
