// numerics.cuh - bit-exact fp32 building blocks of the AWQ scale table and INT4 group quantizer.
//
// Every quantity that is part of the result (scales, codes, steps, zeros) is formed by single IEEE
// fp32 operations with round-to-nearest-even, through the __f*_rn intrinsics so that the compiler can
// neither contract them into FMAs nor reorder them.
#pragma once
#include <cstdint>

namespace awq {

// Constants of the method, as exact fp32 values (nearest fp32 to the decimal constants).
#define AWQ_SCALE_FLOOR 0x1.a36e2ep-14f  // 1e-4: clamp(min=1e-4) of the powered statistic
#define AWQ_STEP_FLOOR 0x1.4f8b58p-17f   // 1e-5: clamp(min=1e-5) of the quantization step

// ===================================================================================================
// Correctly rounded fp32 power a^r for a >= 0 (fp32) and r in [0, 1) (fp32).
//
// Fast path: the fp64 pow of the CUDA math library (documented error <= 2 ulp of fp64). Its result is
// rounded to fp32; that rounding is the correctly rounded one unless the fp64 value lies within a few
// fp64 ulps of a point halfway between two fp32 numbers. The guard below sends every value within 2^11
// fp64 ulps of such a midpoint to the slow path (about one value in 2^17).
//
// Slow path: a^r = exp(r * ln a) in double-double arithmetic (about 100 significant bits), built from
// the error-free transforms TwoSum (Knuth), Fast2Sum and the FMA-based TwoProduct (Dekker 1971), with
// ln by the series 2*atanh((m-1)/(m+1)) and exp by Taylor series after range reduction and 2^9
// squarings; then an exact comparison of the double-double value with the fp32 midpoint.
// ===================================================================================================
struct dd {
  double hi, lo;
};

__device__ __forceinline__ dd two_sum(double a, double b) {
  double s = __dadd_rn(a, b);
  double bb = __dsub_rn(s, a);
  double e = __dadd_rn(__dsub_rn(a, __dsub_rn(s, bb)), __dsub_rn(b, bb));
  return {s, e};
}
__device__ __forceinline__ dd quick_two_sum(double a, double b) {  // requires |a| >= |b|
  double s = __dadd_rn(a, b);
  double e = __dsub_rn(b, __dsub_rn(s, a));
  return {s, e};
}
__device__ __forceinline__ dd two_prod(double a, double b) {
  double p = __dmul_rn(a, b);
  double e = __fma_rn(a, b, -p);
  return {p, e};
}
__device__ __forceinline__ dd dd_add(dd a, dd b) {
  dd s = two_sum(a.hi, b.hi);
  dd t = two_sum(a.lo, b.lo);
  s.lo = __dadd_rn(s.lo, t.hi);
  s = quick_two_sum(s.hi, s.lo);
  s.lo = __dadd_rn(s.lo, t.lo);
  return quick_two_sum(s.hi, s.lo);
}
__device__ __forceinline__ dd dd_neg(dd a) { return {-a.hi, -a.lo}; }
__device__ __forceinline__ dd dd_sub(dd a, dd b) { return dd_add(a, dd_neg(b)); }
__device__ __forceinline__ dd dd_mul(dd a, dd b) {
  dd p = two_prod(a.hi, b.hi);
  p.lo = __dadd_rn(p.lo, __dadd_rn(__dmul_rn(a.hi, b.lo), __dmul_rn(a.lo, b.hi)));
  return quick_two_sum(p.hi, p.lo);
}
__device__ __forceinline__ dd dd_mul_d(dd a, double b) {
  dd p = two_prod(a.hi, b);
  p.lo = __dadd_rn(p.lo, __dmul_rn(a.lo, b));
  return quick_two_sum(p.hi, p.lo);
}
__device__ __forceinline__ dd dd_div(dd a, dd b) {
  double q1 = __ddiv_rn(a.hi, b.hi);
  dd r = dd_sub(a, dd_mul_d(b, q1));
  double q2 = __ddiv_rn(r.hi, b.hi);
  r = dd_sub(r, dd_mul_d(b, q2));
  double q3 = __ddiv_rn(r.hi, b.hi);
  dd q = quick_two_sum(q1, q2);
  return dd_add(q, dd{q3, 0.0});
}
__device__ __forceinline__ dd dd_ldexp(dd a, int e) { return {ldexp(a.hi, e), ldexp(a.lo, e)}; }

// ln 2 as a double-double (hi + lo = ln 2 to about 107 bits).
__device__ __forceinline__ dd dd_ln2() { return {0x1.62e42fefa39efp-1, 0x1.abc9e3b39803fp-56}; }

// ln(a) for a > 0 finite.
__device__ __noinline__ dd dd_log(double a) {
  int e = 0;
  double m = frexp(a, &e);  // a = m 2^e, m in [0.5, 1)
  if (m < 0.70710678118654752) {
    m = ldexp(m, 1);
    e -= 1;
  }  // m in [1/sqrt2, sqrt2)
  dd u = dd_div(dd{__dsub_rn(m, 1.0), 0.0}, dd{__dadd_rn(m, 1.0), 0.0});  // |u| <= 0.1716
  dd v = dd_mul(u, u);                                                     // v <= 0.0295
  // atanh(u)/u = sum_{n>=0} v^n / (2n+1); 28 terms leave a tail below 2^-140.
  dd s = dd_div(dd{1.0, 0.0}, dd{57.0, 0.0});
#pragma unroll 1
  for (int n = 27; n >= 0; --n) s = dd_add(dd_mul(s, v), dd_div(dd{1.0, 0.0}, dd{2.0 * n + 1.0, 0.0}));
  dd lnm = dd_mul_d(dd_mul(u, s), 2.0);
  return dd_add(dd_mul_d(dd_ln2(), static_cast<double>(e)), lnm);
}

// exp(x) for |x| < 700.
__device__ __noinline__ dd dd_exp(dd x) {
  const dd ln2 = dd_ln2();
  double k = rint(__ddiv_rn(x.hi, ln2.hi));
  dd r = dd_sub(x, dd_mul_d(ln2, k));  // |r| <= ~0.35
  r = dd_ldexp(r, -9);                  // |r| <= ~7e-4
  // expm1(r) = r + r^2/2! + ... ; 14 terms leave a tail below 2^-150.
  dd term = r;
  dd sum = r;
#pragma unroll 1
  for (int n = 2; n <= 14; ++n) {
    term = dd_div(dd_mul(term, r), dd{static_cast<double>(n), 0.0});
    sum = dd_add(sum, term);
  }
  // (1 + a)^2 - 1 = 2a + a^2, applied 9 times, undoes the 2^-9 scaling without losing the small part.
#pragma unroll 1
  for (int i = 0; i < 9; ++i) sum = dd_add(dd_mul_d(sum, 2.0), dd_mul(sum, sum));
  dd y = dd_add(dd{1.0, 0.0}, sum);
  return dd_ldexp(y, static_cast<int>(k));
}

// Nearest fp32 to the double-double value y (positive, inside the normal fp32 range).
__device__ __forceinline__ float dd_to_f32_rn(dd y) {
  float f = __double2float_rn(y.hi);
  const double fd = static_cast<double>(f);
  const double d = __dadd_rn(__dsub_rn(y.hi, fd), y.lo);  // y - f (y.hi - fd is exact)
  const float up = nextafterf(f, __int_as_float(0x7f800000));
  const float dn = nextafterf(f, 0.0f);
  const double half_up = 0.5 * (static_cast<double>(up) - fd);
  const double half_dn = 0.5 * (fd - static_cast<double>(dn));
  if (d > half_up || (d == half_up && (__float_as_uint(f) & 1u))) return up;
  if (d < -half_dn || (d == -half_dn && (__float_as_uint(f) & 1u))) return dn;
  return f;
}

__device__ __noinline__ float pow_f32_slow(float a, float r) {
  dd L = dd_log(static_cast<double>(a));
  dd x = dd_mul_d(L, static_cast<double>(r));
  return dd_to_f32_rn(dd_exp(x));
}

// Values below this are certainly below the 1e-4 floor after rounding, so their exact rounding does
// not matter: max(t, 1e-4) replaces them.
#define AWQ_POW_IRRELEVANT 5.0e-5

__device__ __forceinline__ float pow_f32_cr(float a, float r, bool force_slow) {
  if (r == 0.0f) return 1.0f;
  if (a == 0.0f) return 0.0f;
  const double y = pow(static_cast<double>(a), static_cast<double>(r));
  if (y < AWQ_POW_IRRELEVANT) return 0.0f;
  if (!force_slow) {
    const uint64_t low = static_cast<uint64_t>(__double_as_longlong(y)) & ((1ull << 29) - 1ull);
    const int64_t off = static_cast<int64_t>(low) - (1ll << 28);
    if (off > (1ll << 11) || off < -(1ll << 11)) return __double2float_rn(y);
  }
  return pow_f32_slow(a, r);
}

// Same correctly rounded power for results that matter below the 1e-4 floor as well (the scale variants
// divide or normalise before clamping): no shortcut for small results, and every result below the
// smallest normal fp32 (where fewer mantissa bits remain) goes through the double-double path.
__device__ __forceinline__ float pow_f32_cr_full(float a, float r, bool force_slow) {
  if (r == 0.0f) return 1.0f;
  if (a == 0.0f) return 0.0f;
  const double y = pow(static_cast<double>(a), static_cast<double>(r));
  if (!force_slow && y >= 0x1p-126) {
    const uint64_t low = static_cast<uint64_t>(__double_as_longlong(y)) & ((1ull << 29) - 1ull);
    const int64_t off = static_cast<int64_t>(low) - (1ll << 28);
    if (off > (1ll << 11) || off < -(1ll << 11)) return __double2float_rn(y);
  }
  return pow_f32_slow(a, r);
}

#define AWQ_WEIGHT_EPS 0x1.0c6f7ap-20f   // 1e-6 added to the powered weight mean (weight-aware scales)
#define AWQ_RMS_ACT_FLOOR 0x1.4f8b58p-17f  // 1e-5 floor of the statistic (RMS-normalised scales)

// ===================================================================================================
// Asymmetric 4-bit group quantizer (section 二 of the gsyq.cn AWQ page), fp32, one rounding per step.
// ===================================================================================================
struct GroupParams {
  float step;   // max(RN32(RN32(max - min) / 15), 1e-5)
  float zero;   // rint(RN32(-min / step)), -0 turned into +0
  float rstep;  // RN32(1 / step), used only to find the quotient quickly (see code_of)
};

__device__ __forceinline__ GroupParams group_params(float mx, float mn) {
  GroupParams g;
  g.step = fmaxf(__fdiv_rn(__fsub_rn(mx, mn), 15.0f), AWQ_STEP_FLOOR);
  g.zero = __fadd_rn(rintf(__fdiv_rn(-mn, g.step)), 0.0f);
  g.rstep = __frcp_rn(g.step);
  return g;
}

// Exact rint(RN32(wp / step)) through the IEEE division; kept out of line so that the common path
// below issues no division instructions.
__device__ __noinline__ float rint_quotient_exact(float wp, float step) { return rintf(__fdiv_rn(wp, step)); }

// rint(RN32(wp / step)) exactly. For |qa| < 128 the product qa = wp * RN32(1/step) is within
// 1.5 * 2^-23 * 128 < 2.3e-5 of the real quotient, and RN32 moves the quotient by at most 2^-17, so the
// two round to the same integer whenever qa is farther than 2^-14 (6.1e-5) from a half-integer. Only the
// rare remaining cases (about one element in 10^4, and groups with the step at its floor) divide.
__device__ __forceinline__ float rint_quotient(float wp, const GroupParams& g, bool exact) {
  const float qa = __fmul_rn(wp, g.rstep);
  float n = rintf(qa);
  const float d = fabsf(__fsub_rn(qa, n));  // exact: n is within a factor 2 of qa, or n = 0
  if (exact || !(d < 0.5f - 0x1p-14f && fabsf(qa) < 128.0f)) n = rint_quotient_exact(wp, g.step);
  return n;
}

// Code q = min(max(RN32(rint(RN32(w'/step)) + z), 0), 15).
__device__ __forceinline__ float code_of(float wp, const GroupParams& g, bool exact) {
  const float q = __fadd_rn(rint_quotient(wp, g, exact), g.zero);
  return fminf(fmaxf(q, 0.0f), 15.0f);
}

// INT8 symmetric per-channel code q = min(max(rint(RN32(w'/step)), -127), 127) (g.zero is 0).
__device__ __forceinline__ float code_of_int8(float wp, const GroupParams& g, bool exact) {
  return fminf(fmaxf(rint_quotient(wp, g, exact), -127.0f), 127.0f);
}

// Per-channel INT8 parameters from the row's max |w'|: step = max(RN32(amax / 127), 1e-5), zero 0.
__device__ __forceinline__ GroupParams int8_params(float amax) {
  GroupParams g;
  g.step = fmaxf(__fdiv_rn(amax, 127.0f), AWQ_STEP_FLOOR);
  g.zero = 0.0f;
  g.rstep = __frcp_rn(g.step);
  return g;
}

// deq = RN32(RN32(q - z) * step)
__device__ __forceinline__ float dequant(float q, const GroupParams& g) {
  return __fmul_rn(__fsub_rn(q, g.zero), g.step);
}

// ===================================================================================================
// Paired fp32 arithmetic of sm_100 (add/sub/mul .rn.f32x2): two fp32 values in one 64-bit register,
// each lane an ordinary IEEE operation rounded to nearest (the same bits as two scalar __f*_rn
// operations, never contracted), issued as one instruction. Three-input min/max of sm_100.
// ===================================================================================================
__device__ __forceinline__ uint64_t fx2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void fx2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fx2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fx2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fx2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fx2_fma(uint64_t a, uint64_t b, uint64_t c) {  // a * b + c, one rounding
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// ===================================================================================================
// Fast path of the group quantizer, bit-identical to code_of / dequant where it applies.
//
// With C = M + z, M = 1.5 * 2^23, every float in [2^23, 2^24) is an integer, so
//   t = RN(qa + C), qa = RN(w' * RN(1/step)),
// is C + rint(qa) whenever qa is not a tie (z is an integer, |z| < 2^21), r = t - C = rint(qa) exactly,
// and d = qa - r is exact (r is 0 or within a factor 2 of qa). By the argument of rint_quotient,
// |d| < 0.5 - 2^-14 and |qa| < 128 make r = rint(RN(w' / step)); then the unclamped code is r + z and
// t = M + code. The group-level conditions (fast_group):
//   |z| < 2^21;  RN(max(|max|, |min|) * rstep) < 128 (bounds every |qa| by monotonicity of rounding);
//   the t of the group's min and max elements lie in [M, M + 15] (t is monotone in w', so every code
//   of the group lies in [0, 15] and the clamp is the identity).
// The element-level condition |d| < 0.5 - 2^-14 is checked as the max over a lane's elements; a lane
// that fails it (a quotient within 2^-14 of a half-integer, about one element in 10^4) redoes its
// elements with code_of. In the fast path the low byte of t's bit pattern is the code (M = 0x4B400000),
// and RN32(q - z) = r, so the dequantized value is RN(r * step).
// ===================================================================================================
constexpr float kQuantMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kTieMargin = 0.5f - 0x1p-14f;
constexpr float kTieMarginSq = 0.24993896484375f;  // RN32(kTieMargin^2) = RN32(0.25 - 2^-14 + 2^-28) = 0.25 - 2^-14

__device__ __forceinline__ bool fast_group(const GroupParams& g, float mx, float mn, float& C) {
  if (!(fabsf(g.zero) < 2097152.0f)) return false;
  if (!(__fmul_rn(fmaxf(fabsf(mx), fabsf(mn)), g.rstep) < 128.0f)) return false;
  C = __fadd_rn(kQuantMagic, g.zero);
  const float t_mx = __fadd_rn(__fmul_rn(mx, g.rstep), C);
  const float t_mn = __fadd_rn(__fmul_rn(mn, g.rstep), C);
  return t_mn >= kQuantMagic && t_mx <= kQuantMagic + 15.0f;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

}  // namespace awq
