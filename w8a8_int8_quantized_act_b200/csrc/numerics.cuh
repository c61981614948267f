// Scalar numerics shared by the kernels: symmetric quantisation, the exponential used by
// SiLU, and the dequant / gated-activation arithmetic. Every floating-point step that decides
// an integer code (or a bf16 value that is later quantised) is an explicit round-to-nearest
// fp32 operation, so the results are reproducible bit for bit.
#pragma once
#include "ptx.cuh"

namespace w8a8 {

// Symmetric int8: codes in [-127, 127] (num_bits 8, symmetric, as in the group_0 block of the
// Qwen3.6-35B-A3B-w8a8 config page); int4: codes in [-7, 7].
constexpr float kQMaxInt8 = 127.0f;
constexpr float kQMaxInt4 = 7.0f;

// scale = amax / q_max (IEEE divide); 0 when the row is all zeros.
__device__ __forceinline__ float sym_scale(float amax, float qmax) { return __fdiv_rn(amax, qmax); }

// code = clamp(round_half_even(v / scale), -q_max, q_max); 0 when scale is 0.
__device__ __forceinline__ int sym_code(float v, float scale, int qmax) {
  if (scale == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(v, scale));
  return max(-qmax, min(qmax, q));
}

// The same code, with the divide replaced by a multiply where that cannot change the result:
// y = v * rcp_rn(scale) is within 2.3e-5 of fl(v / scale) when |v / scale| <= 127 (two
// round-to-nearest steps, 2^-24 relative each, plus fl(v/scale)'s own half ulp), so if y lies
// more than 3e-5 from every half-integer both round to the same integer; the few values that
// land closer take the true divide. inv = __frcp_rn(scale), computed once per row.
__device__ __forceinline__ int sym_code_fast(float v, float scale, float inv, int qmax) {
  if (scale == 0.0f) return 0;
  const float y = __fmul_rn(v, inv);
  const float f = y - floorf(y);
  int q;
  if (fabsf(f - 0.5f) > 3e-5f) {
    q = __float2int_rn(y);
  } else {
    q = __float2int_rn(__fdiv_rn(v, scale));
  }
  return max(-qmax, min(qmax, q));
}

// exp(x) by Cody-Waite range reduction (ln 2 split into a 15-significant-bit high part and a
// low part) and a degree-7 Taylor polynomial evaluated by Horner's rule with fused
// multiply-adds, then an exact scaling by 2^n. x > 88 -> +inf, x < -87 -> 0.
//   n = rint(x * log2 e); r = fma(-n, ln2_lo, fma(-n, ln2_hi, x)); p = fma(p, r, 1/i!)
// rint(y) for |y| < 2^22 is y + 1.5*2^23 rounded to nearest-even, minus 1.5*2^23 (both steps
// exact apart from that one rounding), and the low bits of the biased sum are n itself.
// exp_cw_core is that computation for -87 <= x <= 88 (where n lies in [-126, 127]).
__device__ __forceinline__ float exp_cw_core(float x) {
  const float log2e = (float)1.4426950408889634;
  const float ln2_hi = (float)0.693145751953125;
  const float ln2_lo = (float)(0.6931471805599453 - 0.693145751953125);
  const float kRound = 12582912.0f;  // 1.5 * 2^23
  const float t = __fadd_rn(__fmul_rn(x, log2e), kRound);
  const float n = __fsub_rn(t, kRound);
  const float r = __fmaf_rn(-n, ln2_lo, __fmaf_rn(-n, ln2_hi, x));
  float p = (float)(1.0 / 5040.0);
  p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  // n + 127 in the exponent field; n = bits(t) - bits(1.5 * 2^23)
  const float two_n = __uint_as_float((__float_as_uint(t) - 0x4B400000u + 127u) << 23);
  return __fmul_rn(p, two_n);
}

// Branch-free: x is clamped to [-87, 88] and the out-of-range results are selected at the end.
__device__ __forceinline__ float exp_cw(float x) {
  const float xc = fminf(fmaxf(x, -87.0f), 88.0f);
  float v = exp_cw_core(xc);
  v = (x > 88.0f) ? __int_as_float(0x7f800000) : v;
  v = (x < -87.0f) ? 0.0f : v;
  return (x != x) ? x : v;
}

// SiLU(g) = g / (1 + exp(-g)) with a true divide.
__device__ __forceinline__ float silu_exact(float g) { return __fdiv_rn(g, __fadd_rn(1.0f, exp_cw(-g))); }

// q = g / d rounded to nearest-even (the IEEE quotient) for d >= 1, without a branch; `ok`
// is false where the fast path cannot prove its answer, and the caller then takes __fdiv_rn.
//   y  ~ 1/d  (hardware approximation, relative error below 2^-22)
//   q0 = fl(g*y); r0 = fma(-d, q0, g); q1 = fma(r0, y, q0)
// The correction step is Markstein's (IBM J. Res. Dev. 34(1), 1990): its pre-rounding value is
// within 2^-44 relative of g/d, so q1 is a faithful rounding, and then r1 = g - d*q1 is exact
// (the remainder of a faithful quotient is a float when nothing underflows; here |q1| >= 2^-100
// and d >= 1). q1 is the nearest float to g/d iff |g/d - q1| < ulp(q1)/2, i.e. iff
// |r1| < (ulp(q1)/2)*d, a product that is exact (a power of two times d). A q1 whose
// significand is 1.0 (the gap below it is half as wide), an exact tie, a non-finite or a tiny
// q1 is not certified; g = 0 returns g (signed zero). r1 = 0 means q1 is the exact quotient.
__device__ __forceinline__ float div_certified(float g, float d, bool& ok) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(d));
  const float q0 = __fmul_rn(g, y);
  const float r0 = __fmaf_rn(-d, q0, g);
  const float q1 = __fmaf_rn(r0, y, q0);
  const float r1 = __fmaf_rn(-d, q1, g);
  const uint32_t qa = __float_as_uint(q1) & 0x7FFFFFFFu;
  const float half_ulp_d = __fmul_rn(__uint_as_float((qa & 0x7F800000u) - (24u << 23)), d);
  const bool in_range = qa >= 0x0D800000u && qa < 0x7F800000u;  // 2^-100 <= |q1| < inf
  const bool nearest = (r1 == 0.0f) || (fabsf(r1) < half_ulp_d && (qa & 0x007FFFFFu) != 0u);
  ok = (g == 0.0f) || (in_range && nearest);
  return (g == 0.0f) ? g : q1;
}

// bf16(fl(SiLU(g) * u)), the gated activation as the layer defines it, S = fl(fl(g / d) * u)
// with d = fl(1 + exp_cw(-g)), evaluated cheaply and certified at the bf16 level:
//   x = -g * log2(e) as xh + xl (xh = fl(-g * L), xl its exact FMA residual plus -g * (log2 e - L));
//   e' = 2^xh (ex2.approx) * (1 + xl ln 2);  d' = fl(1 + e');  Y = fl(fl(g * rcp.approx(d')) * u).
// Error: e' is within eps_ex2 + 2^-23 of e^-g (the split leaves |xl| <= 2^-18, so the first-order
// correction is exact to 2^-36); exp_cw is within 3 ulp (6 * 2^-24) of it; hence
// |d'/d - 1| <= eps_ex2 + 10 * 2^-24, and with the reciprocal's eps_rcp and four fp32 roundings,
// |Y/S - 1| <= eps_ex2 + eps_rcp + 14 * 2^-24. GPU tests measure ex2.approx within 3 ulp and
// rcp.approx within 2 ulp of the correctly rounded results (eps <= 7 and 5 * 2^-24), so Y is
// within 26 fp32 ulps of S whenever Y is a normal number. bf16 rounding looks only at the low 16
// bits of the fp32 pattern (round up above 0x8000, ties to even at 0x8000), so if those bits of Y
// are more than kBf16Margin = 40 ulps away from 0x8000, S lies in the same bf16 rounding interval
// and bf16(Y) = bf16(S). (Near a binade boundary the low bits are near 0 or 0xFFFF and both round
// to the same power of two.) Accepted only for |g| <= 64 (d < 2^93, every step in range) and
// 2^-120 <= |Y| < 2^121; `ok` is false otherwise, and the caller then evaluates silu_exact.
constexpr uint32_t kBf16Margin = 40;
__device__ __forceinline__ float silu_mul_bf16_certified(float g, float u, bool& ok) {
  const float L = 1.44269502162933349609375f;                  // fl(log2 e)
  const float Llo = (float)(1.4426950408889634 - 1.44269502162933349609375);
  const float ng = -g;
  const float xh = __fmul_rn(ng, L);
  float xl = __fmaf_rn(ng, L, -xh);
  xl = __fmaf_rn(ng, Llo, xl);
  float e1;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e1) : "f"(xh));
  const float e = __fmaf_rn(e1, __fmul_rn(xl, 0.693147180559945309f), e1);
  const float d = __fadd_rn(1.0f, e);
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
  const float y = __fmul_rn(__fmul_rn(g, r), u);
  const uint32_t b = __float_as_uint(y);
  const bool normal = ((b >> 23) & 0xFFu) - 7u < 241u;
  const bool clear_of_tie = (((b ^ 0x8000u) + kBf16Margin) & 0xFFFFu) > 2u * kBf16Margin;
  ok = (fabsf(g) <= 64.0f) && normal && clear_of_tie;
  return y;
}

// ((float)acc * s_row) * s_col, each product rounded to fp32.
__device__ __forceinline__ float dequant(int32_t acc, float s_row, float s_col) {
  return __fmul_rn(__fmul_rn(__int2float_rn(acc), s_row), s_col);
}

// Codes of 8 bf16 values (one 16-byte vector) packed into 8 bytes; inv = __frcp_rn(s).
// Each value: y = v * inv; r = y + 1.5 * 2^23 rounds y to the nearest integer, ties to even,
// exactly as __float2int_rn for |y| < 2^22, and the low byte of r's bit pattern is that integer
// as an int8 code (|y| <= 127 * (1 + 2^-22) here, so no clamp is needed). d = y - rint(y) is
// exact; |d| >= 0.5 - 3e-5 is the same near-tie test as sym_code_fast, and a vector holding such a
// value takes the true divide for all eight. A row whose amax is below about 2^-121 has a
// subnormal scale whose reciprocal overflows to +inf: y is then +-inf or NaN, d is NaN, and the
// test is written so that NaN also counts as unsure and takes the true divide.
// The products and sums run two values at a time (packed f32x2 operations, each lane rounded to
// nearest like the scalar operation, subnormals kept).
__device__ __forceinline__ uint2 quant8(const uint4 v, float s, float inv) {
  if (s == 0.0f) return make_uint2(0u, 0u);
  const uint64_t inv2 = (uint64_t(__float_as_uint(inv)) << 32) | __float_as_uint(inv);
  const uint64_t mag2 = (uint64_t(0x4B400000u) << 32) | 0x4B400000u;  // 1.5 * 2^23 in both halves
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[8];
  bool unsure = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint32_t r0, r1, d0, d1;
    asm("{\n\t.reg .b64 x, y, r, t, d;\n\t"
        "mov.b64 x, {%4, %5};\n\t"
        "mul.rn.f32x2 y, x, %6;\n\t"
        "add.rn.f32x2 r, y, %7;\n\t"
        "sub.rn.f32x2 t, r, %7;\n\t"
        "sub.rn.f32x2 d, y, t;\n\t"
        "mov.b64 {%0, %1}, r;\n\t"
        "mov.b64 {%2, %3}, d;\n\t}"
        : "=r"(r0), "=r"(r1), "=r"(d0), "=r"(d1)
        : "r"(w[j] << 16), "r"(w[j] & 0xFFFF0000u), "l"(inv2), "l"(mag2));
    unsure |= !(fabsf(__uint_as_float(d0)) < 0.49997f) || !(fabsf(__uint_as_float(d1)) < 0.49997f);
    c[2 * j] = r0;
    c[2 * j + 1] = r1;
  }
  if (unsure) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      c[2 * j] = uint32_t(sym_code(bf16_lo(w[j]), s, 127));
      c[2 * j + 1] = uint32_t(sym_code(bf16_hi(w[j]), s, 127));
    }
  }
  const uint32_t lo = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040), 0x5410);
  return make_uint2(lo, hi);
}

// max |v| over 8 bf16 values: with the sign bits cleared, the 16-bit patterns of finite bf16
// values (subnormals included) order like the values, so a per-halfword unsigned maximum is exact.
__device__ __forceinline__ float amax8(const uint4 v) {
  const uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                              __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
  return __uint_as_float((m > 0xFFFFu ? (m >> 16) > (m & 0xFFFFu) ? m >> 16 : m & 0xFFFFu : m) << 16);
}

// Quantises one row of K bf16 values with one warp (K a multiple of 8, row 16-byte aligned):
// returns the scale; `emit(i, packed8)` receives the 8 codes of elements i..i+7. With U > 0 the
// row (at most 256 * U values) is read once into registers, every load in flight together;
// U = 0 reads rows of any length twice.
template <int U, typename Emit>
__device__ __forceinline__ float quant_row_warp(const uint16_t* __restrict__ src, int K, Emit emit) {
  const int lane = threadIdx.x & 31;
  if constexpr (U > 0) {
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = lane * 8 + u * 256;
      v[u] = (i < K) ? __ldg(reinterpret_cast<const uint4*>(src + i)) : make_uint4(0, 0, 0, 0);
    }
    float amax = 0.0f;
#pragma unroll
    for (int u = 0; u < U; ++u) amax = fmaxf(amax, amax8(v[u]));
    amax = warp_max(amax);
    const float s = sym_scale(amax, kQMaxInt8);
    const float inv = __frcp_rn(s);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = lane * 8 + u * 256;
      if (i < K) emit(i, quant8(v[u], s, inv));
    }
    return s;
  } else {
    float amax = 0.0f;
    for (int i = lane * 8; i < K; i += 256)
      amax = fmaxf(amax, amax8(__ldg(reinterpret_cast<const uint4*>(src + i))));
    amax = warp_max(amax);
    const float s = sym_scale(amax, kQMaxInt8);
    const float inv = __frcp_rn(s);
    for (int i = lane * 8; i < K; i += 256)
      emit(i, quant8(__ldg(reinterpret_cast<const uint4*>(src + i)), s, inv));
    return s;
  }
}

// Registers-per-lane choice for a row of K values: 0 (two passes) beyond 4096.
inline int row_units(int K) {
  const int u = (K + 255) / 256;
  return u <= 1 ? 1 : u <= 2 ? 2 : u <= 4 ? 4 : u <= 8 ? 8 : u <= 16 ? 16 : 0;
}

}  // namespace w8a8
