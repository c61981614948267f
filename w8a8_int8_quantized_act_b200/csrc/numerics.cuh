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
__device__ __forceinline__ float exp_cw(float x) {
  if (x > 88.0f) return __int_as_float(0x7f800000);
  if (x < -87.0f) return 0.0f;
  const float log2e = (float)1.4426950408889634;
  const float ln2_hi = (float)0.693145751953125;
  const float ln2_lo = (float)(0.6931471805599453 - 0.693145751953125);
  const float n = rintf(__fmul_rn(x, log2e));
  const float r = __fmaf_rn(-n, ln2_lo, __fmaf_rn(-n, ln2_hi, x));
  float p = (float)(1.0 / 5040.0);
  p = __fmaf_rn(p, r, (float)(1.0 / 720.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 120.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 24.0));
  p = __fmaf_rn(p, r, (float)(1.0 / 6.0));
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const float two_n = __int_as_float((static_cast<int>(n) + 127) << 23);
  return __fmul_rn(p, two_n);
}

// SiLU(g) = g / (1 + exp(-g)) with a true divide.
__device__ __forceinline__ float silu_exact(float g) { return __fdiv_rn(g, __fadd_rn(1.0f, exp_cw(-g))); }

// ((float)acc * s_row) * s_col, each product rounded to fp32.
__device__ __forceinline__ float dequant(int32_t acc, float s_row, float s_col) {
  return __fmul_rn(__fmul_rn(__int2float_rn(acc), s_row), s_col);
}

// Codes of 8 bf16 values (one 16-byte vector) packed into 8 bytes; inv = __frcp_rn(s).
__device__ __forceinline__ uint2 quant8(const uint4 v, float s, float inv) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t lo = 0, hi = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t a = uint32_t(sym_code_fast(bf16_lo(w[j]), s, inv, 127)) & 0xFFu;
    const uint32_t b = uint32_t(sym_code_fast(bf16_hi(w[j]), s, inv, 127)) & 0xFFu;
    const uint32_t pair = a | (b << 8);
    if (j < 2) lo |= pair << (16 * j); else hi |= pair << (16 * (j - 2));
  }
  return make_uint2(lo, hi);
}

__device__ __forceinline__ float amax8(const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.0f;
#pragma unroll
  for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_lo(w[j])), fabsf(bf16_hi(w[j]))));
  return m;
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
