// MXFP8 A8W8 (the "MXFP A8w8" row of the accuracy table, section 六 of the AMCT Qwen3-Next page),
// read as the OCP Microscaling FP8 format: blocks of 32 consecutive values along K share one
// power-of-two scale 2^E, stored as the E8M0 byte E + 127, and every element is an FP8 E4M3 byte.
//   E = floor(log2(max |v| over the block)) - 8, clamped to [-127, 127]; a block of zeros takes
//       E = -127 (8 is the exponent of E4M3's largest binade, whose top value is 448);
//   element = E4M3(v * 2^-E), nearest with ties to even, saturating at 448, sign kept at zero.
// The dense MXFP8 linear multiplies the dequantised operands P * 2^E. Each of them is exact in
// bf16 (at most 4 significant bits, and 2^E inside bf16's exponent range), and each product of two
// is exact in fp32, so the tcgen05 kind::f16 MMA on the dequantised bf16 operands computes the MX
// GEMM's sum of products with only its fp32 accumulation rounding; the block-scaled FP8 MMA would
// compute the same sum at twice the rate.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "elementwise.cuh"

namespace w8a8 {

constexpr int kMxBlock = 32;
constexpr int kMxWarps = 8;  // warps per CTA; a warp takes 256 values (8 blocks) of one row

// floor(log2 v) of a nonzero bf16 magnitude pattern (sign bit clear), subnormals included.
__device__ __forceinline__ int bf16_floor_log2(uint32_t mag) {
  const int eb = int(mag >> 7);
  if (eb > 0) return eb - 127;
  return (31 - __clz(int(mag))) - 133;  // a subnormal is m * 2^-133, m its 7-bit mantissa
}

// E4M3 bytes of (lo, hi) in the low and high byte: nearest, ties to even, saturating at 448
// (cvt.rn.satfinite.e4m3x2).
__device__ __forceinline__ uint32_t e4m3_pair(float lo, float hi) {
  return uint32_t(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// 2^E as an fp32 value for E in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2_f32(int E) {
  return E >= -126 ? __int_as_float((E + 127) << 23) : __int_as_float(0x00400000);
}

// Eight elements of one block with the block's scale 2^E into bf16 values P * 2^E, packed. The
// E4M3 -> fp16 conversion and the power-of-two product are exact.
__device__ __forceinline__ uint4 mx_dequant8(uint2 codes, float scale) {
  uint32_t out[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w = (i < 2) ? codes.x : codes.y;
    const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2(__nv_fp8x2_storage_t((w >> ((i & 1) * 16)) & 0xFFFFu),
                                                      __NV_E4M3);
    const float2 f = __half22float2(__half2(h2));
    const __nv_bfloat162 b = __floats2bfloat162_rn(__fmul_rn(f.x, scale), __fmul_rn(f.y, scale));
    out[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// codes [R, K] (E4M3 bytes), scales [R, K / 32] (E8M0 bytes) of the bf16 rows src [R, K], and,
// when deq is not null, the dequantised values P * 2^E as bf16 [R, K]. K is a multiple of 32.
// Lane l of a warp holds values 8l .. 8l+7 of its 256-value piece: block l / 4, four lanes each.
__global__ void __launch_bounds__(kMxWarps * 32) mx_quant_rows_kernel(const uint16_t* __restrict__ src,
                                                                      int64_t R, int K,
                                                                      uint8_t* __restrict__ codes,
                                                                      uint8_t* __restrict__ scales,
                                                                      uint16_t* __restrict__ deq) {
  pdl_wait();
  pdl_launch_dependents();
  const int pieces = (K + 255) / 256;
  const int64_t item = int64_t(blockIdx.x) * kMxWarps + (threadIdx.x >> 5);
  if (item >= R * pieces) return;  // warp-uniform
  const int64_t r = item / pieces;
  const int lane = threadIdx.x & 31;
  const int k0 = int(item - r * pieces) * 256 + lane * 8;
  const bool valid = k0 < K;  // K % 32 == 0: whole blocks are valid or not
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (valid) v = __ldg(reinterpret_cast<const uint4*>(src + r * K + k0));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  // block maximum of the magnitudes: compared as unsigned bf16 patterns with the sign cleared
  uint32_t mag = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) mag = max(mag, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
  mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, 1));
  mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, 2));
  const int E = mag == 0 ? -127 : min(127, max(-127, bf16_floor_log2(mag) - 8));
  const float inv = __int_as_float((127 - E) << 23);  // 2^-E, exact (E <= 119 for bf16 input)
  uint32_t c[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    c[i >> 1] |= e4m3_pair(__fmul_rn(bf16_lo(w[i]), inv), __fmul_rn(bf16_hi(w[i]), inv)) << (16 * (i & 1));
  if (!valid) return;
  *reinterpret_cast<uint2*>(codes + r * K + k0) = make_uint2(c[0], c[1]);
  if ((lane & 3) == 0) scales[r * (K / kMxBlock) + k0 / kMxBlock] = uint8_t(E + 127);
  if (deq != nullptr) *reinterpret_cast<uint4*>(deq + r * K + k0) = mx_dequant8(make_uint2(c[0], c[1]), pow2_f32(E));
}

// The dequantised bf16 values P * 2^(scale - 127) of MXFP8 rows (codes [R, K], scales [R, K / 32]).
__global__ void __launch_bounds__(kMxWarps * 32) mx_dequant_rows_kernel(const uint8_t* __restrict__ codes,
                                                                        const uint8_t* __restrict__ scales,
                                                                        int64_t R, int K,
                                                                        uint16_t* __restrict__ deq) {
  pdl_wait();
  pdl_launch_dependents();
  const int pieces = (K + 255) / 256;
  const int64_t item = int64_t(blockIdx.x) * kMxWarps + (threadIdx.x >> 5);
  if (item >= R * pieces) return;
  const int64_t r = item / pieces;
  const int k0 = int(item - r * pieces) * 256 + (threadIdx.x & 31) * 8;
  if (k0 >= K) return;
  const uint2 c = __ldg(reinterpret_cast<const uint2*>(codes + r * K + k0));
  const int E = int(__ldg(scales + r * (K / kMxBlock) + k0 / kMxBlock)) - 127;
  *reinterpret_cast<uint4*>(deq + r * K + k0) = mx_dequant8(c, pow2_f32(E));
}

}  // namespace w8a8
