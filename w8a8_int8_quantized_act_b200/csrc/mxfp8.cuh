// MXFP8 A8W8 (the "MXFP A8w8" row of the accuracy table, section 六 of the AMCT Qwen3-Next page),
// read as the OCP Microscaling FP8 format: blocks of 32 consecutive values along K share one
// power-of-two scale 2^E, stored as the E8M0 byte E + 127, and every element is an FP8 E4M3 byte.
//   E = floor(log2(max |v| over the block)) - 8, clamped to [-127, 127]; a block of zeros takes
//       E = -127 (8 is the exponent of E4M3's largest binade, whose top value is 448);
//   element = E4M3(v * 2^-E), nearest with ties to even, saturating at 448, sign kept at zero.
// The dense MXFP8 linear runs on the block-scaled FP8 MMA, which takes the codes and the E8M0
// scales as they are and sums the products in fp32.
// MXFP A8W4 (the "MXFP A8w4" row of the same table): the same MXFP8 activations against MXFP4
// weights, the OCP format with FP4 E2M1 elements (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6):
//   E = floor(log2(max |v| over the block)) - 2 (2 is the exponent of E2M1's largest binade);
//   element = E2M1(v * 2^-E), nearest with ties to even, saturating at 6, sign kept at zero;
//   two codes per byte, element 2i in the low nibble of byte i.
// The GEMM kernels below take either weight format: E2M1 weights are loaded by TMA as packed
// 4-bit data (the 16U4_ALIGN16B tensor-map type), which lands in shared memory as 8 bytes of 16
// codes followed by 8 bytes of padding, the operand layout the MMA reads for 4-bit elements of
// kind::mxf8f6f4; the MMA then multiplies E2M1 weights by E4M3 tokens directly.
#pragma once
#include <cuda_fp4.h>
#include <cuda_fp8.h>

#include "elementwise.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"

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

// codes [R, K] (E4M3 bytes), scales [R, K / 32] (E8M0 bytes) of the bf16 rows src [R, K]. K is a
// multiple of 32.
// Lane l of a warp holds values 8l .. 8l+7 of its 256-value piece: block l / 4, four lanes each.
__global__ void __launch_bounds__(kMxWarps * 32) mx_quant_rows_kernel(const uint16_t* __restrict__ src,
                                                                      int64_t R, int K,
                                                                      uint8_t* __restrict__ codes,
                                                                      uint8_t* __restrict__ scales) {
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
}

// E2M1 codes of (lo, hi) in the low and high nibble of a byte: nearest, ties to even, saturating
// at 6 (cvt.rn.satfinite.e2m1x2).
__device__ __forceinline__ uint32_t e2m1_pair(float lo, float hi) {
  return uint32_t(__nv_cvt_float2_to_fp4x2(make_float2(lo, hi), __NV_E2M1, cudaRoundNearest));
}

// MXFP4 weights of the bf16 rows src [R, K]: packed [R, K / 2] (two E2M1 codes per byte, the even
// element low), scales [R, K / 32] (E8M0 bytes). K is a multiple of 32. The same split of the work
// as mx_quant_rows_kernel: lane l holds values 8l .. 8l+7 of its warp's 256-value piece.
__global__ void __launch_bounds__(kMxWarps * 32) mx4_quant_rows_kernel(const uint16_t* __restrict__ src,
                                                                       int64_t R, int K,
                                                                       uint8_t* __restrict__ packed,
                                                                       uint8_t* __restrict__ scales) {
  pdl_wait();
  pdl_launch_dependents();
  const int pieces = (K + 255) / 256;
  const int64_t item = int64_t(blockIdx.x) * kMxWarps + (threadIdx.x >> 5);
  if (item >= R * pieces) return;  // warp-uniform
  const int64_t r = item / pieces;
  const int lane = threadIdx.x & 31;
  const int k0 = int(item - r * pieces) * 256 + lane * 8;
  const bool valid = k0 < K;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (valid) v = __ldg(reinterpret_cast<const uint4*>(src + r * K + k0));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t mag = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) mag = max(mag, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
  mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, 1));
  mag = max(mag, __shfl_xor_sync(0xffffffffu, mag, 2));
  const int E = mag == 0 ? -127 : min(127, max(-127, bf16_floor_log2(mag) - 2));
  const float inv = __int_as_float((127 - E) << 23);  // 2^-E, a normal float (E <= 125 for bf16 input)
  uint32_t c = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) c |= e2m1_pair(__fmul_rn(bf16_lo(w[i]), inv), __fmul_rn(bf16_hi(w[i]), inv)) << (8 * i);
  if (!valid) return;
  *reinterpret_cast<uint32_t*>(packed + r * (K / 2) + k0 / 2) = c;
  if ((lane & 3) == 0) scales[r * (K / kMxBlock) + k0 / kMxBlock] = uint8_t(E + 127);
}

// ---------------------------------------------------------------- block-scaled MXFP8 GEMM
// y[t, n] = bf16(sum_k (P_x[t,k] 2^Ex[t,k/32]) (P_w[n,k] 2^Ew[n,k/32])) with the block-scaled FP8
// MMA (tcgen05.mma kind::mxf8f6f4.block_scale, scale_vec::1X: one E8M0 scale per 32 values of K
// for every row of A and of B). Channels on the MMA's M side (128 weight rows), tokens on N (128).
// A 128-byte K-block of FP8 codes is four MMAs of K = 32, i.e. four MX blocks, whose scales are
// one 32-bit word per row: scales[r, 4kb .. 4kb+3], byte j for the j-th MMA.
// Scale factors live in TMEM, per pipeline stage: SFA in 4 columns, SFB in 4 columns. Row
// 32g + l of a 128-row operand sits in column g, at lane l of every lane quarter (each quarter of
// the tensor core reads its own copy), byte j for K-block j of the four; the MMA names the byte
// in the top two bits of the scale's TMEM address and in the instruction's scale-factor ids.
// Roles per CTA (one per SM, 14 warps):
//   warp 0      TMA producer: weight and token code blocks (128 rows x 128 bytes, 128-byte swizzle);
//   warp 1      TMEM allocator and MMA issuer (one elected thread);
//   warps 2-5   scale writers, one per TMEM lane quarter: each stage's scale words from global
//               memory into the stage's scale columns of their quarter (tcgen05.st);
//   warps 6-13  epilogue: fp32 sums -> bf16 y, two warps per lane quarter.
// Every wait is bounded (ptx.cuh).
struct MxGemmParams {
  CUtensorMap tmA;     // weight codes: E4M3 [N, K] bytes, or E2M1 [N, K/2] packed bytes loaded as
                       // 16U4_ALIGN16B; box 128 rows x 128 values, 128-byte swizzle
  CUtensorMap tmB;     // token codes [M, K] bytes, the same box
  const uint32_t* sfa; // weight scales [N, K/32] bytes, read as words [N, K/128]
  const uint32_t* sfb; // token scales [M, K/32] bytes, read as words [M, K/128]
  int num_kb;          // K / 128
  int n_cb;            // N / 128
  int M;
  int N;
  uint16_t* y;         // [M, N] bf16
  uint64_t timeout_ns;
};

constexpr int kMxNB = 128;                          // tokens per tile (MMA N)
constexpr int kMxStages = 7;
constexpr int kMxSfAhead = 4;                       // scale-word prefetch depth (stages)
constexpr int kMxStageBytes = 2 * kBM * kKBlockBytes;  // weight block + token block
constexpr int kMxAccCols = kMxNB;                   // one accumulator set
constexpr uint32_t kMxSfCol0 = 2 * kMxAccCols;      // scale columns: 8 per stage after both sets
constexpr int kMxTmemCols = 512;
constexpr int kMxThreads = 32 * 14;
constexpr size_t kMxSmemBytes = 1024 + size_t(kMxStages) * kMxStageBytes + 512;
static_assert(kMxSfCol0 + 8 * kMxStages <= kMxTmemCols, "accumulators and scale columns fit in TMEM");

// Element formats of the block-scaled MMA's operands (its format fields): the weights are E4M3
// or E2M1, the tokens always E4M3.
constexpr int kMxE4M3 = 0;
constexpr int kMxE2M1 = 5;
// TMA bytes of one 128-row weight K-block (128 values a row): E2M1 rows are 64 bytes in global
// memory (the transaction count of the 16U4_ALIGN16B load; it fills 128 bytes of shared memory).
template <int WF>
constexpr uint32_t kMxWeightTxBytes = WF == kMxE2M1 ? kBM * kKBlockBytes / 2 : kBM * kKBlockBytes;

// Instruction descriptor of the block-scaled MMA: A (weights) in format WF (bits 7-9), B (tokens)
// E4M3, both K-major, fp32 accumulation, M = 128, N = n, E8M0 scales (bit 23), scale-factor ids of
// A (bits 29-30) and B (bits 4-5) = j.
template <int WF>
__host__ __device__ constexpr uint32_t idesc_mxf8(int n, uint32_t j) {
  return (j << 4) | (uint32_t(WF) << 7) | (uint32_t(n >> 3) << 17) | (1u << 23) | (uint32_t(128 >> 4) << 24) |
         (j << 29);
}

__device__ __forceinline__ void tc_mma_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 4 consecutive 32-bit TMEM columns of the warp's 32 lanes from registers (no wait).
__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(a), "r"(b), "r"(c),
               "r"(d));
}

template <int WF>
__global__ void __launch_bounds__(kMxThreads, 1) mx_gemm_kernel(const __grid_constant__ MxGemmParams p) {
  constexpr int S = kMxStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * kMxStageBytes);
  uint64_t* empty = full + S;
  uint64_t* sfready = empty + S;
  uint64_t* tfull = sfready + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, p.timeout_ns};
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); mbar_init(sfready + s, 4); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull + a, 1); mbar_init(tempty + a, 8); }
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
    tma_prefetch_map(&p.tmA);
    tma_prefetch_map(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kMxTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // the token codes and scales come from the quantisation kernel launched just before
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int m_tiles = (p.M + kMxNB - 1) / kMxNB;
  const int total = m_tiles * p.n_cb;
  const int nkb = p.num_kb;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0, issued = 0, parity = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) { ok = false; break; }
        if (elect_one()) {
          uint8_t* st = smem + stage * kMxStageBytes;
          mbar_arrive_expect_tx(full + stage, kMxWeightTxBytes<WF> + uint32_t(kMxNB * kKBlockBytes));
          tma_load_2d(st, &p.tmA, full + stage, kb * kKBlockBytes, cb * kBM);
          tma_load_2d(st + kBM * kKBlockBytes, &p.tmB, full + stage, kb * kKBlockBytes, mt * kMxNB);  // rows past M: zeros
        }
        __syncwarp();
        issued |= 1u << stage;
        parity = (parity & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
    }
    if (lane == 0 && *abort_flag) {  // loads already issued land before the CTA exits
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, 100000000ull};
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s)) mbar_wait(full + s, (parity >> s) & 1u, dw);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(smem));
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool issued_any = false, ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      if (!mbar_wait_warp(tempty + acc, acc_phase ^ 1u, wc)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + uint32_t(acc * kMxAccCols);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_warp(full + stage, phase, wc)) { ok = false; break; }
        if (!mbar_wait_warp(sfready + stage, phase, wc)) { ok = false; break; }
        tc_fence_after();  // the scale columns written by the scale warps (tcgen05.st) precede
        if (elect_one()) {
          const uint64_t ad = adesc0 + uint64_t(stage * (kMxStageBytes >> 4));
          const uint64_t bd = ad + uint64_t((kBM * kKBlockBytes) >> 4);
          const uint32_t sf = tmem_base + kMxSfCol0 + uint32_t(8 * stage);
#pragma unroll
          for (uint32_t j = 0; j < 4; ++j)
            tc_mma_mxf8(d, ad + uint64_t(2 * j), bd + uint64_t(2 * j), idesc_mxf8<WF>(kMxNB, j), sf + (j << 30),
                        sf + 4u + (j << 30), (kb | int(j)) != 0 ? 1u : 0u);
          tc_commit(empty + stage);
        }
        __syncwarp();
        issued_any = true;
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) tc_commit(tfull + acc);
      __syncwarp();
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0 && *abort_flag && issued_any) {
      tc_commit(drain);
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, 100000000ull};
      mbar_wait(drain, 0, dw);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ scale writers (one per quarter)
    // The scale words of a stage are loaded from global memory kMxSfAhead stages before they are
    // written, so their latency overlaps the MMAs of the stages in between.
    constexpr int D = kMxSfAhead;
    const int q = warp & 3;
    const uint32_t lane_off = uint32_t(q * 32) << 16;
    const int wpr = nkb;  // scale words per row
    const int my_tiles = int(blockIdx.x) < total ? (total - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x) : 0;
    const int n = my_tiles * nkb;  // this CTA's (tile, K-block) items in order
    // rows 32g + lane of A (channels) and of B (tokens) of item i; tokens past M take scale word 0
    auto load = [&](int i, uint32_t (&a)[4], uint32_t (&b)[4]) {
      const int tile = int(blockIdx.x) + (i / nkb) * int(gridDim.x), kb = i % nkb;
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      const int c0 = cb * kBM, t0 = mt * kMxNB;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        a[g] = __ldg(p.sfa + size_t(c0 + 32 * g + lane) * wpr + kb);
        const int t = t0 + 32 * g + lane;
        b[g] = t < p.M ? __ldg(p.sfb + size_t(t) * wpr + kb) : 0u;
      }
    };
    uint32_t ra[D][4], rb[D][4];
#pragma unroll
    for (int d = 0; d < D; ++d)
      if (d < n) load(d, ra[d], rb[d]);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int i0 = 0; i0 < n && ok; i0 += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int i = i0 + d;
        if (i >= n) break;
        // the MMAs that read this stage's previous scales have completed
        if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) { ok = false; break; }
        const uint32_t col = tmem_base + lane_off + kMxSfCol0 + uint32_t(8 * stage);
        tmem_st4(col, ra[d][0], ra[d][1], ra[d][2], ra[d][3]);
        tmem_st4(col + 4u, rb[d][0], rb[d][1], rb[d][2], rb[d][3]);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sfready + stage);
        if (++stage == S) { stage = 0; phase ^= 1u; }
        if (i + D < n) load(i + D, ra[d], rb[d]);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 6-13)
    const int q = warp & 3;
    const int half = (warp - 6) >> 2;  // token columns [64 half, 64 half + 64)
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      const int t0 = mt * kMxNB;
      const int ch = cb * kBM + q * 32 + lane;  // this lane's output channel
      if (!mbar_wait_warp(tfull + acc, acc_phase, wc)) break;
      tc_fence_after();
      const uint32_t t_lane = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * kMxAccCols);
      uint16_t* out = p.y + ch;
#pragma unroll 1
      for (int j0 = half * 64; j0 < half * 64 + 64; j0 += 16) {
        uint32_t r[16];
        tmem_ld16(t_lane + uint32_t(j0), r);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (t0 + j0 + j < p.M)
            out[size_t(t0 + j0 + j) * p.N] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[j])));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty + acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kMxTmemCols);
  }
}

// ---------------------------------------------------------------- the same GEMM on CTA pairs
// Tiles of 256 channels x 192 tokens on the two CTAs of a cluster with M = 256 block-scaled MMAs
// (cta_group::2): rank r supplies its 128 weight rows and 96 of the token rows, and receives the
// sums of its 128 channels for all 192 tokens, so per SM and K-block 16 + 12 KB of codes feed
// 128 x 192 x 128 MACs (the one-CTA tile moves 32 KB for 128 x 128 x 128). Each rank keeps in its
// TMEM, per stage and laid out like the one-CTA kernel's, the scales of its own 128 weight rows
// (4 columns) and those of the tile's token rows (6 of 8 columns): each CTA's half of the tensor
// core scales every column of its accumulators. (Holding only the 96 token rows a rank supplies
// gives wrong sums for the other half of the columns.)
// The scales reach TMEM through shared memory: the scale warps write each stage's words there in
// the order one `tcgen05.cp.32x128b.warpx4` takes (32 rows of 16 bytes: row l holds the words of
// rows l, 32 + l, 64 + l, 96 + l, copied to columns 0-3 of every lane quarter), and the MMA thread
// issues the copies right before the stage's MMAs; copies and MMAs of one thread run in issue
// order, so nothing waits on TMEM stores. (Scale warps storing into TMEM themselves with
// tcgen05.st made every K-block wait for those stores: 45 us against 28 us without them.) The
// token scales are copied as 8 groups of 32 rows from the 4-aligned group at or below the tile's
// first (tiles start at group 6 mt), and the MMA's scale address skips the first 0 or 2 columns.
struct MxPairParams {
  CUtensorMap tmA;     // weight codes (E4M3 or packed E2M1, as in MxGemmParams), box 128 rows x 128
                       // values, 128-byte swizzle
  CUtensorMap tmB;     // token codes [M, K], box 96 rows x 128 bytes, 128-byte swizzle
  const uint32_t* sfa; // weight scales as words [N, K/128]
  const uint32_t* sfb; // token scales as words [M, K/128]
  int num_kb;          // K / 128
  int n_cb;            // N / 256
  int M;
  int N;
  uint16_t* y;         // [M, N] bf16
  uint64_t timeout_ns;
};

constexpr int kMxPairNB = 192;                 // tokens per tile (MMA N)
constexpr int kMxPairHalf = kMxPairNB / 2;     // token rows each rank loads
constexpr int kMxPairStages = 7;
constexpr int kMxPairABytes = kBM * kKBlockBytes;
constexpr int kMxPairBBytes = kMxPairHalf * kKBlockBytes;
constexpr int kMxPairStageBytes = kMxPairABytes + kMxPairBBytes;
constexpr uint32_t kMxPairSfCol0 = 2 * kMxPairNB;  // after both accumulator sets
constexpr int kMxPairSfCols = 12;                  // per stage: SFA 4 + SFB 8 (token groups)
constexpr int kMxPairSfBytes = 3 * 512;            // per stage in shared memory: SFA, SFB groups 0-3, 4-7
constexpr int kMxPairThreads = 32 * 14;
constexpr size_t kMxPairSmemBytes =
    1024 + size_t(kMxPairStages) * kMxPairStageBytes + 512 + size_t(kMxPairStages) * kMxPairSfBytes;
static_assert(kMxPairSfCol0 + kMxPairSfCols * kMxPairStages <= 512, "accumulators and scales fit in TMEM");
static_assert(kMxPairBBytes % 1024 == 0, "128-byte swizzled token rows sit on 1 KB boundaries");

template <int WF>
__host__ __device__ constexpr uint32_t idesc_mxf8_m256(int n, uint32_t j) {
  return (j << 4) | (uint32_t(WF) << 7) | (uint32_t(n >> 3) << 17) | (1u << 23) | (uint32_t(256 >> 4) << 24) |
         (j << 29);
}

// Shared-memory descriptor of a 32-row x 16-byte block for tcgen05.cp: no swizzle, rows 16 bytes
// apart within 8-row core matrices, core matrices 128 bytes apart (stride byte offset), version 1.
__device__ __forceinline__ uint64_t sf_block_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t(1) << 16;          // leading byte offset (one 16-byte column: unused)
  d |= uint64_t(128 >> 4) << 32;   // stride byte offset
  d |= uint64_t(1) << 46;          // descriptor version
  return d;                        // layout type 0: no swizzle
}

// Copies a 32-row x 128-bit block from shared memory into 4 TMEM columns of every lane quarter
// (row l to lane l of each quarter), in both CTAs of the pair (each from its own shared memory).
__device__ __forceinline__ void tc_cp_pair_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_mma_pair_mxf8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

template <int WF>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMxPairThreads, 1)
    mx_pair_kernel(const __grid_constant__ MxPairParams p) {
  constexpr int S = kMxPairStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * kMxPairStageBytes);  // used on rank 0
  uint64_t* empty = full + S;                                                  // each rank
  uint64_t* sfready = empty + S;                                               // used on rank 0
  uint64_t* tfull = sfready + S;                                               // each rank, [2]
  uint64_t* tempty = tfull + 2;                                                // used on rank 0, [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* sf_smem = smem + S * kMxPairStageBytes + 512;  // [S][3][32 rows][16 bytes]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = int(cluster_index());
  const int nclusters = int(cluster_count());
  const WaitCtx wc{abort_flag, p.timeout_ns};
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); mbar_init(sfready + s, 2); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull + a, 1); mbar_init(tempty + a, 16); }
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
    tma_prefetch_map(&p.tmA);
    tma_prefetch_map(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  pdl_wait();  // the token codes and scales come from the quantisation kernel launched just before
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int m_tiles = (p.M + kMxPairNB - 1) / kMxPairNB;
  const int total = m_tiles * p.n_cb;
  const int nkb = p.num_kb;
  const int my_tiles = cluster < total ? (total - cluster + nclusters - 1) / nclusters : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both ranks)
    const uint32_t full0 = map_to_rank(smem_addr(full), 0);
    int stage = 0;
    uint32_t phase = 0, issued = 0, parity = 0;
    bool ok = true;
    for (int tile = cluster; tile < total && ok; tile += nclusters) {
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) { ok = false; break; }
        if (elect_one()) {
          uint8_t* st = smem + stage * kMxPairStageBytes;
          const uint32_t bar = full0 + uint32_t(stage) * 8u;
          if (leader) mbar_arrive_expect_tx(full + stage, 2u * (kMxWeightTxBytes<WF> + uint32_t(kMxPairBBytes)));
          tma_load_2d_pair(st, &p.tmA, bar, kb * kKBlockBytes, cb * 256 + int(rank) * 128);
          tma_load_2d_pair(st + kMxPairABytes, &p.tmB, bar, kb * kKBlockBytes,
                           mt * kMxPairNB + int(rank) * kMxPairHalf);  // rows past M: zeros
        }
        __syncwarp();
        issued |= 1u << stage;
        parity = (parity & ~(1u << stage)) | (phase << stage);
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
    }
    if (ok) {
      // every stage released by the MMAs (their completions reach this CTA) before exit
      for (int i = 0; i < S; ++i) {
        if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) break;
        if (++stage == S) { stage = 0; phase ^= 1u; }
      }
    }
    if (lane == 0 && *abort_flag) {
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, 100000000ull};
      if (leader) {
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) mbar_wait(full + s, (parity >> s) & 1u, dw);
      } else {
        const uint64_t until = globaltimer_ns() + 1000000ull;
        while (globaltimer_ns() < until) __nanosleep(10000);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (leader) {
      const uint32_t empty_own = smem_addr(empty), empty_peer = map_to_rank(smem_addr(empty), 1);
      const uint32_t tfull_own = smem_addr(tfull), tfull_peer = map_to_rank(smem_addr(tfull), 1);
      const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(smem));
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool issued_any = false, ok = true;
      for (int t = 0; t < my_tiles && ok; ++t) {
        if (!mbar_wait_warp(tempty + acc, acc_phase ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + uint32_t(acc * kMxPairNB);
        const int mt = (cluster + t * nclusters) / p.n_cb;
        const uint32_t sfb_skip = uint32_t((6 * mt) & 3);  // the tile's first token group within the copied 8
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_warp(full + stage, phase, wc)) { ok = false; break; }
          if (!mbar_wait_warp(sfready + stage, phase, wc)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
            const uint64_t ad = adesc0 + uint64_t(stage * (kMxPairStageBytes >> 4));
            const uint64_t bd = ad + uint64_t(kMxPairABytes >> 4);
            const uint32_t sf = tmem_base + kMxPairSfCol0 + uint32_t(kMxPairSfCols * stage);
            const uint32_t sfs = smem_addr(sf_smem + stage * kMxPairSfBytes);
            tc_cp_pair_32x128b_x4(sf, sf_block_desc(sfs));                // weight rows: columns 0-3
            tc_cp_pair_32x128b_x4(sf + 4u, sf_block_desc(sfs + 512u));    // token groups 0-3
            tc_cp_pair_32x128b_x4(sf + 8u, sf_block_desc(sfs + 1024u));   // token groups 4-7
            const uint32_t sfb = sf + 4u + sfb_skip;
#pragma unroll
            for (uint32_t j = 0; j < 4; ++j)
              tc_mma_pair_mxf8(d, ad + uint64_t(2 * j), bd + uint64_t(2 * j), idesc_mxf8_m256<WF>(kMxPairNB, j),
                               sf + (j << 30), sfb + (j << 30), (kb | int(j)) != 0 ? 1u : 0u);
            tc_commit_pair(empty_own + uint32_t(stage) * 8u);
            tc_commit_pair(empty_peer + uint32_t(stage) * 8u);
          }
          __syncwarp();
          issued_any = true;
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) {
          tc_commit_pair(tfull_own + uint32_t(acc) * 8u);
          tc_commit_pair(tfull_peer + uint32_t(acc) * 8u);
        }
        __syncwarp();
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (ok && !*abort_flag) {
        for (int i = 0; i < 2; ++i) {
          if (!mbar_wait_warp(tempty + acc, acc_phase ^ 1u, wc)) break;
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
      }
      if (lane == 0 && *abort_flag && issued_any) {
        tc_commit_pair(smem_addr(drain));
        volatile int no_abort = 0;
        const WaitCtx dw{&no_abort, 100000000ull};
        mbar_wait(drain, 0, dw);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ scale writers (both ranks)
    // The four warps take the stages in turn (warp 2 + w the items w, w + 4, ...), so each has
    // four K-blocks of time for one stage's loads, stores, proxy fence and remote arrival. Lane l
    // writes row l of the three 32-row blocks: the words of weight rows l, 32 + l, 64 + l, 96 + l
    // and of token groups 0-3 and 4-7 (row l of each), one 16-byte store per block.
    const int w = warp - 2;
    const uint32_t sfready0 = map_to_rank(smem_addr(sfready), 0);
    const int wpr = nkb;
    const int n = my_tiles * nkb;
    auto load = [&](int i, uint32_t (&v)[12]) {
      const int tile = cluster + (i / nkb) * nclusters, kb = i % nkb;
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      const int c0 = cb * 256 + int(rank) * 128 + lane;
      const int t0 = 32 * ((6 * mt) & ~3) + lane;  // row l of the first copied token group
#pragma unroll
      for (int g = 0; g < 4; ++g) v[g] = __ldg(p.sfa + size_t(c0 + 32 * g) * wpr + kb);
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int t = t0 + 32 * g;
        v[4 + g] = t < p.M ? __ldg(p.sfb + size_t(t) * wpr + kb) : 0u;
      }
    };
    uint32_t v[12];
    if (w < n) load(w, v);
    for (int i = w; i < n; i += 4) {
      const int stage = i % S;
      const uint32_t phase = uint32_t(i / S) & 1u;
      // the stage's previous copies have completed (they precede the MMAs whose commit this is)
      if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) break;
      uint4* blk = reinterpret_cast<uint4*>(sf_smem + stage * kMxPairSfBytes) + lane;
      blk[0] = make_uint4(v[0], v[1], v[2], v[3]);
      blk[32] = make_uint4(v[4], v[5], v[6], v[7]);
      blk[64] = make_uint4(v[8], v[9], v[10], v[11]);
      fence_proxy_async_smem();  // generic-proxy writes become visible to tcgen05.cp
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(sfready0 + uint32_t(stage) * 8u);
      if (i + 4 < n) load(i + 4, v);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both ranks)
    const int q = warp & 3;
    const int half = (warp - 6) >> 2;  // token columns [96 half, 96 half + 96)
    const uint32_t tempty0 = map_to_rank(smem_addr(tempty), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = cluster; tile < total; tile += nclusters) {
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      const int t0 = mt * kMxPairNB;
      const int ch = cb * 256 + int(rank) * 128 + q * 32 + lane;
      if (!mbar_wait_warp(tfull + acc, acc_phase, wc)) break;
      tc_fence_after();
      const uint32_t t_lane = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * kMxPairNB);
      uint16_t* out = p.y + ch;
#pragma unroll 1
      for (int j0 = half * kMxPairHalf; j0 < half * kMxPairHalf + kMxPairHalf; j0 += 16) {
        uint32_t r[16];
        tmem_ld16(t_lane + uint32_t(j0), r);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (t0 + j0 + j < p.M)
            out[size_t(t0 + j0 + j) * p.N] = __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[j])));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + uint32_t(acc) * 8u);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace w8a8
