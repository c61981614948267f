// Dense W4A8 linear on the 5th-generation tensor cores (sm_100a):
//
//   y[t, n] = bf16( s_x[t] * acc_f ),  acc_f = fma((float)acc_g, s_w[n, g], acc_f) over g in order
//   acc_g[t, n] = sum over the g-th group of 128 K values of xq[t, k] * w[n, k]   (int32)
//
// The weights arrive as 4-bit two's-complement codes, two per byte (even k in the low nibble),
// with one fp32 scale per (output channel, group of 128 along K) ("4bit 权重" section of the
// Qwen3-1.7B-W4A8 page). One 128-byte K-block of int8 is exactly one scale group, so the int32
// partial of each group is read out of TMEM and scaled on its own.
// Roles per CTA (one CTA per SM, 14 warps), tile = 128 channels (MMA M) x NB tokens (MMA N):
//   warp 0      TMA producer: packed weight tile (128 rows x 64 bytes, no swizzle) into a
//               staging slot, token rows (128-byte swizzled, like the int8 GEMMs);
//   warp 1      TMEM allocator and MMA issuer: one tcgen05.mma kind::i8 group per K-block into
//               alternating TMEM buffers;
//   warps 2-5   converters: sign-extend the nibbles to int8 and write them in the 128-byte
//               swizzled K-major layout the MMA reads, then fence the async proxy;
//   warps 6-13  epilogue: per K-block, acc = fma((float)acc_g, s_w[n, g], acc) in fp32 registers;
//               at the tile's end store bf16(acc * s_x[t]).
// Four TMEM buffers let the MMA run up to three K-blocks ahead of the epilogue.
#pragma once
#include "gemm.cuh"

namespace w8a8 {

constexpr int kW4Threads = 64 + 128 + 32 * kEpiWarps;

struct W4A8Params {
  CUtensorMap tmW;   // packed weights [N, K/2] bytes, box 128 rows x 64 bytes, no swizzle
  CUtensorMap tmX;   // xq [Mp, K] int8, box 16 rows x 128 bytes, 128-byte swizzle
  CUtensorMap tmX2;  // xq, box NB rows (full token tiles)
  int num_kb;        // K / 128 (= number of scale groups)
  int n_cb;          // N / 128
  int M;             // tokens
  int N;
  const float* sw;   // [N, num_kb]
  const float* sx;   // [M]
  uint16_t* y;       // [M, N] bf16
  uint64_t timeout_ns;
};

template <int NB>
struct W4Cfg {
  static constexpr int kPackedBytes = kBM * 64;
  static constexpr int kABytes = kBM * kKBlockBytes;
  static constexpr int kBBytes = NB * kKBlockBytes;
  static constexpr int kStageBytes = kPackedBytes + kABytes + kBBytes;
  static constexpr int kStages = (192 * 1024) / kStageBytes > 8 ? 8 : (192 * 1024) / kStageBytes;
  static constexpr int kAccBufs = 4;
  static constexpr int kTmemCols = (kAccBufs * NB <= 128) ? 128 : (kAccBufs * NB <= 256 ? 256 : 512);
  static_assert(kAccBufs * NB <= 512, "accumulator buffers must fit in TMEM");
  static constexpr size_t kSmemBytes = 1024 + size_t(kStages) * kStageBytes + 512;
  static_assert(kStages >= 2, "pipeline too shallow");
};

// Four 4-bit two's-complement codes (one per byte, low nibbles) sign-extended to int8 lanes:
// bit 3 set means negative, and (bit 3) * 30 = 0xF0 fills the high nibble of that byte alone
// (8 * 30 = 240 < 256, so no product carries into the next byte).
__device__ __forceinline__ uint32_t sext_nibbles(uint32_t v) {
  return (v & 0x0F0F0F0Fu) | ((v & 0x08080808u) * 30u);
}

// 8 packed bytes (16 int4 codes) -> 16 sign-extended int8 codes in k order.
__device__ __forceinline__ uint4 unpack_int4x16(uint2 pk) {
  const uint32_t w[2] = {pk.x, pk.y};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t lo = sext_nibbles(w[i]);       // even k
    const uint32_t hi = sext_nibbles(w[i] >> 4);  // odd k
    o[2 * i] = __byte_perm(lo, hi, 0x5140);      // l0 h0 l1 h1
    o[2 * i + 1] = __byte_perm(lo, hi, 0x7362);  // l2 h2 l3 h3
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Exact int -> fp32 for |x| < 2^22 without the conversion pipe: 1.5 * 2^23 + x is an fp32
// with x in its low mantissa bits, and subtracting 1.5 * 2^23 is exact. A group partial is
// at most 127 * 7 * 128 < 2^22 in magnitude.
__device__ __forceinline__ float small_int_to_float(int32_t x) {
  return __fsub_rn(__int_as_float(x + 0x4B400000), 12582912.0f);
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

template <int NB>
__global__ void __launch_bounds__(kW4Threads, 1) w4a8_gemm_kernel(const __grid_constant__ W4A8Params p) {
  using Cfg = W4Cfg<NB>;
  constexpr int STAGES = Cfg::kStages;
  constexpr uint32_t IDESC0 = idesc_s8s8s32(0);
  constexpr int HALFC = NB / 2;  // token columns per epilogue warp

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::kStageBytes);
  uint64_t* conv = full + STAGES;
  uint64_t* empty = conv + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + Cfg::kAccBufs;
  uint64_t* drain = tempty + Cfg::kAccBufs;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, globaltimer_ns() + p.timeout_ns};
  auto packed_of = [&](int s) { return smem + s * Cfg::kStageBytes; };
  auto a_of = [&](int s) { return smem + s * Cfg::kStageBytes + Cfg::kPackedBytes; };
  auto b_of = [&](int s) { return smem + s * Cfg::kStageBytes + Cfg::kPackedBytes + Cfg::kABytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full + s, 1);
      mbar_init(conv + s, 128);
      mbar_init(empty + s, 1);
    }
    for (int a = 0; a < Cfg::kAccBufs; ++a) { mbar_init(tfull + a, 1); mbar_init(tempty + a, kEpiWarps * 32); }
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
    tma_prefetch_map(&p.tmW);
    tma_prefetch_map(&p.tmX);
    tma_prefetch_map(&p.tmX2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();  // xq and sx come from the quantisation kernel launched just before
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int m_tiles = (p.M + NB - 1) / NB;
  const int total_tiles = m_tiles * p.n_cb;
  const int nkb = p.num_kb;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Converged warp, one elected lane issues.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      const int tok0 = mt * NB, rows = min(NB, p.M - tok0), nb = (rows + 15) & ~15;
      const uint32_t bytes = uint32_t(Cfg::kPackedBytes + nb * kKBlockBytes);
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) { ok = false; break; }
        if (elect_one()) {
          mbar_arrive_expect_tx(full + stage, bytes);
          tma_load_2d(packed_of(stage), &p.tmW, full + stage, kb * 64, cb * kBM);
          if (nb == NB) {
            tma_load_2d(b_of(stage), &p.tmX2, full + stage, kb * 128, tok0);
          } else {
            for (int b = 0; b < nb; b += kBBoxRows)
              tma_load_2d(b_of(stage) + b * kKBlockBytes, &p.tmX, full + stage, kb * 128, tok0 + b);
          }
        }
        __syncwarp();
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (lane == 0 && *abort_flag) {
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, globaltimer_ns() + 100000000ull};
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) mbar_wait(full + s, (issued_parity >> s) & 1u, dw);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Converged warp, warp-uniform descriptors, one elected lane issues.
    const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(a_of(0)));
    const uint64_t bdesc0 = sw128_kmajor_desc(smem_addr(b_of(0)));
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool issued_any = false;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const int mt = tile / p.n_cb;
      const int rows = min(NB, p.M - mt * NB), nb = (rows + 15) & ~15;
      const uint32_t idesc = IDESC0 | (uint32_t(nb >> 3) << 17);
      for (int kb = 0; kb < nkb; ++kb) {
        // one scale group per K-block: a fresh accumulator in the free TMEM buffer
        if (!mbar_wait_warp(tempty + acc, acc_phase ^ 1u, wc)) { ok = false; break; }
        if (!mbar_wait_warp(conv + stage, phase, wc)) { ok = false; break; }
        tc_fence_after();  // the converters' shared-memory writes (generic proxy, fenced) precede
        const uint32_t d = tmem_base + uint32_t(acc * NB);
        if (elect_one()) {
          const uint64_t ad = adesc0 + uint64_t(stage * (Cfg::kStageBytes >> 4));
          const uint64_t bd = bdesc0 + uint64_t(stage * (Cfg::kStageBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < kKBlockBytes / 32; ++kk)
            tc_mma<kKindI8>(d, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), idesc, kk != 0 ? 1u : 0u);
          tc_commit(empty + stage);
          tc_commit(tfull + acc);
        }
        __syncwarp();
        issued_any = true;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        if (++acc == Cfg::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
    }
    if (lane == 0 && *abort_flag && issued_any) {
      tc_commit(drain);
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, globaltimer_ns() + 100000000ull};
      mbar_wait(drain, 0, dw);
    }
    __syncwarp();
  } else if (warp < 6) {
    // ------------------------------------------------------------ converters (warps 2..5)
    const int ct = threadIdx.x - 64;  // 0..127
    int stage = 0;
    uint32_t phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait(full + stage, phase, wc)) { ok = false; break; }
        const uint8_t* src = packed_of(stage);
        uint8_t* dst = a_of(stage);
        // 128 rows x 64 packed bytes: item = (row, 16-byte packed chunk) -> two 16-byte int8 chunks
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int item = ct + 128 * q;
          const int r = item >> 2, pch = item & 3;
          const uint4 pk = *reinterpret_cast<const uint4*>(src + r * 64 + pch * 16);
          const uint4 o0 = unpack_int4x16(make_uint2(pk.x, pk.y));
          const uint4 o1 = unpack_int4x16(make_uint2(pk.z, pk.w));
          const int c0 = 2 * pch, c1 = 2 * pch + 1;  // logical 16-byte chunks of the int8 row
          *reinterpret_cast<uint4*>(dst + r * 128 + ((c0 ^ (r & 7)) << 4)) = o0;
          *reinterpret_cast<uint4*>(dst + r * 128 + ((c1 ^ (r & 7)) << 4)) = o1;
        }
        fence_proxy_async_smem();  // generic-proxy writes become visible to the tensor core
        mbar_arrive(conv + stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 6..13)
    const int q = warp & 3;
    const int half = (warp - 6) >> 2;
    const int ch = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      const int tok0 = mt * NB, rows = min(NB, p.M - tok0);
      const int n = cb * kBM + ch;
      const int j0 = half * HALFC;  // this warp's token columns [j0, j0 + HALFC)
      const float* __restrict__ swr = p.sw + size_t(n) * nkb;
      float accf[HALFC];
#pragma unroll
      for (int j = 0; j < HALFC; ++j) accf[j] = 0.0f;
      bool ok = true;
      float s_next = __ldg(swr);
      for (int kb = 0; kb < nkb; ++kb) {
        const float s = s_next;
        if (kb + 1 < nkb) s_next = __ldg(swr + kb + 1);  // next group's scale, loaded early
        if (!mbar_wait(tfull + acc, acc_phase, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t t_lane = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * NB);
        if (j0 < rows) {
#pragma unroll
          for (int c16 = 0; c16 < HALFC; c16 += 16) {
            uint32_t r[16];
            tmem_ld16(t_lane + j0 + c16, r);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              accf[c16 + i] = __fmaf_rn(small_int_to_float(int32_t(r[i])), s, accf[c16 + i]);
          }
        }
        tc_fence_before();
        mbar_arrive(tempty + acc);
        if (++acc == Cfg::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) break;
      uint16_t* out = p.y + n;
#pragma unroll
      for (int j = 0; j < HALFC; ++j) {
        const int t = j0 + j;
        if (t < rows)
          out[size_t(tok0 + t) * p.N] =
              __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(accf[j], __ldg(p.sx + tok0 + t))));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace w8a8
