// Dense W4A8 linear on the 5th-generation tensor cores (sm_100a):
//
//   y[t, n] = bf16( s_x[t] * acc_f ),  acc_f = fma((float)acc_g, s_w[n, g], acc_f) over g in order
//   acc_g[t, n] = sum over the g-th group of 128 K values of xq[t, k] * w[n, k]   (int32)
//
// The weights arrive as 4-bit two's-complement codes, two per byte (even k in the low nibble),
// with one fp32 scale per (output channel, group of 128 along K) ("4bit 权重" section of the
// Qwen3-1.7B-W4A8 page). One 128-byte K-block of int8 is exactly one scale group, so the int32
// partial of each group is read out of TMEM and scaled on its own.
// Two exact rewrites keep the per-element work small:
//   - the weights go to shared memory as the int8 byte 16 * code (the nibble masked in place,
//     or shifted up by 4), so the tensor core sums 16 * acc_g;
//   - every accumulator starts from the bit pattern of the fp32 1.5 * 2^19 instead of 0. Float
//     spacing in [2^19, 2^20) is 2^-4, so adding the integer 16 * acc_g to those bits adds acc_g
//     to the float's value; |16 * acc_g| <= 16 * 127 * 8 * 128 < 2^21 keeps it in that binade.
//     The register then holds the fp32 1.5 * 2^19 + acc_g exactly, and subtracting 1.5 * 2^19
//     (exact) returns (float)acc_g: one packed subtract and one packed FMA per two values.
// Roles per CTA (one CTA per SM, 2 + CV + EW warps), tile = 128 channels (MMA M) x NB tokens (MMA N),
// K-blocks of 128 taken in one sequence across the CTA's tiles:
//   warp 0      TMA producer: packed weight blocks (128 rows x 64 bytes, no swizzle) into their
//               own ring, token rows (128-byte swizzled, like the int8 GEMMs) into another;
//   warp 1      TMEM allocator and MMA issuer: one tcgen05.mma kind::i8 group per K-block into
//               one of four TMEM buffers;
//   CV warps    converters: each packed block into a third ring (16 * code int8 bytes in the
//               128-byte swizzled K-major layout the MMA reads, async proxy fenced), up to
//               kASlots K-blocks ahead of the MMA;
//   EW warps    epilogue: each K-block out of TMEM, acc = fma((float)acc_g, s_w[n, g], acc) in
//               fp32 registers, and the TMEM buffer reset to the start pattern. At a tile's end
//               bf16(acc * s_x[t]) goes into a shared-memory copy of the output tile, which one
//               thread hands to a TMA bulk store while the warps go on with the next tile.
// The packed ring is released as soon as a block is in registers, so weight loads run far ahead;
// the MMA waits only for the converted block, its token rows and a free TMEM buffer.
#pragma once
#include "gemm.cuh"

namespace w8a8 {

struct W4A8Params {
  CUtensorMap tmW;   // packed weights [N, K/2] bytes, box 128 rows x 64 bytes, no swizzle
  CUtensorMap tmX;   // xq [Mp, K] int8, box 16 rows x 128 bytes, 128-byte swizzle
  CUtensorMap tmX2;  // xq, box NB rows (full token tiles)
  CUtensorMap tmY;   // y [M, N] bf16 seen as bytes, box NB rows x 256 bytes (128 channels), no swizzle
  int num_kb;        // K / 128 (= number of scale groups)
  int n_cb;          // N / 128
  int M;             // tokens
  int N;
  const float* sw;   // [N, num_kb]
  int sw_vec;        // rows of sw start on 16-byte boundaries (num_kb % 4 == 0, sw aligned)
  const float* sx;   // [M]
  uint64_t timeout_ns;
};

// NB tokens per tile, CV converter warps, EW epilogue warps.
template <int NB, int CV, int EW>
struct W4Cfg {
  static constexpr int kThreads = 64 + 32 * (CV + EW);
  static constexpr int kConverters = 32 * CV;
  static constexpr int kItems = 512 / kConverters;  // 16-byte packed chunks per thread and K-block
  static_assert(kItems * kConverters == 512, "a packed K-block is 512 chunks");
  static constexpr int kEpilogue = 32 * EW;
  static constexpr int kCols = NB * 4 / EW;  // token columns per epilogue warp
  static_assert(EW % 4 == 0 && kCols % 32 == 0, "epilogue warps cover whole lane quarters");
  static constexpr int kEpiWarp0 = 2 + CV;  // first epilogue warp
  static constexpr int kXBytes = NB * kKBlockBytes;   // token rows of one K-block
  static constexpr int kABytes = kBM * kKBlockBytes;  // converted weights of one K-block
  static constexpr int kWBytes = kBM * 64;            // packed weights of one K-block
  static constexpr int kXStages = 6;
  static constexpr int kASlots = 3;
  static constexpr int kWStages = 5;
  static constexpr int kAccBufs = 4;
  static constexpr int kTmemCols = 512;
  static_assert(kAccBufs * NB <= kTmemCols, "accumulator buffers must fit in TMEM");
  static constexpr int kXOff = 0;
  static constexpr int kAOff = kXOff + kXStages * kXBytes;
  static constexpr int kWOff = kAOff + kASlots * kABytes;
  static constexpr int kBarOff = kWOff + kWStages * kWBytes;
  static constexpr int kOutOff = kBarOff + 512;
  static constexpr int kOutBytes = NB * kBM * 2;  // the bf16 output tile, [token][channel]
  static constexpr int kSxOff = kOutOff + kOutBytes;
  static constexpr int kSxBytes = EW * kCols * 4;       // per warp: its tokens' s_x
  static constexpr size_t kSmemBytes = 1024 + size_t(kSxOff) + kSxBytes;
  static_assert(kXBytes % 1024 == 0 && kABytes % 1024 == 0, "128-byte swizzled tiles sit on 1 KB boundaries");
  static_assert(2 * (kXStages + kWStages + kASlots + kAccBufs + 1) * 8 + 8 + 8 + 8 <= 512, "barrier block");
};

// 8 packed bytes (16 int4 codes) -> 16 int8 bytes in k order holding 16 * code: the high nibble
// masked in place is 16 * (odd-k code) as a two's-complement byte, the low nibble shifted up by
// four is 16 * (even-k code).
__device__ __forceinline__ uint4 unpack_int4x16_x16(uint2 pk) {
  const uint32_t w[2] = {pk.x, pk.y};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint32_t lo = (w[i] << 4) & 0xF0F0F0F0u;  // even k
    const uint32_t hi = w[i] & 0xF0F0F0F0u;         // odd k
    o[2 * i] = __byte_perm(lo, hi, 0x5140);         // l0 h0 l1 h1
    o[2 * i + 1] = __byte_perm(lo, hi, 0x7362);     // l2 h2 l3 h3
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Start pattern of every accumulator: the fp32 1.5 * 2^19 (see the top of this file).
constexpr uint32_t kW4AccStartBits = 0x49400000u;
constexpr float kW4AccStart = 786432.0f;

// The same 32-bit value into 16 consecutive TMEM columns of the warp's 32 lanes (no wait). Two
// 8-column stores: a store's source registers are consecutive, and 8 copies of the value are
// cheap to keep next to the loaded columns.
__device__ __forceinline__ void tmem_fill16(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr), "r"(v));
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr + 8u),
               "r"(v));
}
__device__ __forceinline__ void tmem_fill8(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr), "r"(v));
}
// 8 consecutive 32-bit TMEM columns of the warp's 32 lanes (wait included).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// a_i = fma(x_i - c, s, a_i) for i = 0, 1 with packed fp32 operations; each lane is rounded
// exactly like the scalar subtract and FMA.
__device__ __forceinline__ void sub_fma_x2(float& a0, float& a1, uint32_t x0, uint32_t x1, uint64_t neg_c2,
                                           uint64_t s2) {
  asm("{\n\t.reg .b64 x, a;\n\t"
      "mov.b64 x, {%2, %3};\n\t"
      "mov.b64 a, {%0, %1};\n\t"
      "add.rn.f32x2 x, x, %4;\n\t"
      "fma.rn.f32x2 a, x, %5, a;\n\t"
      "mov.b64 {%0, %1}, a;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "r"(x0), "r"(x1), "l"(neg_c2), "l"(s2));
}
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  return uint64_t(__float_as_uint(lo)) | (uint64_t(__float_as_uint(hi)) << 32);
}


template <int NB, int CV, int EW>
__global__ void __launch_bounds__(W4Cfg<NB, CV, EW>::kThreads, 1)
    w4a8_gemm_kernel(const __grid_constant__ W4A8Params p) {
  using Cfg = W4Cfg<NB, CV, EW>;
  constexpr int E0 = Cfg::kEpiWarp0;
  constexpr int XS = Cfg::kXStages, AS = Cfg::kASlots, WS = Cfg::kWStages;
  constexpr uint32_t IDESC0 = idesc_s8s8s32(0);
  constexpr int CW = Cfg::kCols;  // token columns per epilogue warp

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* xfull = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
  uint64_t* xempty = xfull + XS;
  uint64_t* wfull = xempty + XS;
  uint64_t* wempty = wfull + WS;
  uint64_t* aready = wempty + WS;
  uint64_t* aempty = aready + AS;
  uint64_t* tfull = aempty + AS;
  uint64_t* tempty = tfull + Cfg::kAccBufs;
  uint64_t* ofree = tempty + Cfg::kAccBufs;  // the output tile may be rewritten
  uint64_t* ostaged = ofree + 1;              // the output tile is written
  uint64_t* drain = ostaged + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* out_tile = smem + Cfg::kOutOff;
  float* sx_smem = reinterpret_cast<float*>(smem + Cfg::kSxOff);
  auto x_of = [&](int s) { return smem + Cfg::kXOff + s * Cfg::kXBytes; };
  auto a_of = [&](int s) { return smem + Cfg::kAOff + s * Cfg::kABytes; };
  auto w_of = [&](int s) { return smem + Cfg::kWOff + s * Cfg::kWBytes; };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < XS; ++s) { mbar_init(xfull + s, 1); mbar_init(xempty + s, 1); }
    for (int s = 0; s < WS; ++s) { mbar_init(wfull + s, 1); mbar_init(wempty + s, Cfg::kConverters); }
    for (int s = 0; s < AS; ++s) { mbar_init(aready + s, Cfg::kConverters); mbar_init(aempty + s, 1); }
    for (int a = 0; a < Cfg::kAccBufs; ++a) { mbar_init(tfull + a, 1); mbar_init(tempty + a, Cfg::kEpilogue); }
    mbar_init(ofree, 1);
    mbar_init(ostaged, Cfg::kEpilogue);
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
    tma_prefetch_map(&p.tmW);
    tma_prefetch_map(&p.tmX);
    tma_prefetch_map(&p.tmX2);
    tma_prefetch_map(&p.tmY);
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
  if (warp >= E0) {  // every accumulator buffer starts from the start pattern
    const uint32_t t_lane = tmem_base + (uint32_t((warp & 3) * 32) << 16) + uint32_t(((warp - E0) >> 2) * CW);
#pragma unroll
    for (int c = 0; c < Cfg::kAccBufs * NB; c += NB)
#pragma unroll
      for (int h = 0; h < CW; h += 16) tmem_fill16(t_lane + uint32_t(c + h), kW4AccStartBits);
    tmem_wait_st();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int m_tiles = (p.M + NB - 1) / NB;
  const int total_tiles = m_tiles * p.n_cb;
  const int nkb = p.num_kb;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // Converged warp, one elected lane issues. Packed weights and token rows go to separate rings.
    int xs = 0, ws = 0;
    uint32_t xph = 0, wph = 0;
    uint32_t x_issued = 0, x_parity = 0, w_issued = 0, w_parity = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      const int tok0 = mt * NB, rows = min(NB, p.M - tok0), nb = (rows + 15) & ~15;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait_warp(wempty + ws, wph ^ 1u, wc)) { ok = false; break; }
        if (elect_one()) {
          mbar_arrive_expect_tx(wfull + ws, uint32_t(Cfg::kWBytes));
          tma_load_2d(w_of(ws), &p.tmW, wfull + ws, kb * 64, cb * kBM);
        }
        __syncwarp();
        w_issued |= 1u << ws;
        w_parity = (w_parity & ~(1u << ws)) | (wph << ws);
        if (++ws == WS) { ws = 0; wph ^= 1u; }
        if (!mbar_wait_warp(xempty + xs, xph ^ 1u, wc)) { ok = false; break; }
        if (elect_one()) {
          mbar_arrive_expect_tx(xfull + xs, uint32_t(nb * kKBlockBytes));
          if (nb == NB) {
            tma_load_2d(x_of(xs), &p.tmX2, xfull + xs, kb * 128, tok0);
          } else {
            for (int b = 0; b < nb; b += kBBoxRows)
              tma_load_2d(x_of(xs) + b * kKBlockBytes, &p.tmX, xfull + xs, kb * 128, tok0 + b);
          }
        }
        __syncwarp();
        x_issued |= 1u << xs;
        x_parity = (x_parity & ~(1u << xs)) | (xph << xs);
        if (++xs == XS) { xs = 0; xph ^= 1u; }
      }
    }
    if (lane == 0 && *abort_flag) {  // loads still in flight land before the CTA exits
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, 100000000ull};
      for (int s = 0; s < XS; ++s)
        if (x_issued & (1u << s)) mbar_wait(xfull + s, (x_parity >> s) & 1u, dw);
      for (int s = 0; s < WS; ++s)
        if (w_issued & (1u << s)) mbar_wait(wfull + s, (w_parity >> s) & 1u, dw);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Converged warp, warp-uniform descriptors, one elected lane issues.
    const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(a_of(0)));
    const uint64_t bdesc0 = sw128_kmajor_desc(smem_addr(x_of(0)));
    int xs = 0, as = 0, acc = 0;
    uint32_t xph = 0, aph = 0, acc_phase = 0;
    bool issued_any = false;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const int mt = tile / p.n_cb;
      const int rows = min(NB, p.M - mt * NB), nb = (rows + 15) & ~15;
      const uint32_t idesc = IDESC0 | (uint32_t(nb >> 3) << 17);
      for (int kb = 0; kb < nkb; ++kb) {
        // one scale group per K-block: the free TMEM buffer holds the start pattern
        if (!mbar_wait_warp(tempty + acc, acc_phase ^ 1u, wc)) { ok = false; break; }
        if (!mbar_wait_warp(aready + as, aph, wc)) { ok = false; break; }
        if (!mbar_wait_warp(xfull + xs, xph, wc)) { ok = false; break; }
        tc_fence_after();  // the converters' shared-memory writes (generic proxy, fenced) precede
        const uint32_t d = tmem_base + uint32_t(acc * NB);
        if (elect_one()) {
          const uint64_t ad = adesc0 + uint64_t(as * (Cfg::kABytes >> 4));
          const uint64_t bd = bdesc0 + uint64_t(xs * (Cfg::kXBytes >> 4));
#pragma unroll
          for (int kk = 0; kk < kKBlockBytes / 32; ++kk)
            tc_mma<kKindI8>(d, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), idesc, 1u);
          tc_commit(xempty + xs);
          tc_commit(aempty + as);
          tc_commit(tfull + acc);
        }
        __syncwarp();
        issued_any = true;
        if (++xs == XS) { xs = 0; xph ^= 1u; }
        if (++as == AS) { as = 0; aph ^= 1u; }
        if (++acc == Cfg::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
    }
    if (lane == 0 && *abort_flag && issued_any) {
      tc_commit(drain);
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, 100000000ull};
      mbar_wait(drain, 0, dw);
    }
    __syncwarp();
  } else if (warp < E0) {
    // ------------------------------------------------------------ converters (warps 2 .. E0 - 1)
    // Packed K-block -> the next converted slot. Each thread takes kItems of the block's 512
    // (row, 16-byte packed chunk) items; the packed stage is released once they are in registers.
    const int ct = threadIdx.x - 64;  // 0 .. kConverters - 1
    const int my_kbs = ((total_tiles - int(blockIdx.x) + int(gridDim.x) - 1) / int(gridDim.x)) * nkb;
    int ws = 0, as = 0;
    uint32_t wph = 0, aph = 0;
    for (int i = 0; i < my_kbs; ++i) {
      if (!mbar_wait(wfull + ws, wph, wc)) break;
      const uint8_t* src = w_of(ws);
      uint4 pks[Cfg::kItems];
#pragma unroll
      for (int j = 0; j < Cfg::kItems; ++j)
        pks[j] = *reinterpret_cast<const uint4*>(src + (ct + Cfg::kConverters * j) * 16);
      mbar_arrive(wempty + ws);
      if (++ws == WS) { ws = 0; wph ^= 1u; }
      if (!mbar_wait(aempty + as, aph ^ 1u, wc)) break;
      uint8_t* dst = a_of(as);
#pragma unroll
      for (int j = 0; j < Cfg::kItems; ++j) {
        const int item = ct + Cfg::kConverters * j;
        const int r = item >> 2, pch = item & 3;
        const uint4 o0 = unpack_int4x16_x16(make_uint2(pks[j].x, pks[j].y));
        const uint4 o1 = unpack_int4x16_x16(make_uint2(pks[j].z, pks[j].w));
        const int c0 = 2 * pch, c1 = 2 * pch + 1;  // logical 16-byte chunks of the int8 row
        *reinterpret_cast<uint4*>(dst + r * 128 + ((c0 ^ (r & 7)) << 4)) = o0;
        *reinterpret_cast<uint4*>(dst + r * 128 + ((c1 ^ (r & 7)) << 4)) = o1;
      }
      fence_proxy_async_smem();  // generic-proxy writes become visible to the tensor core
      mbar_arrive(aready + as);
      if (++as == AS) { as = 0; aph ^= 1u; }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps E0 ..)
    const int q = warp & 3;
    const int j0 = ((warp - E0) >> 2) * CW;  // this warp's token columns [j0, j0 + CW)
    const bool leader = threadIdx.x == E0 * 32;  // hands the output tile to the TMA store
    float* sxw = sx_smem + (warp - E0) * CW;
    const uint64_t neg_c2 = pack_f32x2(-kW4AccStart, -kW4AccStart);
    // s_w of this lane's channel, four K-blocks per load, one group of four ahead
    auto load_s4 = [&](const float* row, int k0) -> float4 {
      if (p.sw_vec) return __ldg(reinterpret_cast<const float4*>(row + k0));
      float4 v;
      v.x = k0 < nkb ? __ldg(row + k0) : 0.0f;
      v.y = k0 + 1 < nkb ? __ldg(row + k0 + 1) : 0.0f;
      v.z = k0 + 2 < nkb ? __ldg(row + k0 + 2) : 0.0f;
      v.w = k0 + 3 < nkb ? __ldg(row + k0 + 3) : 0.0f;
      return v;
    };
    bool ok = true;
    int acc = 0;
    uint32_t acc_phase = 0;
    int stored = 0;  // output tiles handed to the TMA store so far
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const int mt = tile / p.n_cb, cb = tile - mt * p.n_cb;
      const int tok0 = mt * NB, rows = min(NB, p.M - tok0);
      const int ch = q * 32 + lane;  // channel within the tile
      const float* __restrict__ swr = p.sw + size_t(cb * kBM + ch) * nkb;
      float accf[CW];
#pragma unroll
      for (int j = 0; j < CW; ++j) accf[j] = 0.0f;
      float4 s_cur = load_s4(swr, 0);
      float4 s_nxt = nkb > 4 ? load_s4(swr, 4) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);  // no read past the row
      // the s_x of the warp's tokens, needed only at the tile's end: loaded now
      float sxr[CW / 32];
#pragma unroll
      for (int i = 0; i < CW / 32; ++i)
        sxr[i] = (j0 + 32 * i + lane < rows) ? __ldg(p.sx + tok0 + j0 + 32 * i + lane) : 0.0f;
      for (int kb = 0; kb < nkb; ++kb) {
        const int k4 = kb & 3;
        const float s = k4 == 0 ? s_cur.x : (k4 == 1 ? s_cur.y : (k4 == 2 ? s_cur.z : s_cur.w));
        if (k4 == 3) {
          s_cur = s_nxt;
          if (kb + 5 < nkb) s_nxt = load_s4(swr, kb + 5);
        }
        // warp-uniform outcome: the TMEM loads and stores below are warp-collective
        if (!mbar_wait_warp(tfull + acc, acc_phase, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t t_lane = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * NB + j0);
        if (j0 < rows) {
          const uint64_t s2 = pack_f32x2(s, s);
#pragma unroll
          for (int h = 0; h < CW; h += 8) {
            uint32_t r[8];
            tmem_ld8(t_lane + uint32_t(h), r);
            // the columns just read start the buffer's next K-block from the pattern; the store
            // runs while the values are scaled
            tmem_fill8(t_lane + uint32_t(h), kW4AccStartBits);
#pragma unroll
            for (int j = 0; j < 8; j += 2)
              sub_fma_x2(accf[h + j], accf[h + j + 1], r[j], r[j + 1], neg_c2, s2);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(tempty + acc);
        if (++acc == Cfg::kAccBufs) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) break;
      // the previous tile's bulk store has read the output tile: it may be rewritten
      if (stored > 0) {
        if (leader) {
          bulk_wait_read_all();
          mbar_arrive(ofree);
        }
        if (!mbar_wait(ofree, uint32_t(stored - 1) & 1u, wc)) { ok = false; break; }
      }
      if (j0 < rows) {
#pragma unroll
        for (int i = 0; i < CW / 32; ++i) sxw[32 * i + lane] = sxr[i];
        __syncwarp();
        uint16_t* orow = reinterpret_cast<uint16_t*>(out_tile) + j0 * kBM + ch;
#pragma unroll
        for (int j = 0; j < CW; j += 4) {
          const float4 sv = *reinterpret_cast<const float4*>(sxw + j);
          orow[(j + 0) * kBM] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(accf[j + 0], sv.x)));
          orow[(j + 1) * kBM] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(accf[j + 1], sv.y)));
          orow[(j + 2) * kBM] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(accf[j + 2], sv.z)));
          orow[(j + 3) * kBM] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(accf[j + 3], sv.w)));
        }
        __syncwarp();  // sxw is rewritten by the next tile
      }
      fence_proxy_async_smem();  // the tile's generic-proxy writes become visible to the TMA store
      mbar_arrive(ostaged);
      if (leader) {
        if (!mbar_wait(ostaged, uint32_t(stored) & 1u, wc)) { ok = false; break; }
        tma_store_2d(&p.tmY, out_tile, cb * kBM * 2, tok0);  // rows past M are not written
        bulk_commit_group();
      }
      ++stored;
    }
    if (leader) bulk_wait_all();  // the CTA's shared memory outlives every bulk store
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace w8a8
