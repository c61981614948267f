// Persistent, warp-specialised grouped GEMM on the 5th-generation tensor cores (sm_100a).
//
//   D[r, n] = sum_k A[r, k] * B[n, k]      (A and B K-major; D accumulated in TMEM)
//
// A holds activation rows, grouped: rows offsets[g] .. offsets[g+1]-1 belong to group g
// (an expert). B holds one weight block per group. Each CTA owns one SM and walks a static
// list of 128 x BN output tiles; per CTA:
//   warp 0      TMA producer: 128-byte-swizzled K-blocks of A (128 rows) and B (BN rows)
//               into a STAGES-deep shared-memory ring (mbarrier full/empty pairs);
//   warp 1      TMEM allocator and MMA issuer: one thread issues tcgen05.mma
//               (kind::i8 -> s32, or kind::f16 bf16 -> f32) into one of two TMEM
//               accumulators, so the epilogue of tile i overlaps the MMAs of tile i+1;
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes (one output row per thread),
//               fused dequantisation / activation / routing, stores to global memory.
// Every mbarrier wait is bounded; a timeout aborts the CTA cleanly (see ptx.cuh).
#pragma once
#include "numerics.cuh"

namespace w8a8 {

enum EpiKind : int {
  kEpiRawS32 = 0,   // int32 accumulators stored as they are (exact integer GEMM)
  kEpiRouter = 1,   // fp32 logits -> (+bias) softmax, top-k, weights, per-tile expert histogram
  kEpiGateUp = 2,   // int32 gate|up -> dequant, SiLU(gate)*up -> bf16 h
  kEpiDown = 3,     // int32 -> dequant -> bf16 o written to the assignment's slot row
  kEpiDense = 4,    // int32 -> dequant -> bf16 y (dense W8A8 linear)
};

constexpr int kBM = 128;            // output rows per tile (tcgen05 M)
constexpr int kKBlockBytes = 128;   // K bytes per pipeline stage (one swizzle atom row)
constexpr int kGemmThreads = 192;   // 6 warps
constexpr int kMaxGroups = 1024;
constexpr int kMaxTopK = 16;

struct GemmParams {
  CUtensorMap tmA;  // A: [rowsA, K] K-major, box 128 rows x 128 bytes
  CUtensorMap tmB;  // B: [G * b_rows_per_group, K] K-major, box BN/2 rows x 128 bytes
  int num_kb;                  // K-blocks of 128 bytes
  int n_tiles;                 // tiles along N per group
  int num_groups;              // G
  const int* group_offsets;    // [G+1] row offsets into A (device); nullptr: one group of M rows
  int M;                       // rows of A when group_offsets is null
  int b_rows_per_group;        // rows of B per group
  int b_n_step;                // B row advance per N tile
  int b_half_offset;           // B row offset of the second half-box of a tile
  uint64_t timeout_ns;         // bound on every mbarrier wait
  // epilogue operands
  void* out;                   // see EpiKind
  int ldo;                     // output row stride, elements
  int out_col_step;            // output column advance per N tile
  int n_valid;                 // valid output columns (router: E)
  const float* row_scale;      // per A-row scale (x scale, or the requantisation scale of h)
  const float* col_scale;      // per output channel scale, group-major
  int col_scale_stride;        // per group
  int up_offset;               // gate_up: column offset of the up half inside col_scale
  const int* row_map;          // down: sorted row -> slot row (t*k + j)
  // router
  const float* bias;
  int topk;
  int renorm;
  float* topk_w;
  int* tile_counts;            // expert histogram rows (nullptr: none); zeroed before the launch
  int tile_count_stride;       // elements between the rows of consecutive m-tiles (0: one shared row)
};

template <int BN>
struct GemmCfg {
  static constexpr int kABytes = kBM * kKBlockBytes;
  static constexpr int kBBytes = BN * kKBlockBytes;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (BN >= 256) ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int kTmemCols = (2 * BN <= 32) ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512)));
  static constexpr int kBarBytes = 256;
  static constexpr size_t kSmemBytes =
      1024 + size_t(kStages) * kStageBytes + kBarBytes + sizeof(int) * (kMaxGroups + 1);
};

// Largest g with prefix[g] <= mt (prefix is non-decreasing, prefix[0] = 0).
__device__ __forceinline__ int find_group(const int* prefix, int G, int mt) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= mt) lo = mid; else hi = mid - 1;
  }
  return lo;
}

struct TileCoord {
  int g, m0, nt, row0, rows;
};

__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, const int* mt_prefix, int tile) {
  TileCoord c;
  const int mt = tile / p.n_tiles;
  c.nt = tile - mt * p.n_tiles;
  if (p.group_offsets == nullptr) {
    c.g = 0;
    c.m0 = mt * kBM;
    c.row0 = c.m0;
    c.rows = min(kBM, p.M - c.m0);
  } else {
    c.g = find_group(mt_prefix, p.num_groups, mt);
    c.m0 = (mt - mt_prefix[c.g]) * kBM;
    const int off = __ldg(p.group_offsets + c.g);
    const int cnt = __ldg(p.group_offsets + c.g + 1) - off;
    c.row0 = off + c.m0;
    c.rows = min(kBM, cnt - c.m0);
  }
  return c;
}

// ---------------------------------------------------------------------------- epilogues
// Each runs on the 128 epilogue threads; thread (quarter q, lane l) owns tile row 32q + l.
template <int BN, int EPI>
__device__ __forceinline__ void run_epilogue(const GemmParams& p, const TileCoord& c, uint32_t taddr,
                                             int row_local, int mt) {
  const bool valid = row_local < c.rows;
  const int row = c.row0 + row_local;
  uint32_t r[32];
  if constexpr (EPI == kEpiRawS32) {
    int32_t* out = static_cast<int32_t*>(p.out) + size_t(row) * p.ldo + size_t(c.nt) * p.out_col_step;
#pragma unroll 1
    for (int col = 0; col < BN; col += 32) {
      tmem_ld32(taddr + col, r);
      if (valid) {
        int4* dst = reinterpret_cast<int4*>(out + col);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_int4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
      }
    }
  } else if constexpr (EPI == kEpiGateUp) {
    // TMEM columns [0, BN/2) are gate channels, [BN/2, BN) the matching up channels.
    constexpr int HALF = BN / 2;
    const int hc0 = c.nt * HALF;  // first h column of this tile
    const float sx = valid ? __ldg(p.row_scale + row) : 0.0f;
    const float* sg = p.col_scale + size_t(c.g) * p.col_scale_stride + hc0;
    const float* su = sg + p.up_offset;
    uint16_t* out = static_cast<uint16_t*>(p.out) + size_t(row) * p.ldo + hc0;
    uint32_t ru[32];
#pragma unroll 1
    for (int col = 0; col < HALF; col += 32) {
      tmem_ld32(taddr + col, r);
      tmem_ld32(taddr + HALF + col, ru);
      uint32_t packed[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        float h2[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const float g = dequant(int32_t(r[i + j]), sx, __ldg(sg + col + i + j));
          const float u = dequant(int32_t(ru[i + j]), sx, __ldg(su + col + i + j));
          h2[j] = __fmul_rn(silu_exact(g), u);
        }
        packed[i / 2] = pack_bf16(h2[0], h2[1]);
      }
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
      }
    }
  } else if constexpr (EPI == kEpiDown || EPI == kEpiDense) {
    const int n0 = c.nt * p.out_col_step;
    const float srow = valid ? __ldg(p.row_scale + row) : 0.0f;
    const float* sc = p.col_scale + size_t(c.g) * p.col_scale_stride + n0;
    int orow = row;
    if constexpr (EPI == kEpiDown) orow = valid ? __ldg(p.row_map + row) : 0;
    uint16_t* out = static_cast<uint16_t*>(p.out) + size_t(orow) * p.ldo + n0;
#pragma unroll 1
    for (int col = 0; col < BN; col += 32) {
      tmem_ld32(taddr + col, r);
      uint32_t packed[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const float a = dequant(int32_t(r[i]), srow, __ldg(sc + col + i));
        const float b = dequant(int32_t(r[i + 1]), srow, __ldg(sc + col + i + 1));
        packed[i / 2] = pack_bf16(a, b);
      }
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
      }
    }
  } else if constexpr (EPI == kEpiRouter) {
    // One token per thread: logits of experts 0..E-1 in TMEM columns 0..E-1 (fp32).
    const int E = p.n_valid;
    const int k = p.topk;
    float tv[kMaxTopK];
    int ti[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) { tv[j] = -INFINITY; ti[j] = 0x7fffffff; }
#pragma unroll 1
    for (int col = 0; col < BN; col += 32) {
      tmem_ld32(taddr + col, r);
#pragma unroll 1
      for (int i = 0; i < 32; ++i) {
        const int e = col + i;
        if (e >= E) break;
        float l = __uint_as_float(r[i]);
        if (p.bias) l += __ldg(p.bias + e);
        // insert keeping descending values; equal values keep the lower expert first
        if (l > tv[k - 1]) {
          int pos = k - 1;
          while (pos > 0 && l > tv[pos - 1]) { tv[pos] = tv[pos - 1]; ti[pos] = ti[pos - 1]; --pos; }
          tv[pos] = l;
          ti[pos] = e;
        }
      }
    }
    // a slot left unfilled (only possible with non-finite logits) is reported, never used
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < k && (ti[j] < 0 || ti[j] >= E)) {
        atomicOr(&g_error_word, kErrBadIndex);
        ti[j] = j;
        tv[j] = tv[0];
      }
    }
    const float m = tv[0];
    float sel_sum = 0.0f;
    float ev[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      ev[j] = (j < k) ? expf(tv[j] - m) : 0.0f;
      sel_sum += ev[j];
    }
    float denom = sel_sum;
    if (!p.renorm) {
      denom = 0.0f;
#pragma unroll 1
      for (int col = 0; col < BN; col += 32) {
        tmem_ld32(taddr + col, r);
#pragma unroll 1
        for (int i = 0; i < 32; ++i) {
          const int e = col + i;
          if (e >= E) break;
          float l = __uint_as_float(r[i]);
          if (p.bias) l += __ldg(p.bias + e);
          denom += expf(l - m);
        }
      }
    }
    if (valid) {
      int* ids = static_cast<int*>(p.out) + size_t(row) * k;
      float* w = p.topk_w + size_t(row) * k;
      for (int j = 0; j < k; ++j) {
        ids[j] = ti[j];
        w[j] = ev[j] / denom;
      }
      if (p.tile_counts != nullptr) {
        int* counts = p.tile_counts + size_t(mt) * p.tile_count_stride;
        for (int j = 0; j < k; ++j) atomicAdd(counts + ti[j], 1);
      }
    }
  }
}

template <int BN, int EPI, int KIND>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  using Cfg = GemmCfg<BN>;
  constexpr int STAGES = Cfg::kStages;
  constexpr uint32_t IDESC = (KIND == kKindI8) ? idesc_s8s8s32(BN) : idesc_bf16f32(BN);
  constexpr int KB_ELEMS = (KIND == kKindI8) ? 128 : 64;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * Cfg::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + STAGES * Cfg::kBBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* mt_prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + Cfg::kBarBytes);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, globaltimer_ns() + p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull + a, 1); mbar_init(tempty + a, 4 * 32); }
    mbar_init(drain, 1);
    fence_mbar_init();
    *abort_flag = 0;
    // m-tile prefix over groups
    if (p.group_offsets != nullptr) {
      int acc = 0;
      mt_prefix[0] = 0;
      for (int g = 0; g < p.num_groups; ++g) {
        const int cnt = __ldg(p.group_offsets + g + 1) - __ldg(p.group_offsets + g);
        acc += (cnt + kBM - 1) / kBM;
        mt_prefix[g + 1] = acc;
      }
    } else {
      mt_prefix[0] = 0;
      mt_prefix[1] = (p.M + kBM - 1) / kBM;
    }
    tma_prefetch_map(&p.tmA);
    tma_prefetch_map(&p.tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int groups_for_prefix = (p.group_offsets != nullptr) ? p.num_groups : 1;
  const int total_tiles = mt_prefix[groups_for_prefix] * p.n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      for (int tile = blockIdx.x; tile < total_tiles && !*abort_flag; tile += gridDim.x) {
        const TileCoord c = decode_tile(p, mt_prefix, tile);
        const int b_row0 = c.g * p.b_rows_per_group + c.nt * p.b_n_step;
        const int b_row1 = b_row0 + p.b_half_offset;
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(empty + stage, phase ^ 1u, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(full + stage, Cfg::kStageBytes);
          const int x = kb * KB_ELEMS;
          tma_load_2d(sA + stage * Cfg::kABytes, &p.tmA, full + stage, x, c.row0);
          tma_load_2d(sB + stage * Cfg::kBBytes, &p.tmB, full + stage, x, b_row0);
          tma_load_2d(sB + stage * Cfg::kBBytes + Cfg::kBBytes / 2, &p.tmB, full + stage, x, b_row1);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        // let every load already issued land before the CTA's shared memory goes away
        volatile int no_abort = 0;
        const WaitCtx dw{&no_abort, globaltimer_ns() + 100000000ull};
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) mbar_wait(full + s, (issued_parity >> s) & 1u, dw);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued_any = false;
      for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
        if (!mbar_wait(tempty + acc, acc_phase ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + uint32_t(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(full + stage, phase, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_addr(sA + stage * Cfg::kABytes);
          const uint32_t b0 = smem_addr(sB + stage * Cfg::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kKBlockBytes / 32; ++kk)
            tc_mma<KIND>(d_tmem, sw128_kmajor_desc(a0 + kk * 32), sw128_kmajor_desc(b0 + kk * 32), IDESC,
                         (kb | kk) != 0 ? 1u : 0u);
          issued_any = true;
          tc_commit(empty + stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull + acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (*abort_flag && issued_any) {
        // wait for the MMAs already issued before TMEM is released
        tc_commit(drain);
        volatile int no_abort = 0;
        const WaitCtx dw{&no_abort, globaltimer_ns() + 100000000ull};
        mbar_wait(drain, 0, dw);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row_local = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x) {
      const TileCoord c = decode_tile(p, mt_prefix, tile);
      if (!mbar_wait(tfull + acc, acc_phase, wc)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * BN);
      run_epilogue<BN, EPI>(p, c, taddr, row_local, tile / p.n_tiles);
      tc_fence_before();
      mbar_arrive(tempty + acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
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
