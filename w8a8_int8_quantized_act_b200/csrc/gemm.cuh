// Persistent, warp-specialised grouped GEMM on the 5th-generation tensor cores (sm_100a).
//
//   D[m, n] = sum_k A[m, k] * B[n, k]      (A and B K-major; D accumulated in TMEM)
//
// The MMA's M side (128 TMEM lanes) holds A rows, its N side holds up to NB B rows.
//   * Expert GEMMs (kind::i8) put weight channels on M and token rows on N ("swap-AB"): a tile
//     is (expert g, token block of at most NB sorted rows, block of 128 channels), and the MMA
//     N is the token count of the block rounded up to 16, so decode tiles with a handful of
//     tokens stream their weights without dragging 128 activation rows along. gate_up loads
//     two A blocks per stage (128 gate rows and the matching 128 up rows) into two
//     accumulators, so one thread holds gate and up of the same channel.
//   * The router (kind::f16) puts 128 token rows on M and the E experts on N, so one thread
//     owns all logits of its token.
// Roles per CTA (one CTA per SM, 10 warps):
//   warp 0      TMA producer: 128-byte-swizzled K-blocks (128 bytes of K) into a ring of
//               STAGES shared-memory slots guarded by mbarrier full/empty pairs;
//   warp 1      TMEM allocator and MMA issuer (one thread): tcgen05.mma into one of two
//               accumulator sets, so the epilogue of a tile overlaps the next tile's MMAs;
//   warps 2-9   epilogue: tcgen05.ld of their TMEM lane quarter, fused dequantisation,
//               activation, routing, stores. Two warps share a quarter and split columns.
// Every mbarrier wait is bounded; a timeout aborts the CTA cleanly (see ptx.cuh).
#pragma once
#include "routing.cuh"

namespace w8a8 {

enum EpiKind : int {
  kEpiRawS32 = 0,   // int32 accumulators stored as they are (exact integer GEMM)
  kEpiRouter = 1,   // fp32 logits -> (+bias) softmax, top-k, weights, expert histogram
  kEpiGateUp = 2,   // int32 gate|up -> dequant, SiLU(gate)*up -> bf16 h
  kEpiDown = 3,     // int32 -> dequant -> bf16 o written to the assignment's slot row
  kEpiDense = 4,    // int32 -> dequant -> bf16 y (dense W8A8 linear)
};

constexpr int kBM = 128;            // MMA M (TMEM lanes)
constexpr int kKBlockBytes = 128;   // K bytes per pipeline stage (one swizzle row)
constexpr int kBBoxRows = 16;       // rows per TMA box on the N side
constexpr int kEpiWarps = 8;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxGroups = 1024;

struct GemmParams {
  CUtensorMap tmA;   // M side: boxes of 128 rows x 128 bytes
  CUtensorMap tmB;   // N side: boxes of 16 rows x 128 bytes (ragged tiles)
  CUtensorMap tmB2;  // N side: boxes of NB rows x 128 bytes (full tiles: one copy per stage)
  int num_kb;                  // K-blocks of 128 bytes
  int n_cb;                    // 128-channel blocks per group (router: 1)
  int num_groups;              // G
  const int* group_offsets;    // [G+1] token-row offsets (device); nullptr: one group of M rows
  int M;                       // token rows when group_offsets is null
  int a_rows_per_group;        // weight rows per group (gate_up: 2I, down: H, dense: 0)
  int a_second_offset;         // row offset of the second A block (gate_up: I; wide tiles: 128)
  int a_cb_step;               // A rows per channel block (128, or 256 with two 128-row blocks)
  int n_channels;              // valid output channels per group (second blocks past it are skipped)
  int nb_fixed;                // router: N side rows (E rounded up to 16); else 0
  uint64_t timeout_ns;         // bound on every mbarrier wait
  // epilogue operands
  void* out;                   // see EpiKind
  int ldo;                     // output row stride, elements
  int n_valid;                 // router: E
  const float* row_scale;      // per token-row scale (sx, or the requantisation scale of h)
  const float* col_scale;      // per channel scale, group-major
  int col_scale_stride;        // per group
  int up_offset;               // gate_up: offset of the up scales inside a group's scales
  const int* row_map;          // down: sorted row -> slot row (t*k + j)
  // router
  const float* bias;
  int topk;
  int renorm;
  float* topk_w;
  int* tile_counts;            // expert histogram rows (nullptr: none); zeroed before the launch
  int tile_count_stride;       // elements between the rows of consecutive 128-token chunks (0: one row)
  int router_rows;             // router: tokens per tile (32 or 64; the A map's box height)
  // down with the requantisation of h fused into the B operand (template QKB > 0): the bf16 rows
  // of h [rows, K] the CTA quantises itself, and where the tiles of channel block 0 leave the
  // codes and scales (hq [rows, K], s_h [rows])
  const uint16_t* qb_h;
  int8_t* qb_hq;
  float* qb_s;
};

// QKB > 0 (down GEMM of short token lists): the B operand of a tile is not loaded by TMA but made
// by the CTA itself from bf16 h, QKB K-blocks at most, into one of two resident buffers.
// Router tiles hold at most this many tokens (the A rows its TMA loads per K-block); its MMA keeps
// M = 128 and reads the stage's next bytes as rows 64-127, whose results nobody reads.
constexpr int kRouterMaxRows = 64;
constexpr int kRouterPitch = kRouterMaxRows + 1;  // floats per expert row of the transposed logits

template <int NA, int NB, int EPI, int QKB = 0>
struct GemmCfg {
  static constexpr int kABytes = (EPI == kEpiRouter ? kRouterMaxRows : kBM) * kKBlockBytes;
  static constexpr int kBBytes = NB * kKBlockBytes;
  static constexpr int kStageBytes = NA * kABytes + (QKB > 0 ? 0 : kBBytes);
  // router: logits of one tile transposed to [expert][token] (row pitch 65 floats, so both the
  // per-token writes and the per-expert reads are free of bank conflicts); resident B: two
  // buffers of QKB 128-byte-swizzled K-blocks of NB rows, then their row scales
  static constexpr int kQBBufBytes = QKB * NB * kKBlockBytes;
  static constexpr int kXBytes =
      (EPI == kEpiRouter) ? NB * kRouterPitch * 4 : (QKB > 0 ? 2 * kQBBufBytes + 2 * NB * 4 : 0);
  static_assert(QKB == 0 || (NB * kKBlockBytes) % 1024 == 0, "resident K-blocks sit on 1 KB boundaries");
  static constexpr int kStagesRaw = (196 * 1024 - kXBytes) / kStageBytes;
  static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
  static constexpr int kAccCols = NA * NB;  // TMEM columns of one accumulator set
  static constexpr int kTmemCols =
      (2 * kAccCols <= 32)
          ? 32
          : (2 * kAccCols <= 64 ? 64 : (2 * kAccCols <= 128 ? 128 : (2 * kAccCols <= 256 ? 256 : 512)));
  static constexpr int kBarBytes = 512;
  // after the barriers: token-block prefix [G+1], cached group offsets [G+1], router exchange
  static constexpr size_t kSmemBytes =
      1024 + size_t(kStages) * kStageBytes + kBarBytes + 2 * sizeof(int) * (kMaxGroups + 1) + kXBytes;
  static_assert(2 * kAccCols <= 512, "two accumulator sets must fit in TMEM");
  // (the router with 128 < E <= 256 keeps one stage: its transposed logits fill the rest)
  static_assert(kStages >= 2 || (EPI == kEpiRouter && kStages >= 1), "pipeline too shallow");
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

struct Tile {
  int g;       // group (expert)
  int cb;      // channel block (router: 0)
  int tok0;    // first token row of the tile
  int rows;    // valid token rows
  int a_row;   // first A row (weights, or router tokens)
  int b_row;   // first B row (tokens, or router experts)
  int nb;      // B rows loaded (multiple of 16) = MMA N
  int tt;      // token-tile index (router histogram row)
};

template <int EPI, int NB>
__device__ __forceinline__ Tile decode_tile(const GemmParams& p, const int* mt_prefix, const int* goff, int tile) {
  Tile c;
  if constexpr (EPI == kEpiRouter) {
    // router_rows tokens per tile (the MMA keeps M = 128: lanes past them compute values that
    // nobody reads); the histogram row is the tile's 128-token chunk
    c.g = 0;
    c.cb = 0;
    c.tok0 = tile * p.router_rows;
    c.tt = c.tok0 / kBM;
    c.rows = min(p.router_rows, p.M - c.tok0);
    c.a_row = c.tok0;
    c.b_row = 0;
    c.nb = p.nb_fixed;
  } else {
    const int mt = tile / p.n_cb;
    c.cb = tile - mt * p.n_cb;
    c.tt = mt;
    int off, cnt, blk;
    if (p.group_offsets == nullptr) {
      c.g = 0;
      off = 0;
      cnt = p.M;
      blk = mt;
    } else {
      c.g = find_group(mt_prefix, p.num_groups, mt);
      off = goff[c.g];
      cnt = goff[c.g + 1] - off;
      blk = mt - mt_prefix[c.g];
    }
    c.tok0 = off + blk * NB;
    c.rows = min(NB, cnt - blk * NB);
    c.a_row = c.g * p.a_rows_per_group + c.cb * p.a_cb_step;
    c.b_row = c.tok0;
    c.nb = (c.rows + 15) & ~15;
  }
  return c;
}

// 16 consecutive 32-bit TMEM columns of the warp's 32 lanes (wait included). TMEM is not
// addressable memory, so the statement carries no memory clobber: values already loaded from
// global or shared memory stay in registers across it.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

// 16 columns without the wait: the registers are valid only after tmem_wait16 on the same array,
// which names them as operands so that no use can move above it. Lets a warp load the next
// chunk while it computes on the current one.
__device__ __forceinline__ void tmem_ld16_async(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]));
}

// Two 16-column loads (e.g. the gate and up accumulators of the same tokens) behind one wait.
__device__ __forceinline__ void tmem_ld16x2(uint32_t ta, uint32_t tb, uint32_t (&a)[16], uint32_t (&b)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%32];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%33];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]),
        "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]), "=r"(b[15])
      : "r"(ta), "r"(tb));
}

// ---------------------------------------------------------------------------- epilogues
// Expert GEMM epilogues: thread = one channel (TMEM lane), columns = the tile's token rows.
// The two epilogue warps of a lane quarter take alternate 16-column chunks.
// tile_scale (down with a resident B): the tile's row scales in shared memory, indexed by the
// row's position in the tile; nullptr: p.row_scale in global memory, indexed by sorted row.
template <int EPI, int NB>
__device__ __forceinline__ void epilogue_channels(const GemmParams& p, const Tile& c, uint32_t t_lane, int lane_ch,
                                                  int half, const float* tile_scale = nullptr) {
  const int ch = c.cb * p.a_cb_step + lane_ch;  // channel within the group
  const size_t ldo = size_t(p.ldo);
  const float* __restrict__ row_scale = p.row_scale;
  uint32_t r[16];
  if constexpr (EPI == kEpiGateUp) {
    const float sg = __ldg(p.col_scale + size_t(c.g) * p.col_scale_stride + ch);
    const float su = __ldg(p.col_scale + size_t(c.g) * p.col_scale_stride + p.up_offset + ch);
    uint16_t* out = static_cast<uint16_t*>(p.out) + ch;
    uint32_t ru[16];
#pragma unroll 1
    for (int j0 = half * 16; j0 < c.rows; j0 += 32) {
      const int nj = min(16, c.rows - j0);
      const int row0 = c.tok0 + j0;
      // every load of the chunk before any store, so the 16 values are independent chains
      float sx[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) sx[j] = (j < nj) ? __ldg(row_scale + row0 + j) : 0.0f;
      tmem_ld16x2(t_lane + j0, t_lane + NB + j0, r, ru);  // gate | up accumulators
      uint32_t hb[16];
      uint32_t uncertified = 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const float g = dequant(int32_t(r[j]), sx[j], sg);
        const float u = dequant(int32_t(ru[j]), sx[j], su);
        bool ok;
        const float s = div_certified(g, __fadd_rn(1.0f, exp_cw(-g)), ok);
        uncertified |= ok ? 0u : (1u << j);
        hb[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(s, u)));
      }
      if (uncertified != 0u) {  // rare: quotients the fast divide could not prove
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if ((uncertified >> j) & 1u) {
            const float g = dequant(int32_t(r[j]), sx[j], sg);
            const float u = dequant(int32_t(ru[j]), sx[j], su);
            hb[j] = __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(silu_exact(g), u)));
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j < nj) out[size_t(row0 + j) * ldo] = uint16_t(hb[j]);
    }
  } else if constexpr (EPI == kEpiDown || EPI == kEpiDense) {
    // two 128-channel blocks: accumulator columns [0, NB) and [NB, 2NB)
    const bool second = ch + kBM < p.n_channels;
    const float sc0 = __ldg(p.col_scale + size_t(c.g) * p.col_scale_stride + ch);
    const float sc1 = second ? __ldg(p.col_scale + size_t(c.g) * p.col_scale_stride + ch + kBM) : 0.0f;
    const int* __restrict__ row_map = p.row_map;
    uint16_t* out = static_cast<uint16_t*>(p.out) + ch;
    uint32_t r1[16];
#pragma unroll 1
    for (int j0 = half * 16; j0 < c.rows; j0 += 32) {
      const int nj = min(16, c.rows - j0);
      const int row0 = c.tok0 + j0;
      float srow[16];
      int orow[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        srow[j] = (j < nj) ? (tile_scale != nullptr ? tile_scale[j0 + j] : __ldg(row_scale + row0 + j)) : 0.0f;
        orow[j] = (EPI == kEpiDown) ? ((j < nj) ? __ldg(row_map + row0 + j) : 0) : row0 + j;
      }
      tmem_ld16x2(t_lane + j0, t_lane + NB + j0, r, r1);
      uint32_t v0[16], v1[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        v0[j] = __bfloat16_as_ushort(__float2bfloat16_rn(dequant(int32_t(r[j]), srow[j], sc0)));
        v1[j] = __bfloat16_as_ushort(__float2bfloat16_rn(dequant(int32_t(r1[j]), srow[j], sc1)));
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j < nj) {
          uint16_t* o = out + size_t(orow[j]) * ldo;
          o[0] = uint16_t(v0[j]);
          if (second) o[kBM] = uint16_t(v1[j]);
        }
      }
    }
  } else if constexpr (EPI == kEpiRawS32) {
    int32_t* out = static_cast<int32_t*>(p.out) + ch;
    const bool second = ch + kBM < p.n_channels;
    uint32_t r1[16];
#pragma unroll 1
    for (int j0 = half * 16; j0 < c.rows; j0 += 32) {
      tmem_ld16(t_lane + j0, r);
      tmem_ld16(t_lane + NB + j0, r1);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (j0 + j < c.rows) {
          int32_t* o = out + size_t(c.tok0 + j0 + j) * ldo;
          o[0] = int32_t(r[j]);
          if (second) o[kBM] = int32_t(r1[j]);
        }
      }
    }
  }
}

// Router epilogue. The logits of a 128-token tile arrive one token per thread (TMEM lane);
// the two epilogue warps of each lane quarter copy half the experts each into shared memory,
// transposed to [expert][token]. After all 256 epilogue threads have written (bounded mbarrier),
// each warp takes whole tokens: lane l holds experts l, l+32, ... as order-preserving integer
// keys, and each of the k rounds is two warp reductions: the largest key, then the lowest
// expert holding it (equal values go to the lower expert). The winner's lane drops the entry.
// Lanes 0..k-1 end up holding pick j = lane, normalise and store them; a second barrier phase
// marks the buffer free for the CTA's next tile.
template <int NB>
__device__ __forceinline__ void epilogue_router(const GemmParams& p, const Tile& c, uint32_t t_lane, int lane_row,
                                                int half, int ew, float* xs, uint64_t* xbar, uint32_t& xphase,
                                                const WaitCtx& wc) {
  constexpr int SPAN = NB >= 32 ? NB / 2 : NB;  // experts each warp of a quarter copies
  constexpr int PER = (NB + 31) / 32;  // experts per lane in the per-token phase
  const int E = p.n_valid;
  const int k = p.topk;
  const float* __restrict__ bias = p.bias;
  // 1. TMEM -> shared memory, transposed (with 16 experts the lower warp copies them all; lane
  //    quarters past the tile's tokens are skipped)
  if ((NB >= 32 || half == 0) && lane_row - int(threadIdx.x & 31) < c.rows) {
    const int c0 = NB >= 32 ? half * SPAN : 0;
#pragma unroll
    for (int c16 = 0; c16 < SPAN; c16 += 16) {
      uint32_t r[16];
      tmem_ld16(t_lane + c0 + c16, r);
#pragma unroll
      for (int i = 0; i < 16; ++i) xs[(c0 + c16 + i) * kRouterPitch + lane_row] = __uint_as_float(r[i]);
    }
  }
  mbar_arrive(xbar);
  if (!mbar_wait(xbar, xphase, wc)) return;
  xphase ^= 1u;
  // 2. each warp takes tokens ew, ew + 8, ... four at a time (their selections interleaved)
  int* counts = p.tile_counts != nullptr ? p.tile_counts + size_t(c.tt) * p.tile_count_stride : nullptr;
  constexpr int NT = 4;
#pragma unroll 1
  for (int tb = ew; tb < c.rows; tb += kEpiWarps * NT) {
    const int nt = min(NT, (c.rows - tb + kEpiWarps - 1) / kEpiWarps);
    const int row = c.tok0 + tb;
    warp_topk_tokens<PER, NT>([&](int u, int e) { return xs[e * kRouterPitch + tb + u * kEpiWarps]; }, nt, E, k,
                              p.renorm != 0, bias, static_cast<int*>(p.out) + size_t(row) * k,
                              p.topk_w + size_t(row) * k, kEpiWarps * k, counts);
  }
  // 3. buffer free for the next tile once every epilogue thread is past step 2
  mbar_arrive(xbar);
  mbar_wait(xbar, xphase, wc);
  xphase ^= 1u;
}

template <int NA, int NB, int EPI, int KIND, int QKB = 0>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  using Cfg = GemmCfg<NA, NB, EPI, QKB>;
  constexpr int STAGES = Cfg::kStages;
  constexpr int KB_ELEMS = (KIND == kKindI8) ? 128 : 64;
  constexpr uint32_t IDESC0 = (KIND == kKindI8) ? idesc_s8s8s32(0) : idesc_bf16f32(0);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // QKB: the two resident B buffers (1 KB aligned after the stages) and their row scales [2][NB]
  uint8_t* qb_buf = smem + STAGES * Cfg::kStageBytes;
  float* qb_scale = reinterpret_cast<float*>(qb_buf + 2 * Cfg::kQBBufBytes);
  uint64_t* full =
      reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::kStageBytes + (QKB > 0 ? Cfg::kXBytes : 0));
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1 + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* mt_prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(full) + Cfg::kBarBytes);
  int* goff = mt_prefix + (kMaxGroups + 1);
  float* xs = reinterpret_cast<float*>(goff + (kMaxGroups + 1));  // router: [NB][65] logits
  uint64_t* xbar = drain + 1;  // router: all epilogue threads, two phases per tile
  uint64_t* bready = drain + 2;  // QKB: resident B buffer [2] written (all epilogue threads)
  uint64_t* bfree = drain + 4;   // QKB: resident B buffer [2] read by the tile's MMAs (commit)
  uint64_t* ebar = drain + 6;    // QKB: all epilogue threads done with a tile's row scales

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const WaitCtx wc{abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull + a, 1); mbar_init(tempty + a, kEpiWarps * 32); }
    mbar_init(drain, 1);
    mbar_init(xbar, 32 * kEpiWarps);
    for (int b = 0; b < 2; ++b) { mbar_init(bready + b, 32 * kEpiWarps); mbar_init(bfree + b, 1); }
    mbar_init(ebar, 32 * kEpiWarps);
    fence_mbar_init();
    *abort_flag = 0;
    mt_prefix[0] = 0;
    if (!(EPI != kEpiRouter && p.group_offsets != nullptr))
      mt_prefix[1] = (EPI == kEpiRouter) ? (p.M + p.router_rows - 1) / p.router_rows : (p.M + NB - 1) / NB;
    tma_prefetch_map(&p.tmA);
    tma_prefetch_map(&p.tmB);
    tma_prefetch_map(&p.tmB2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  // everything above touches only this CTA's own resources; inputs written by the previous
  // kernel in the stream are read only below
  pdl_wait();
  pdl_launch_dependents();
  if (EPI != kEpiRouter && p.group_offsets != nullptr && warp >= 2) {
    // cache the group offsets and build the token-block prefix: one warp-wide scan per 32 groups
    for (int g = threadIdx.x - 64; g <= p.num_groups; g += 32 * kEpiWarps) goff[g] = __ldg(p.group_offsets + g);
    asm volatile("bar.sync 1, %0;" ::"r"(32 * kEpiWarps) : "memory");
    if (warp == 2) {
      int carry = 0;
      for (int g0 = 0; g0 < p.num_groups; g0 += 32) {
        const int g = g0 + lane;
        const int v = (g < p.num_groups) ? (goff[g + 1] - goff[g] + NB - 1) / NB : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += u;
        }
        if (g < p.num_groups) mt_prefix[g + 1] = carry + incl;
        carry += __shfl_sync(0xffffffffu, incl, 31);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int groups_for_prefix = (EPI != kEpiRouter && p.group_offsets != nullptr) ? p.num_groups : 1;
  const int total_tiles = mt_prefix[groups_for_prefix] * p.n_cb;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // The whole warp runs the loop (converged, warp-uniform values); one elected lane issues.
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x) {
      const Tile c = decode_tile<EPI, NB>(p, mt_prefix, goff, tile);
      const uint32_t a_bytes = (EPI == kEpiRouter) ? uint32_t(p.router_rows * kKBlockBytes) : uint32_t(Cfg::kABytes);
      const uint32_t bytes = uint32_t(NA * a_bytes + (QKB > 0 ? 0 : c.nb * kKBlockBytes));
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) { ok = false; break; }
        if (elect_one()) {
          uint8_t* st = smem + stage * Cfg::kStageBytes;
          mbar_arrive_expect_tx(full + stage, bytes);
          const int x = kb * KB_ELEMS;
          tma_load_2d(st, &p.tmA, full + stage, x, c.a_row);
          if (NA == 2) tma_load_2d(st + Cfg::kABytes, &p.tmA, full + stage, x, c.a_row + p.a_second_offset);
          uint8_t* sb = st + NA * Cfg::kABytes;
          if constexpr (QKB == 0) {
            if (c.nb == NB) {
              tma_load_2d(sb, &p.tmB2, full + stage, x, c.b_row);
            } else {
              for (int b = 0; b < c.nb; b += kBBoxRows)
                tma_load_2d(sb + b * kKBlockBytes, &p.tmB, full + stage, x, c.b_row + b);
            }
          }
        }
        __syncwarp();
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (lane == 0 && *abort_flag) {
      // let every load already issued land before the CTA's shared memory goes away
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, 100000000ull};
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) mbar_wait(full + s, (issued_parity >> s) & 1u, dw);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Converged warp; descriptors are warp-uniform (stage and K offsets added to the 14-bit
    // start-address field, which cannot carry: shared memory ends below 256 KB); one elected
    // lane issues every MMA and commit.
    const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(smem));
    const uint64_t qdesc0 = sw128_kmajor_desc(smem_addr(qb_buf));
    int stage = 0;
    uint32_t phase = 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    int local_tile = 0;
    bool issued_any = false;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total_tiles && ok; tile += gridDim.x, ++local_tile) {
      const Tile c = decode_tile<EPI, NB>(p, mt_prefix, goff, tile);
      const uint32_t idesc = IDESC0 | (uint32_t(c.nb >> 3) << 17);
      const int qb = local_tile & 1;
      if (!mbar_wait_warp(tempty + acc, acc_phase ^ 1u, wc)) break;
      if constexpr (QKB > 0) {
        // the tile's resident B (written by the epilogue warps, fenced for the async proxy)
        if (!mbar_wait_warp(bready + qb, uint32_t(local_tile >> 1) & 1u, wc)) break;
      }
      tc_fence_after();
      const uint32_t d0 = tmem_base + uint32_t(acc * Cfg::kAccCols);
      for (int kb = 0; kb < p.num_kb; ++kb) {
        // TMA completions on this barrier; the MMAs read the stage through the same async proxy
        if (!mbar_wait_warp(full + stage, phase, wc)) { ok = false; break; }
        if (elect_one()) {
          const uint64_t ad = adesc0 + uint64_t(stage * (Cfg::kStageBytes >> 4));
          const uint64_t bd = (QKB > 0) ? qdesc0 + uint64_t((qb * Cfg::kQBBufBytes + kb * NB * kKBlockBytes) >> 4)
                                        : ad + uint64_t(NA * (Cfg::kABytes >> 4));
#pragma unroll
          for (int kk = 0; kk < kKBlockBytes / 32; ++kk) {
            const uint32_t accum = (kb | kk) != 0 ? 1u : 0u;
            tc_mma<KIND>(d0, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), idesc, accum);
            if (NA == 2)
              tc_mma<KIND>(d0 + NB, ad + uint64_t((Cfg::kABytes >> 4) + 2 * kk), bd + uint64_t(2 * kk), idesc,
                           accum);
          }
          tc_commit(empty + stage);
        }
        __syncwarp();
        issued_any = true;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) {
        tc_commit(tfull + acc);
        if constexpr (QKB > 0) tc_commit(bfree + qb);  // the resident B may be rewritten
      }
      __syncwarp();
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0 && *abort_flag && issued_any) {
      // wait for the MMAs already issued (by lane 0, the elected lane of the converged warp)
      // before TMEM is released
      tc_commit(drain);
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, 100000000ull};
      mbar_wait(drain, 0, dw);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;             // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;   // which of the quarter's two warps
    const int lane_idx = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t xphase = 0;
    // Resident B (QKB > 0): the epilogue warps quantise each tile's bf16 h rows into one of two
    // shared-memory buffers, warp w taking rows w, w + 8, ...: the row maximum, the scale and the
    // codes exactly as the per-row requantisation kernel computes them (quant_row_warp), written as
    // 128-byte swizzled K-blocks; the tiles of channel block 0 also leave the codes and scales in
    // global memory (hq, s_h). A tile's buffer is made two tiles ahead, once the MMAs of the tile
    // that last used it have completed and every epilogue thread is done with its row scales.
    auto make_b = [&](const Tile& t, int b) {
      if constexpr (QKB > 0) {
        const int K = p.num_kb * kKBlockBytes;
        uint8_t* buf = qb_buf + b * Cfg::kQBBufBytes;
        for (int r = warp - 2; r < t.rows; r += kEpiWarps) {
          const float sc = quant_row_warp<QKB / 2>(p.qb_h + size_t(t.tok0 + r) * K, K, [&](int i, uint2 v) {
            const int kb = i >> 7, ch16 = (i & 127) >> 4, hv = (i >> 3) & 1;
            *reinterpret_cast<uint2*>(buf + kb * (NB * kKBlockBytes) + r * kKBlockBytes + ((ch16 ^ (r & 7)) << 4) +
                                      hv * 8) = v;
            if (t.cb == 0) *reinterpret_cast<uint2*>(p.qb_hq + size_t(t.tok0 + r) * K + i) = v;
          });
          if (lane == 0) {
            qb_scale[b * NB + r] = sc;
            if (t.cb == 0) p.qb_s[t.tok0 + r] = sc;
          }
        }
        fence_proxy_async_smem();  // generic-proxy writes become visible to the tensor core
        mbar_arrive(bready + b);
      }
    };
    if constexpr (QKB > 0) {
      for (int i = 0; i < 2; ++i) {
        const int tl = int(blockIdx.x) + i * int(gridDim.x);
        if (tl < total_tiles) make_b(decode_tile<EPI, NB>(p, mt_prefix, goff, tl), i);
      }
    }
    uint32_t ephase = 0;
    int local_tile = 0;
    for (int tile = blockIdx.x; tile < total_tiles; tile += gridDim.x, ++local_tile) {
      const Tile c = decode_tile<EPI, NB>(p, mt_prefix, goff, tile);
      if (!mbar_wait(tfull + acc, acc_phase, wc)) break;
      tc_fence_after();
      const uint32_t t_lane = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * Cfg::kAccCols);
      const int qb = local_tile & 1;
      if constexpr (EPI == kEpiRouter) {
        epilogue_router<NB>(p, c, t_lane, lane_idx, half, warp - 2, xs, xbar, xphase, wc);
      } else {
        epilogue_channels<EPI, NB>(p, c, t_lane, lane_idx, half, QKB > 0 ? qb_scale + qb * NB : nullptr);
      }
      tc_fence_before();
      mbar_arrive(tempty + acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      if constexpr (QKB > 0) {
        const int t2 = tile + 2 * int(gridDim.x);
        if (t2 < total_tiles) {
          mbar_arrive(ebar);  // every epilogue thread is done with this tile's row scales
          if (!mbar_wait(ebar, ephase, wc)) break;
          ephase ^= 1u;
          if (!mbar_wait(bfree + qb, uint32_t(local_tile >> 1) & 1u, wc)) break;
          make_b(decode_tile<EPI, NB>(p, mt_prefix, goff, t2), qb);
        }
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
