// Grouped INT8 GEMM on CTA pairs (cta_group::2) for long token lists (prefill):
//
//   D[c, t] = sum_k W[c, k] * X[t, k]      (weights on the MMA's M side, token rows on its N side)
//
// One tile is (group g, block of at most 256 sorted token rows, block of channels) and is
// computed by the two CTAs of a cluster with one M = 256 MMA per K step: rank r supplies its
// 128 weight rows and its half of the token rows (N/2) from its own shared memory and receives
// the accumulators of its 128 weight rows for all N tokens in its own TMEM. Per SM and K-block
// that is 16 KB of weights + 16 KB of tokens for 128 x 256 x 128 MACs, twice the operand reuse of
// a one-CTA 128 x 128 tile, which is what the L2 -> SM bandwidth needs to keep the tensor pipe
// busy.
//   gate_up: a pair covers 128 channels; rank r's 128 weight rows are 4 x (16 gate rows, 16 up
//            rows) of channels cb*128 + 64r + [0, 64), so within every TMEM lane quarter lanes
//            0-15 hold gate and lanes 16-31 hold up of the same 16 channels, and one shuffle
//            pairs them for SiLU(gate) * up.
//   down / dense / raw: a pair covers 256 output channels, 128 per rank.
// Roles per CTA: warp 0 TMA producer (both ranks, completions counted on rank 0's barriers);
// warp 1 TMEM allocator (both) and MMA issuer (rank 0, one thread); warps 2.. the epilogue of
// the CTA's own 128 lanes, 3 (gate_up) or 4 warps per TMEM lane quarter taking 16-column chunks
// in turn. Two accumulator sets of 256 columns fill the TMEM, so the epilogue of one tile
// overlaps the MMAs of the next. Every wait is bounded (ptx.cuh).
#pragma once
#include "gemm.cuh"

namespace w8a8 {

constexpr int kPairNB = 256;  // token rows per tile (MMA N at most)

struct PairParams {
  CUtensorMap tmA;     // weights, 128-byte swizzle. gate_up: the 5-D view (k, row in 16, gate/up,
                       // 16-channel group, expert) with a (128 B, 16, 2, 4, 1) box; others: 128-row box
  CUtensorMap tmB128;  // token rows: 128-row box
  CUtensorMap tmB16;   // 16-row box
  CUtensorMap tmB8;    // 8-row box
  int num_kb;                // K-blocks of 128 bytes
  int n_cb;                  // channel blocks per group (gate_up: I / 128; others: ceil(N / 256))
  int num_groups;
  const int* group_offsets;  // [G+1] token-row offsets; nullptr: one group of M rows
  int M;
  int a_rows_per_group;      // gate_up: 2I; down: H; dense / raw: 0
  int n_channels;            // valid output channels per group (down / dense / raw)
  uint64_t timeout_ns;
  void* out;
  int ldo;
  const float* row_scale;
  const float* col_scale;
  int col_scale_stride;
  int up_offset;
  const int* row_map;
};

// Epilogue warps per CTA: several per TMEM lane quarter, so that while one waits on a TMEM or
// memory load the others issue.
template <int EPI>
struct PairCfg {
  static constexpr int kEpiWarps = (EPI == kEpiGateUp) ? 12 : 16;
  static constexpr int kThreads = 64 + 32 * kEpiWarps;
  static constexpr int kABytes = kBM * kKBlockBytes;           // 128 weight rows
  static constexpr int kBBytes = (kPairNB / 2) * kKBlockBytes;  // up to 128 token rows
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = 6;
  static constexpr int kAccCols = kPairNB;
  static constexpr int kTmemCols = 2 * kAccCols;
  static constexpr int kBarBytes = 512;
  // per accumulator set: the tile's row scales and row map, staged once for all epilogue warps
  static constexpr int kRowBytes = 2 * 2 * kPairNB * 4;
  // down / dense: per epilogue warp a 16-token x 32-channel bf16 block, transposed through
  // shared memory so that the output leaves in 16-byte row pieces
  static constexpr int kXposeBytes = (EPI == kEpiDown || EPI == kEpiDense) ? kEpiWarps * 16 * 32 * 2 : 0;
  static constexpr size_t kSmemBytes = 1024 + size_t(kStages) * kStageBytes + kBarBytes + kRowBytes + kXposeBytes +
                                       2 * sizeof(int) * (kMaxGroups + 1);
  static_assert(kTmemCols <= 512, "two accumulator sets must fit in TMEM");
  static_assert(kEpiWarps % 4 == 0, "whole lane quarters");
};

struct PairTile {
  int g, cb, tok0, rows, n;  // n: MMA N = rows rounded up to 16
};

// Decodes tile (mt, cb). `g_hint` is the group of an earlier token block (0 at first): every
// role walks its tiles in increasing order, so the group is found by stepping forward.
__device__ __forceinline__ PairTile pair_tile(const PairParams& p, const int* mt_prefix, const int* goff, int mt,
                                              int cb, int& g_hint) {
  PairTile c;
  c.cb = cb;
  int off, cnt, blk;
  if (p.group_offsets == nullptr) {
    c.g = 0;
    off = 0;
    cnt = p.M;
    blk = mt;
  } else {
    int g = g_hint;
    while (g + 1 < p.num_groups && mt_prefix[g + 1] <= mt) ++g;
    g_hint = g;
    c.g = g;
    off = goff[g];
    cnt = goff[g + 1] - off;
    blk = mt - mt_prefix[g];
  }
  c.tok0 = off + blk * kPairNB;
  c.rows = min(kPairNB, cnt - blk * kPairNB);
  c.n = (c.rows + 15) & ~15;
  return c;
}

// Runs process(r, j0) on this warp's 16-column chunks j0 = 16 wq, 16 wq + 16 W, ... < rows,
// loading each next chunk from TMEM while the current one is processed.
template <int W, typename F>
__device__ __forceinline__ void pair_chunks(uint32_t t_lane, int rows, int wq, F&& process) {
  constexpr int kStep = 16 * W;
  int j0 = wq * 16;
  if (j0 >= rows) return;
  uint32_t ra[16], rb[16];
  tmem_ld16_async(t_lane + j0, ra);
  tmem_wait16(ra);
  while (true) {
    const int j1 = j0 + kStep;
    if (j1 < rows) tmem_ld16_async(t_lane + j1, rb);
    process(ra, j0);
    if (j1 >= rows) break;
    tmem_wait16(rb);
    const int j2 = j1 + kStep;
    if (j2 < rows) tmem_ld16_async(t_lane + j2, ra);
    process(rb, j1);
    if (j2 >= rows) break;
    tmem_wait16(ra);
    j0 = j2;
  }
}

// A cluster's tiles in order: cluster, cluster + nclusters, ... as (token block mt, channel
// block cb), stepped without divisions.
struct PairTileIter {
  int mt, cb, dmt, dcb, n_cb;
  __device__ __forceinline__ PairTileIter(int first, int stride, int ncb) : n_cb(ncb) {
    mt = first / ncb;
    cb = first - mt * ncb;
    dmt = stride / ncb;
    dcb = stride - dmt * ncb;
  }
  __device__ __forceinline__ void next() {
    mt += dmt;
    cb += dcb;
    if (cb >= n_cb) { cb -= n_cb; ++mt; }
  }
};

// gate_up epilogue. Lane L of the warp's quarter holds gate (L < 16) or up (L >= 16) of channel
// `ch` for 16 token columns; the two halves swap 8 raw accumulators through one shuffle each, so
// that lane L < 16 owns (gate, up) of tokens 0-7 of the chunk and lane L + 16 those of tokens 8-15.
// srow: the tile's row scales in shared memory.
template <int W>
__device__ __forceinline__ void pair_epilogue_gate_up(const PairParams& p, const PairTile& c, uint32_t t_lane,
                                                      int ch, bool is_up, int wq, const float* srow) {
  const float sg = __ldg(p.col_scale + size_t(c.g) * p.col_scale_stride + ch);
  const float su = __ldg(p.col_scale + size_t(c.g) * p.col_scale_stride + p.up_offset + ch);
  uint16_t* out = static_cast<uint16_t*>(p.out) + ch;
  const size_t ldo = size_t(p.ldo);
  const int my0 = is_up ? 8 : 0;  // first token of the chunk this lane computes
  const int rows = c.rows;
  pair_chunks<W>(t_lane, rows, wq, [&](uint32_t(&r)[16], int j0) {
    const int nj = min(16, rows - j0);
    const float4 sa = *reinterpret_cast<const float4*>(srow + j0 + my0);
    const float4 sb = *reinterpret_cast<const float4*>(srow + j0 + my0 + 4);
    const float sx[8] = {sa.x, sa.y, sa.z, sa.w, sb.x, sb.y, sb.z, sb.w};
    float g[8], u[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t send = is_up ? r[j] : r[j + 8];
      const uint32_t recv = __shfl_xor_sync(0xffffffffu, send, 16);
      const int32_t ga = int32_t(is_up ? recv : r[j]);
      const int32_t ua = int32_t(is_up ? r[j + 8] : recv);
      g[j] = dequant(ga, sx[j], sg);
      u[j] = dequant(ua, sx[j], su);
    }
    float y[8];
    uint32_t exact = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      bool ok;
      y[j] = silu_mul_bf16_certified(g[j], u[j], ok);
      exact |= ok ? 0u : (1u << j);
    }
    exact &= (nj - my0 >= 8) ? 0xFFu : ((nj > my0) ? ((1u << (nj - my0)) - 1u) : 0u);  // stored tokens only
    if (exact != 0u) {  // rare: values the fast evaluation cannot certify
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if ((exact >> j) & 1u) y[j] = __fmul_rn(silu_exact(g[j]), u[j]);
    }
    uint32_t hb[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __nv_bfloat162 h2 = __floats2bfloat162_rn(y[2 * j], y[2 * j + 1]);
      hb[j] = *reinterpret_cast<const uint32_t*>(&h2);
    }
    const int row0 = c.tok0 + j0 + my0;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (my0 + j < nj) out[size_t(row0 + j) * ldo] = uint16_t(hb[j >> 1] >> (16 * (j & 1)));
  });
}

// down / dense / raw epilogue: lane = one output channel of the CTA's 128, columns = tokens.
// srow / smap: the tile's row scales and (down) output rows in shared memory; xp: this warp's
// 16 x 32 bf16 transpose block (down / dense).
template <int EPI, int W>
__device__ __forceinline__ void pair_epilogue_channels(const PairParams& p, const PairTile& c, uint32_t t_lane,
                                                       int ch, int wq, const float* srow, const int* smap,
                                                       uint16_t* xp) {
  const bool valid = ch < p.n_channels;
  const size_t ldo = size_t(p.ldo);
  const int rows = c.rows;
  if constexpr (EPI == kEpiRawS32) {
    int32_t* out = static_cast<int32_t*>(p.out) + ch;
    pair_chunks<W>(t_lane, rows, wq, [&](uint32_t(&r)[16], int j0) {
      const int nj = min(16, rows - j0);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (valid && j < nj) out[size_t(c.tok0 + j0 + j) * ldo] = int32_t(r[j]);
    });
  } else {
    // bf16 values go through this warp's 16 x 32 shared-memory block: lane = channel on the way
    // in, then four lanes per token row (8 channels = 16 bytes each) on the way out
    const float s_col = valid ? __ldg(p.col_scale + size_t(c.g) * p.col_scale_stride + ch) : 0.0f;
    const int lane = threadIdx.x & 31;
    const int ch0 = ch - lane;                      // first channel of the warp's 32
    const int jr = lane >> 2, cc = (lane & 3) * 8;  // token row (and row + 8), channel piece
    uint16_t* outb = static_cast<uint16_t*>(p.out) + ch0 + cc;
    pair_chunks<W>(t_lane, rows, wq, [&](uint32_t(&r)[16], int j0) {
      const int nj = min(16, rows - j0);
      float sr[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 f = *reinterpret_cast<const float4*>(srow + j0 + 4 * i);
        sr[4 * i] = f.x; sr[4 * i + 1] = f.y; sr[4 * i + 2] = f.z; sr[4 * i + 3] = f.w;
      }
#pragma unroll
      for (int j = 0; j < 16; j += 2) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(dequant(int32_t(r[j]), sr[j], s_col),
                                                        dequant(int32_t(r[j + 1]), sr[j + 1], s_col));
        const uint32_t v = *reinterpret_cast<const uint32_t*>(&h2);
        xp[j * 32 + lane] = uint16_t(v);
        xp[(j + 1) * 32 + lane] = uint16_t(v >> 16);
      }
      __syncwarp();
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int j = jr + 8 * hr;
        const uint4 piece = *reinterpret_cast<const uint4*>(xp + j * 32 + cc);
        if (j < nj && ch0 < p.n_channels) {
          const int orow = (EPI == kEpiDown) ? smap[j0 + j] : c.tok0 + j0 + j;
          *reinterpret_cast<uint4*>(outb + size_t(orow) * ldo) = piece;
        }
      }
      __syncwarp();  // the block is rewritten by the next chunk
    });
  }
}

template <int EPI>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<EPI>::kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ PairParams p) {
  using Cfg = PairCfg<EPI>;
  constexpr int STAGES = Cfg::kStages;
  constexpr int EW = Cfg::kEpiWarps;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * Cfg::kStageBytes);  // used on rank 0
  uint64_t* empty = full + STAGES;                                                  // each rank
  uint64_t* tfull = empty + STAGES;                                                 // each rank, [2]
  uint64_t* tempty = tfull + 2;                                                     // rank 0, [2]
  uint64_t* drain = tempty + 2;
  uint64_t* rready = drain + 1;                                                     // each rank, [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rready + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* rows_smem = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + Cfg::kBarBytes);  // [2][2][256]
  uint16_t* xpose = reinterpret_cast<uint16_t*>(rows_smem + 4 * kPairNB);  // [EW][16][32] (down / dense)
  int* mt_prefix = reinterpret_cast<int*>(reinterpret_cast<uint8_t*>(xpose) + Cfg::kXposeBytes);
  int* goff = mt_prefix + (kMaxGroups + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cluster = int(cluster_index());
  const int nclusters = int(cluster_count());
  const WaitCtx wc{abort_flag, p.timeout_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full + s, 1); mbar_init(empty + s, 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(tfull + a, 1); mbar_init(tempty + a, 2 * EW); }
    mbar_init(drain, 1);
    for (int a = 0; a < 2; ++a) mbar_init(rready + a, 32 * EW);
    fence_mbar_init();
    *abort_flag = 0;
    mt_prefix[0] = 0;
    if (p.group_offsets == nullptr) mt_prefix[1] = (p.M + kPairNB - 1) / kPairNB;
    tma_prefetch_map(&p.tmA);
    tma_prefetch_map(&p.tmB128);
    tma_prefetch_map(&p.tmB16);
    tma_prefetch_map(&p.tmB8);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish_pair();
  }
  // everything above touches only this CTA's own resources; inputs written by the previous
  // kernel in the stream are read only below
  pdl_wait();
  pdl_launch_dependents();
  if (p.group_offsets != nullptr && warp >= 2) {
    for (int g = threadIdx.x - 64; g <= p.num_groups; g += 32 * EW) goff[g] = __ldg(p.group_offsets + g);
    asm volatile("bar.sync 1, %0;" ::"r"(32 * EW) : "memory");
    if (warp == 2) {
      int carry = 0;
      for (int g0 = 0; g0 < p.num_groups; g0 += 32) {
        const int g = g0 + lane;
        const int v = (g < p.num_groups) ? (goff[g + 1] - goff[g] + kPairNB - 1) / kPairNB : 0;
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
  // barriers of both ranks initialised and the TMEM address published before any use
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int groups_for_prefix = (p.group_offsets != nullptr) ? p.num_groups : 1;
  const int total_mt = mt_prefix[groups_for_prefix];  // token blocks over all groups

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both ranks)
    // The whole warp runs the loop (converged, warp-uniform values); one elected lane issues.
    const uint32_t full0 = map_to_rank(smem_addr(full), 0);  // rank 0's full barriers
    int stage = 0, g_hint = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0, issued_parity = 0;
    bool ok = true;
    for (PairTileIter it(cluster, nclusters, p.n_cb); it.mt < total_mt && ok; it.next()) {
      const PairTile c = pair_tile(p, mt_prefix, goff, it.mt, it.cb, g_hint);
      const int hn = c.n >> 1;  // token rows this rank loads
      const uint32_t bytes = uint32_t(Cfg::kABytes + hn * kKBlockBytes);
      const int b_row = c.tok0 + int(rank) * hn;
      const int a_y = (EPI == kEpiGateUp) ? (c.cb * 128 + int(rank) * 64) / 16
                                          : c.g * p.a_rows_per_group + c.cb * 256 + int(rank) * 128;
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) { ok = false; break; }
        if (elect_one()) {
          uint8_t* sa = smem + stage * Cfg::kStageBytes;
          uint8_t* sb = sa + Cfg::kABytes;
          const uint32_t bar = full0 + uint32_t(stage) * 8u;
          if (leader) mbar_arrive_expect_tx(full + stage, 2u * bytes);
          const int x = kb * kKBlockBytes;
          if constexpr (EPI == kEpiGateUp) {
            // 4 x (16 gate rows, 16 up rows) of channels cb*128 + 64*rank + [0, 64), one copy
            tma_load_5d_pair(sa, &p.tmA, bar, x, 0, 0, a_y, c.g);
          } else {
            tma_load_2d_pair(sa, &p.tmA, bar, x, a_y);
          }
          if (hn == 128) {
            tma_load_2d_pair(sb, &p.tmB128, bar, x, b_row);
          } else {
            int b = 0;
            for (; b + 16 <= hn; b += 16) tma_load_2d_pair(sb + b * kKBlockBytes, &p.tmB16, bar, x, b_row + b);
            if (b < hn) tma_load_2d_pair(sb + b * kKBlockBytes, &p.tmB8, bar, x, b_row + b);
          }
        }
        __syncwarp();
        issued_mask |= 1u << stage;
        issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (ok) {
      // every stage released by the MMAs (their completions reach this CTA's barriers) before exit
      for (int i = 0; i < STAGES; ++i) {
        if (!mbar_wait_warp(empty + stage, phase ^ 1u, wc)) break;
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (lane == 0 && *abort_flag) {
      // let every load already issued land before the CTA's shared memory goes away: rank 0
      // sees both ranks' bytes on its barriers; rank 1 cannot observe them and waits 1 ms
      volatile int no_abort = 0;
      const WaitCtx dw{&no_abort, 100000000ull};
      if (leader) {
        for (int s = 0; s < STAGES; ++s)
          if (issued_mask & (1u << s)) mbar_wait(full + s, (issued_parity >> s) & 1u, dw);
      } else {
        const uint64_t until = globaltimer_ns() + 1000000ull;
        while (globaltimer_ns() < until) __nanosleep(10000);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    // Converged warp; descriptors are warp-uniform (stage and K offsets added to the 14-bit
    // start-address field, which cannot carry: shared memory ends below 256 KB); one elected
    // lane issues every MMA and commit.
    if (leader) {
      const uint32_t empty_own = smem_addr(empty), empty_peer = map_to_rank(smem_addr(empty), 1);
      const uint32_t tfull_own = smem_addr(tfull), tfull_peer = map_to_rank(smem_addr(tfull), 1);
      const uint64_t adesc0 = sw128_kmajor_desc(smem_addr(smem));
      int stage = 0, g_hint = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued_any = false;
      bool ok = true;
      for (PairTileIter it(cluster, nclusters, p.n_cb); it.mt < total_mt && ok; it.next()) {
        const PairTile c = pair_tile(p, mt_prefix, goff, it.mt, it.cb, g_hint);
        const uint32_t idesc = idesc_s8s8s32_m256(c.n);
        if (!mbar_wait_warp(tempty + acc, acc_phase ^ 1u, wc)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + uint32_t(acc * Cfg::kAccCols);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          // the stage's operands have landed (TMA completions on this barrier); the MMAs read
          // them through the same async proxy, so no tcgen05 fence is needed here (only at the
          // accumulator handoff above)
          if (!mbar_wait_warp(full + stage, phase, wc)) { ok = false; break; }
          if (elect_one()) {
            const uint64_t ad = adesc0 + uint64_t(stage * (Cfg::kStageBytes >> 4));
            const uint64_t bd = ad + uint64_t(Cfg::kABytes >> 4);
#pragma unroll
            for (int kk = 0; kk < kKBlockBytes / 32; ++kk)
              tc_mma_pair_i8(d0, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), idesc, (kb | kk) != 0 ? 1u : 0u);
            tc_commit_pair(empty_own + uint32_t(stage) * 8u);
            tc_commit_pair(empty_peer + uint32_t(stage) * 8u);
          }
          __syncwarp();
          issued_any = true;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) {
          tc_commit_pair(tfull_own + uint32_t(acc) * 8u);
          tc_commit_pair(tfull_peer + uint32_t(acc) * 8u);
        }
        __syncwarp();
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (ok) {
        // both epilogues have released both accumulators (their arrivals have landed here)
        for (int i = 0; i < 2; ++i) {
          if (!mbar_wait_warp(tempty + acc, acc_phase ^ 1u, wc)) break;
          if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
        }
      }
      if (lane == 0 && *abort_flag && issued_any) {
        // wait for the MMAs already issued (by lane 0, the elected lane of the converged warp)
        // before TMEM is released
        tc_commit_pair(smem_addr(drain));
        volatile int no_abort = 0;
        const WaitCtx dw{&no_abort, 100000000ull};
        mbar_wait(drain, 0, dw);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2.., both ranks)
    const int q = warp & 3;
    const int wq = (warp - 2) >> 2;  // index among the warps of this lane quarter
    const int et = threadIdx.x - 64;  // epilogue thread index
    const uint32_t tempty0 = map_to_rank(smem_addr(tempty), 0);
    int acc = 0, g_hint = 0;
    uint32_t acc_phase = 0;
    // Row scales (and output rows) of a tile are loaded into registers one tile ahead, so their
    // memory latency overlaps the previous tile's epilogue; thread et holds row et (< 256).
    static_assert(32 * EW >= kPairNB, "one row per epilogue thread");
    float pre_s = 0.0f;
    int pre_m = 0;
    auto load_rows = [&](const PairTile& t) {
      const bool in = et < t.rows;
      if constexpr (EPI != kEpiRawS32) pre_s = in ? __ldg(p.row_scale + t.tok0 + et) : 0.0f;
      if constexpr (EPI == kEpiDown) pre_m = in ? __ldg(p.row_map + t.tok0 + et) : 0;
    };
    PairTileIter it(cluster, nclusters, p.n_cb);
    PairTile c{};
    if (it.mt < total_mt) {
      c = pair_tile(p, mt_prefix, goff, it.mt, it.cb, g_hint);
      load_rows(c);
    }
    while (it.mt < total_mt) {
      // stage the tile's rows for all epilogue warps. The buffer of this accumulator set was last
      // read two tiles ago, and every epilogue thread has arrived on the previous tile's rready
      // barrier, so all of them are done with it. (An mbarrier, not a named barrier: its wait
      // is bounded, so a CTA that aborts cannot strand the others.)
      float* srow = rows_smem + acc * 2 * kPairNB;
      int* smap = reinterpret_cast<int*>(srow + kPairNB);
      if (et < kPairNB) {
        srow[et] = pre_s;
        smap[et] = pre_m;
      }
      mbar_arrive(rready + acc);
      if (!mbar_wait(rready + acc, acc_phase, wc)) break;
      PairTileIter nx = it;
      nx.next();
      PairTile cn{};
      if (nx.mt < total_mt) {
        cn = pair_tile(p, mt_prefix, goff, nx.mt, nx.cb, g_hint);
        load_rows(cn);
      }
      if (!mbar_wait(tfull + acc, acc_phase, wc)) break;
      tc_fence_after();
      const uint32_t t_lane = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc * Cfg::kAccCols);
      if constexpr (EPI == kEpiGateUp) {
        const int ch = c.cb * 128 + int(rank) * 64 + q * 16 + (lane & 15);
        pair_epilogue_gate_up<EW / 4>(p, c, t_lane, ch, lane >= 16, wq, srow);
      } else {
        pair_epilogue_channels<EPI, EW / 4>(p, c, t_lane, c.cb * 256 + int(rank) * 128 + q * 32 + lane, wq, srow,
                                            smap, xpose + (warp - 2) * 16 * 32);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + uint32_t(acc) * 8u);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      it = nx;
      c = cn;
    }
  }

  // no MMA, commit or remote arrival is outstanding in either CTA past this point
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::kTmemCols);
  }
}

}  // namespace w8a8
