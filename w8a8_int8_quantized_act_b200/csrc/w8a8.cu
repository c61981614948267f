// libw8a8: C ABI entry points (declared in include/w8a8.h). Host code only checks arguments,
// encodes TMA tensor maps and launches the kernels; every step of the path runs on the GPU.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdlib.h>

#include <mutex>
#include <vector>

#include "../../include/w8a8.h"
#include "elementwise.cuh"
#include "front.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "gemm_w4a8.cuh"
#include "mxfp8.cuh"

namespace w8a8 {
namespace {

constexpr int kVersion = 220;  // 0.2.2

cudaStream_t as_stream(w8a8_stream s) { return static_cast<cudaStream_t>(s); }

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cached[dev] = n > 0 ? n : 148;
  }
  return cached[dev];
}

uint64_t wait_timeout_ns() {
  static uint64_t ns = [] {
    const char* env = getenv("W8A8_WAIT_TIMEOUT_MS");
    const double ms = env ? atof(env) : 2000.0;
    return uint64_t((ms > 0 ? ms : 2000.0) * 1e6);
  }();
  return ns;
}

// ------------------------------------------------------------------ TMA tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D K-major map over [rows, inner] elements with a (box_rows x 128-byte) box, 128-byte swizzle,
// zero fill outside the tensor.
bool make_kmajor_map(CUtensorMap* m, const void* base, bool bf16, uint64_t inner, uint64_t rows,
                     uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || inner == 0) return false;
  const uint32_t esize = bf16 ? 2 : 1;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * esize};
  const cuuint32_t box[2] = {128u / esize, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D K-major map over packed 4-bit rows [rows, inner values] (inner / 2 bytes a row) with a
// (box_rows x 128-value) box of the 16U4_ALIGN16B type: each 8 bytes of 16 codes land in 16
// bytes of shared memory (the padded 4-bit operand layout of the block-scaled MMA), 128-byte
// swizzle. The type needs a 32-byte aligned base, rows of a multiple of 32 bytes and inner a
// multiple of 128 values.
bool make_kmajor_map_e2m1(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || inner == 0 || inner % 128 || (reinterpret_cast<uintptr_t>(base) & 31u)) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner / 2};
  const cuuint32_t box[2] = {128u, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over [rows, inner_bytes] bytes with an unswizzled (box_rows x box_bytes) box.
bool make_plain_map(CUtensorMap* m, const void* base, uint64_t inner_bytes, uint64_t rows, uint32_t box_bytes,
                    uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows == 0 || inner_bytes == 0) return false;
  const cuuint64_t dims[2] = {inner_bytes, rows};
  const cuuint64_t strides[1] = {inner_bytes};
  const cuuint32_t box[2] = {box_bytes, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// gate_up weights [E, 2I, H] int8 seen as the 5-D tensor (k, row within a 16-channel group,
// gate or up half, 16-channel group, expert), so that one (128 B, 16, 2, 4, 1) box brings
// 4 x (16 gate rows, the matching 16 up rows): the interleaved 128-row tile of the pair GEMM.
// Every coordinate range stays inside the tensor.
bool make_gate_up_pair_map(CUtensorMap* m, const void* base, uint64_t H, uint64_t I, uint64_t E) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || H == 0 || I % 64 || E == 0) return false;
  const cuuint64_t dims[5] = {H, 16, 2, I / 16, E};
  const cuuint64_t strides[4] = {H, I * H, 16 * H, 2 * I * H};
  const cuuint32_t box[5] = {128, 16, 2, 4, 1};
  const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ launch helpers
int launch_status() { return cudaGetLastError() == cudaSuccess ? W8A8_OK : W8A8_ERR_LAUNCH; }

// Launches `kern` with programmatic stream serialization: it may begin while the previous
// kernel in the stream finishes (each kernel waits in pdl_wait() before using its inputs).
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess ? W8A8_OK : W8A8_ERR_LAUNCH;
}

template <int NA, int NB, int EPI, int KIND, int QKB = 0>
int launch_gemm(const GemmParams& p, int max_tiles, cudaStream_t stream) {
  using Cfg = GemmCfg<NA, NB, EPI, QKB>;
  auto kern = gemm_tc_kernel<NA, NB, EPI, KIND, QKB>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Cfg::kSmemBytes)) !=
      cudaSuccess)
    return W8A8_ERR_LAUNCH;
  const int grid = max(1, min(num_sms(), max_tiles));
  return launch_pdl(kern, dim3(grid), dim3(kGemmThreads), Cfg::kSmemBytes, stream, p);
}

// Clusters of gemm_pair_kernel<EPI> that fit on the device at once (one CTA per SM), cached.
template <int EPI>
int pair_clusters() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  if (cached[dev] == 0) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(unsigned(num_sms() & ~1), 1, 1);
    cfg.blockDim = dim3(PairCfg<EPI>::kThreads, 1, 1);
    cfg.dynamicSmemBytes = PairCfg<EPI>::kSmemBytes;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<EPI>, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms() / 2;
    }
    cached[dev] = n;
  }
  return cached[dev];
}

template <int EPI>
int launch_pair(const PairParams& p, int max_tiles, cudaStream_t stream) {
  auto kern = gemm_pair_kernel<EPI>;
  using Cfg = PairCfg<EPI>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Cfg::kSmemBytes)) != cudaSuccess)
    return W8A8_ERR_LAUNCH;
  const int clusters = max(1, min(pair_clusters<EPI>(), max_tiles));
  return launch_pdl(kern, dim3(2 * clusters), dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, p);
}

// Token-row maps of a K-major int8 operand for the pair kernel: 128-, 16- and 8-row boxes.
bool make_pair_b_maps(PairParams* p, const void* base, uint64_t inner, uint64_t rows) {
  return make_kmajor_map(&p->tmB128, base, false, inner, rows, 128) &&
         make_kmajor_map(&p->tmB16, base, false, inner, rows, 16) &&
         make_kmajor_map(&p->tmB8, base, false, inner, rows, 8);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

// Router column tile: the smallest supported MMA N that covers E experts.
int router_bn(int64_t E) {
  for (int bn : {16, 32, 64, 128, 256})
    if (E <= bn) return bn;
  return 0;
}

int check_moe_shape(int64_t T, int64_t H, int64_t E, int k, int64_t I) {
  if (T < 0 || H <= 0 || E <= 0 || I <= 0 || k <= 0) return W8A8_ERR_ARG;
  if (k > E) return W8A8_ERR_ARG;
  if (H % 128 || I % 128 || E > 256 || k > kMaxTopK) return W8A8_ERR_UNSUPPORTED;
  if (T * k >= (int64_t(1) << 31) / 2) return W8A8_ERR_UNSUPPORTED;
  if (E * 2 * I >= (int64_t(1) << 31) || E * H >= (int64_t(1) << 31)) return W8A8_ERR_UNSUPPORTED;
  return W8A8_OK;
}

// Token block of the expert GEMMs: 32 rows when experts see few tokens (decode), else 256 on
// CTA pairs.
bool small_token_blocks(int64_t A, int64_t E) { return A <= 32 * E; }

void fill_layout(int64_t T, int64_t H, int64_t E, int k, int64_t I, w8a8_moe_ws_layout* L) {
  const int64_t A = T * k;
  const int64_t Ap = round_up(A > 0 ? A : 1, 128);
  const int64_t C = (T + kChunk - 1) / kChunk;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L->topk_ids = take(sizeof(int32_t) * A);
  L->topk_w = take(sizeof(float) * A);
  L->tile_counts = take(sizeof(int32_t) * C * E);
  L->offsets = take(sizeof(int32_t) * (E + 1));
  L->perm = take(sizeof(int32_t) * A);
  L->sx = take(sizeof(float) * T);
  L->sx_sorted = take(sizeof(float) * Ap);
  L->xq = take(size_t(Ap) * H);
  L->h = take(size_t(Ap) * I * 2);
  L->s_h = take(sizeof(float) * Ap);
  L->hq = take(size_t(Ap) * I);
  L->o = take(size_t(A) * H * 2);
  L->logits = take(sizeof(float) * T * E);
  L->sync = take(sizeof(uint32_t));
  L->total = off;
}

// Shared-expert regions after the routed layer's (the routed offsets are those of fill_layout).
void fill_shared_layout(int64_t T, int64_t H, int64_t E, int k, int64_t I, int64_t Is, w8a8_moe_shared_ws_layout* L) {
  fill_layout(T, H, E, k, I, &L->routed);
  size_t off = L->routed.total;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  L->xq = take(size_t(T) * H);
  L->sx = take(sizeof(float) * T);
  L->h = take(size_t(T) * Is * 2);
  L->s_h = take(sizeof(float) * T);
  L->hq = take(size_t(T) * Is);
  L->o = take(size_t(T) * H * 2);
  L->gate = take(sizeof(float) * T);
  L->total = off;
}

// Router: tcgen05 bf16 GEMM with the softmax / top-k epilogue. tile_counts is zeroed here.
// counts: expert histogram rows (nullptr: none) with `count_stride` elements between the rows of
// consecutive 128-token tiles (0: every tile adds into one row of E counters).
// Short batches (T <= kSmallRouterMaxT): fp32 logits on the CUDA cores spread over many CTAs,
// then a warp-per-token top-k; `logits` is T*E floats of scratch. Longer batches: the
// tensor-core router with the top-k in its epilogue (logits unused).
constexpr int64_t kSmallRouterMaxT = 512;

int run_router_small(const uint16_t* x, const uint16_t* wg, const float* bias, int64_t T, int64_t H, int64_t E,
                     int k, int renorm, int* ids, float* w, int* counts, int64_t count_stride, float* logits,
                     cudaStream_t stream) {
  const dim3 grid1(unsigned((E + 7) / 8), unsigned((T + kSmallRouterTokens - 1) / kSmallRouterTokens));
  const dim3 blk(256);
  const int Ti = int(T), Hi = int(H), Ei = int(E);
  const size_t xs_bytes = sizeof(uint16_t) * size_t(kSmallRouterTokens) * size_t(H);  // <= 32 KB (H <= 4096)
  int rc;
  switch (row_units(Hi)) {
    case 1: rc = launch_pdl(router_logits_small_kernel<1>, grid1, blk, xs_bytes, stream, x, wg, Ti, Hi, Ei, logits); break;
    case 2: rc = launch_pdl(router_logits_small_kernel<2>, grid1, blk, xs_bytes, stream, x, wg, Ti, Hi, Ei, logits); break;
    case 4: rc = launch_pdl(router_logits_small_kernel<4>, grid1, blk, xs_bytes, stream, x, wg, Ti, Hi, Ei, logits); break;
    case 8: rc = launch_pdl(router_logits_small_kernel<8>, grid1, blk, xs_bytes, stream, x, wg, Ti, Hi, Ei, logits); break;
    case 16: rc = launch_pdl(router_logits_small_kernel<16>, grid1, blk, xs_bytes, stream, x, wg, Ti, Hi, Ei, logits); break;
    default: return W8A8_ERR_UNSUPPORTED;
  }
  if (rc != W8A8_OK) return rc;
  const dim3 grid2(unsigned((T + 7) / 8));
  const int cs = int(count_stride);
  switch ((E + 31) / 32) {
    case 1: return launch_pdl(router_topk_kernel<1>, grid2, blk, 0, stream, logits, bias, Ti, Ei, k, renorm, ids, w, counts, cs);
    case 2: return launch_pdl(router_topk_kernel<2>, grid2, blk, 0, stream, logits, bias, Ti, Ei, k, renorm, ids, w, counts, cs);
    case 3:
    case 4: return launch_pdl(router_topk_kernel<4>, grid2, blk, 0, stream, logits, bias, Ti, Ei, k, renorm, ids, w, counts, cs);
    default: return launch_pdl(router_topk_kernel<8>, grid2, blk, 0, stream, logits, bias, Ti, Ei, k, renorm, ids, w, counts, cs);
  }
}

int run_router(const uint16_t* x, const uint16_t* wg, const float* bias, int64_t T, int64_t H, int64_t E, int k,
               int renorm, int* ids, float* w, int* counts, int64_t count_stride, float* logits,
               cudaStream_t stream) {
  const int nb = router_bn(E);
  // 64 tokens per tile (the top-k epilogue spreads over twice as many CTAs as with 128: 128 of
  // them for 8192 tokens), or 32 where that still fits the SMs in one wave (4096 tokens: 128
  // CTAs instead of 64; each CTA streams all of W_gate, so fewer tokens per CTA leave the bytes
  // per CTA nearly unchanged but use twice the SMs)
  const int kRouterRows = (T + 31) / 32 <= num_sms() ? 32 : kRouterMaxRows;
  GemmParams p{};
  if (!make_kmajor_map(&p.tmA, x, true, H, T, kRouterRows) || !make_kmajor_map(&p.tmB, wg, true, H, E, kBBoxRows) ||
      !make_kmajor_map(&p.tmB2, wg, true, H, E, uint32_t(nb)))
    return W8A8_ERR_UNSUPPORTED;
  const int64_t C = (T + kChunk - 1) / kChunk;
  if (counts != nullptr) {
    const size_t rows = count_stride ? size_t(C) : 1;
    if (cudaMemsetAsync(counts, 0, sizeof(int) * rows * E, stream) != cudaSuccess) return W8A8_ERR_LAUNCH;
  }
  if (logits != nullptr && T <= kSmallRouterMaxT && H <= 4096)
    return run_router_small(x, wg, bias, T, H, E, k, renorm, ids, w, counts, count_stride, logits, stream);
  p.num_kb = int(H / 64);
  p.n_cb = 1;
  p.num_groups = 1;
  p.group_offsets = nullptr;
  p.M = int(T);
  p.nb_fixed = nb;
  p.timeout_ns = wait_timeout_ns();
  p.out = ids;
  p.n_valid = int(E);
  p.bias = bias;
  p.topk = k;
  p.renorm = renorm;
  p.topk_w = w;
  p.tile_counts = counts;
  p.tile_count_stride = int(count_stride);
  p.router_rows = kRouterRows;
  const int tiles = int((T + kRouterRows - 1) / kRouterRows);
  switch (nb) {
    case 16: return launch_gemm<1, 16, kEpiRouter, kKindBF16>(p, tiles, stream);
    case 32: return launch_gemm<1, 32, kEpiRouter, kKindBF16>(p, tiles, stream);
    case 64: return launch_gemm<1, 64, kEpiRouter, kKindBF16>(p, tiles, stream);
    case 128: return launch_gemm<1, 128, kEpiRouter, kKindBF16>(p, tiles, stream);
    default: return launch_gemm<1, 256, kEpiRouter, kKindBF16>(p, tiles, stream);
  }
}

// Launches quant_rows_kernel with the register depth that fits rows of K values.
// MXFP8 codes and scales of the bf16 rows src [R, K].
int launch_mx_rows(const w8a8_bf16* src, int64_t R, int K, uint8_t* codes, uint8_t* scales, cudaStream_t s) {
  const int64_t items = R * ((K + 255) / 256);
  const dim3 grid(unsigned((items + kMxWarps - 1) / kMxWarps));
  return launch_pdl(mx_quant_rows_kernel, grid, dim3(kMxWarps * 32), 0, s, reinterpret_cast<const uint16_t*>(src), R,
                    K, codes, scales);
}

// MXFP4 weights (packed E2M1 codes and E8M0 scales) of the bf16 rows src [R, K].
int launch_mx4_rows(const w8a8_bf16* src, int64_t R, int K, uint8_t* packed, uint8_t* scales, cudaStream_t s) {
  const int64_t items = R * ((K + 255) / 256);
  const dim3 grid(unsigned((items + kMxWarps - 1) / kMxWarps));
  return launch_pdl(mx4_quant_rows_kernel, grid, dim3(kMxWarps * 32), 0, s, reinterpret_cast<const uint16_t*>(src),
                    R, K, packed, scales);
}

// MX GEMMs with more token rows than this (and N a multiple of 256) run on CTA pairs.
constexpr int64_t kMxPairMinRows = 192;

// Weight map of the MX GEMMs: E4M3 codes [N, K] or packed E2M1 codes [N, K/2], 128-row box.
template <int WF>
bool make_mx_weight_map(CUtensorMap* m, const uint8_t* wc, int64_t K, int64_t N) {
  if constexpr (WF == kMxE2M1) return make_kmajor_map_e2m1(m, wc, uint64_t(K), uint64_t(N), 128);
  return make_kmajor_map(m, wc, false, uint64_t(K), uint64_t(N), 128);
}

// y [M, N] = the MX product of token codes / scales (MXFP8) and weight codes / scales (MXFP8, or
// MXFP4 for WF = kMxE2M1) on the block-scaled MMA. K % 128 == 0, N % 128 == 0; checked by the
// callers.
template <int WF>
int mx_gemm(const uint8_t* xc, const uint8_t* xs, const uint8_t* wc, const uint8_t* ws, int64_t M, int64_t K,
            int64_t N, w8a8_bf16* y, cudaStream_t s) {
  if (M > kMxPairMinRows && N % 256 == 0) {
    MxPairParams q{};
    if (!make_mx_weight_map<WF>(&q.tmA, wc, K, N) || !make_kmajor_map(&q.tmB, xc, false, K, M, kMxPairHalf))
      return W8A8_ERR_UNSUPPORTED;
    q.sfa = reinterpret_cast<const uint32_t*>(ws);
    q.sfb = reinterpret_cast<const uint32_t*>(xs);
    q.num_kb = int(K / 128);
    q.n_cb = int(N / 256);
    q.M = int(M);
    q.N = int(N);
    q.y = reinterpret_cast<uint16_t*>(y);
    q.timeout_ns = wait_timeout_ns();
    auto kern = mx_pair_kernel<WF>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kMxPairSmemBytes)) != cudaSuccess)
      return W8A8_ERR_LAUNCH;
    const int tiles = int((M + kMxPairNB - 1) / kMxPairNB) * q.n_cb;
    const int clusters = max(1, min(num_sms() / 2, tiles));
    return launch_pdl(kern, dim3(2 * clusters), dim3(kMxPairThreads), kMxPairSmemBytes, s, q);
  }
  MxGemmParams p{};
  if (!make_mx_weight_map<WF>(&p.tmA, wc, K, N) || !make_kmajor_map(&p.tmB, xc, false, K, M, 128))
    return W8A8_ERR_UNSUPPORTED;
  p.sfa = reinterpret_cast<const uint32_t*>(ws);
  p.sfb = reinterpret_cast<const uint32_t*>(xs);
  p.num_kb = int(K / 128);
  p.n_cb = int(N / 128);
  p.M = int(M);
  p.N = int(N);
  p.y = reinterpret_cast<uint16_t*>(y);
  p.timeout_ns = wait_timeout_ns();
  auto kern = mx_gemm_kernel<WF>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kMxSmemBytes)) != cudaSuccess)
    return W8A8_ERR_LAUNCH;
  const int tiles = int((M + kMxNB - 1) / kMxNB) * p.n_cb;
  return launch_pdl(kern, dim3(max(1, min(num_sms(), tiles))), dim3(kMxThreads), kMxSmemBytes, s, p);
}

// quant_rows_stream_kernel<U> over R rows: as many CTAs as are resident at once (cached per U),
// fewer for short inputs.
template <int U>
int launch_quant_rows_stream(const uint16_t* src, int64_t R, int K, int8_t* q, float* scale, cudaStream_t s) {
  static const int per_sm = [] {
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, quant_rows_stream_kernel<U>, kRowWarps * 32, 0) !=
            cudaSuccess ||
        b < 1)
      b = 1;
    return b;
  }();
  const int64_t want = (R + kRowWarps - 1) / kRowWarps;
  const int64_t resident = int64_t(num_sms()) * per_sm;
  const dim3 grid(unsigned(want < resident ? want : resident)), blk(kRowWarps * 32);
  return launch_pdl(quant_rows_stream_kernel<U>, grid, blk, 0, s, src, R, K, q, scale);
}

int launch_quant_rows(const uint16_t* src, int64_t R, int K, int8_t* q, float* scale, cudaStream_t s) {
  // rows of 768 and 1536 values (the h rows of the 30B- and 235B-shaped layers) hold exactly 3
  // and 6 vectors a lane, which leaves room for more resident warps than 4 and 8
  const int u = (K + 255) / 256;
  if (u == 3) return launch_quant_rows_stream<3>(src, R, K, q, scale, s);
  if (u == 5 || u == 6) return launch_quant_rows_stream<6>(src, R, K, q, scale, s);
  switch (row_units(K)) {
    case 1: return launch_quant_rows_stream<1>(src, R, K, q, scale, s);
    case 2: return launch_quant_rows_stream<2>(src, R, K, q, scale, s);
    case 4: return launch_quant_rows_stream<4>(src, R, K, q, scale, s);
    case 8: return launch_quant_rows_stream<8>(src, R, K, q, scale, s);
    case 16: return launch_quant_rows_stream<16>(src, R, K, q, scale, s);
    default: {
      const dim3 grid(unsigned((R + kRowWarps - 1) / kRowWarps)), blk(kRowWarps * 32);
      return launch_pdl(quant_rows_kernel<0>, grid, blk, 0, s, src, R, K, q, scale);
    }
  }
}

int launch_group_quant(dim3 grid, size_t smem, cudaStream_t s, const uint16_t* x, const int* ids,
                       const int* tile_counts, int T, int H, int E, int k, int* offsets, int* perm, float* sx,
                       float* sx_sorted, int8_t* xq) {
  switch (row_units(H)) {
#define W8A8_GQ(U_)                                                                                        \
  case U_:                                                                                                 \
    return launch_pdl(group_quant_kernel<U_>, grid, dim3(kPermThreads), smem, s, x, ids, tile_counts, T, H, E, k, \
                      offsets, perm, sx, sx_sorted, xq);
    W8A8_GQ(1) W8A8_GQ(2) W8A8_GQ(4) W8A8_GQ(8) W8A8_GQ(16) W8A8_GQ(0)
#undef W8A8_GQ
  }
  return W8A8_ERR_UNSUPPORTED;
}

// The fused short-batch front end (front.cuh): one cooperative launch of up to one CTA per SM
// (all resident at once, which its grid barriers need), for rows of at most kFrontMaxH values
// (the router's token rows are staged in shared memory, the weight slices kept in registers).
template <int RU, int PER>
int launch_front_t(const uint16_t* x, const uint16_t* wg, const float* bias, int T, int H, int E, int k, int renorm,
                   float* logits, unsigned* sync, int* ids, float* w, int* tile_counts, int* offsets, int* perm,
                   float* sx, float* sx_sorted, int8_t* xq, cudaStream_t s) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(unsigned(min(num_sms(), kFrontMaxT)));
  cfg.blockDim = dim3(kFrontThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const uint64_t timeout = wait_timeout_ns();
  return cudaLaunchKernelEx(&cfg, front_small_kernel<RU, PER>, x, wg, bias, T, H, E, k, renorm, logits, sync,
                            timeout, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq) == cudaSuccess
             ? W8A8_OK
             : W8A8_ERR_LAUNCH;
}

template <int RU>
int launch_front_per(const uint16_t* x, const uint16_t* wg, const float* bias, int T, int H, int E, int k,
                     int renorm, float* logits, unsigned* sync, int* ids, float* w, int* tile_counts, int* offsets,
                     int* perm, float* sx, float* sx_sorted, int8_t* xq,
                     cudaStream_t s) {
  switch ((E + 31) / 32) {
    case 1: return launch_front_t<RU, 1>(x, wg, bias, T, H, E, k, renorm, logits, sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
    case 2: return launch_front_t<RU, 2>(x, wg, bias, T, H, E, k, renorm, logits, sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
    case 3:
    case 4: return launch_front_t<RU, 4>(x, wg, bias, T, H, E, k, renorm, logits, sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
    default: return launch_front_t<RU, 8>(x, wg, bias, T, H, E, k, renorm, logits, sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
  }
}

int launch_front_small(const uint16_t* x, const uint16_t* wg, const float* bias, int T, int H, int E, int k,
                       int renorm, float* logits, unsigned* sync, int* ids, float* w, int* tile_counts, int* offsets,
                       int* perm, float* sx, float* sx_sorted, int8_t* xq,
                     cudaStream_t s) {
  switch (row_units(H)) {
    case 1: return launch_front_per<1>(x, wg, bias, T, H, E, k, renorm, logits, sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
    case 2: return launch_front_per<2>(x, wg, bias, T, H, E, k, renorm, logits, sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
    case 4: return launch_front_per<4>(x, wg, bias, T, H, E, k, renorm, logits, sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
    case 8: return launch_front_per<8>(x, wg, bias, T, H, E, k, renorm, logits, sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
    default: return W8A8_ERR_UNSUPPORTED;
  }
}

// Upper bound of the number of token blocks of `nb` rows over all groups: ceil(A/nb) + min(E, A).
int max_token_blocks(int64_t A, int64_t E, int nb) { return int((A + nb - 1) / nb + (E < A ? E : A)); }

// Dense GEMMs with more token rows than this run on CTA pairs.
constexpr int64_t kPairMinRows = 128;


// CTAs per 128-token chunk of the grouping kernel (each re-derives the chunk's positions and
// quantises every 8th token of the chunk).
int group_quant_splits() { return 8; }

}  // namespace
}  // namespace w8a8

using namespace w8a8;

extern "C" {

int w8a8_version(void) { return kVersion; }

const char* w8a8_status_string(int status) {
  switch (status) {
    case W8A8_OK: return "ok";
    case W8A8_ERR_ARG: return "bad argument (null pointer or inconsistent size)";
    case W8A8_ERR_UNSUPPORTED: return "unsupported shape or alignment";
    case W8A8_ERR_WORKSPACE: return "workspace too small";
    case W8A8_ERR_LAUNCH: return "CUDA launch or runtime error";
    case W8A8_ERR_DEVICE: return "device error word set (a bounded wait ran out or an index was invalid)";
    default: return "unknown status";
  }
}

int w8a8_check_status(w8a8_stream stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return W8A8_ERR_LAUNCH;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return W8A8_ERR_LAUNCH;
  if (word != 0) {
    const unsigned int zero = 0;
    cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero));
    return W8A8_ERR_DEVICE;
  }
  return W8A8_OK;
}

int w8a8_quantize_weight_per_channel(const w8a8_bf16* w, int64_t G, int64_t N, int64_t K, int8_t* q, float* scale,
                                     w8a8_stream stream) {
  if (G < 0 || N < 0 || K <= 0) return W8A8_ERR_ARG;
  const int64_t R = G * N;
  if (R == 0) return W8A8_OK;
  if (!w || !q || !scale) return W8A8_ERR_ARG;
  if (K % 8 || !aligned16(w) || (K % 16 && !aligned16(q)) || K > (1 << 30)) return W8A8_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(q) & 7u) return W8A8_ERR_UNSUPPORTED;
  return launch_quant_rows(w, R, int(K), q, scale, as_stream(stream));
}

int w8a8_quantize_weight_int4_per_group(const w8a8_bf16* w, int64_t N, int64_t K, int group, uint8_t* packed,
                                        float* scale, w8a8_stream stream) {
  if (N < 0 || K <= 0 || group <= 0) return W8A8_ERR_ARG;
  if (group != 128 || K % group) return W8A8_ERR_UNSUPPORTED;
  if (N == 0) return W8A8_OK;
  if (!w || !packed || !scale) return W8A8_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(w) & 7u) || (reinterpret_cast<uintptr_t>(packed) & 1u))
    return W8A8_ERR_UNSUPPORTED;
  const int64_t items = N * (K / group);
  const int64_t blocks = (items + kRowWarps - 1) / kRowWarps;
  quant_int4_group128_kernel<<<unsigned(blocks), kRowWarps * 32, 0, as_stream(stream)>>>(w, N, int(K), packed,
                                                                                        scale);
  return launch_status();
}

int w8a8_quant_act_per_token(const w8a8_bf16* x, int64_t T, int64_t K, int8_t* q, float* scale,
                             w8a8_stream stream) {
  if (T < 0 || K <= 0) return W8A8_ERR_ARG;
  if (T == 0) return W8A8_OK;
  if (!x || !q || !scale) return W8A8_ERR_ARG;
  if (K % 8 || !aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 7u) || K > (1 << 30))
    return W8A8_ERR_UNSUPPORTED;
  return launch_quant_rows(x, T, int(K), q, scale, as_stream(stream));
}

int w8a8_moe_route(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, int64_t T, int64_t H, int64_t E,
                   int k, int renorm, int32_t* topk_ids, float* topk_w, int32_t* expert_counts,
                   w8a8_stream stream) {
  if (T < 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return W8A8_ERR_ARG;
  if (H % 128 || E > 256 || k > kMaxTopK) return W8A8_ERR_UNSUPPORTED;
  if (T == 0) {
    if (expert_counts) return cudaMemsetAsync(expert_counts, 0, sizeof(int) * E, as_stream(stream)) == cudaSuccess
                                  ? W8A8_OK : W8A8_ERR_LAUNCH;
    return W8A8_OK;
  }
  if (!x || !wg || !topk_ids || !topk_w) return W8A8_ERR_ARG;
  if (!aligned16(x) || !aligned16(wg)) return W8A8_ERR_UNSUPPORTED;
  // every tile adds its tokens' experts into the single row expert_counts[E]
  return run_router(x, wg, bias, T, H, E, k, renorm, topk_ids, topk_w, expert_counts, 0, nullptr, as_stream(stream));
}

int w8a8_moe_workspace_layout(int64_t T, int64_t H, int64_t E, int k, int64_t I, w8a8_moe_ws_layout* layout) {
  if (!layout) return W8A8_ERR_ARG;
  const int st = check_moe_shape(T, H, E, k, I);
  if (st != W8A8_OK) return st;
  fill_layout(T, H, E, k, I, layout);
  return W8A8_OK;
}

size_t w8a8_moe_workspace_size(int64_t T, int64_t H, int64_t E, int k, int64_t I) {
  w8a8_moe_ws_layout L;
  return w8a8_moe_workspace_layout(T, H, E, k, I, &L) == W8A8_OK ? L.total : 0;
}

}  // extern "C"

namespace w8a8 {
namespace {

// Records stage event `i` (if events were supplied) on the stream.
inline void mark(void* const* events, int i, cudaStream_t s) {
  if (events != nullptr && events[i] != nullptr) cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
}

int linear_gemm(const int8_t* xq, const float* sx, const void* wq, const float* sw, int w_format, int64_t M,
                int64_t K, int64_t N, w8a8_bf16* y, cudaStream_t s);

// The shared expert of a layer (bf16 gate [H], packed int8 gate_up [2Is, H] with its scales,
// int8 down [H, Is] with its scales).
struct SharedExpert {
  const w8a8_bf16* wsg;
  const int8_t* wgu;
  const float* s_gu;
  const int8_t* wd;
  const float* s_d;
  int64_t Is;
};

// Dense gate_up GEMM of every token (one group of T rows in token order) with the dequant +
// SiLU(gate)*up epilogue: h [T, Is] from xq [T, H], sx [T] and the packed weight [2Is, H].
int dense_gate_up(const int8_t* xq, const float* sx, const int8_t* wgu, const float* s_gu, int64_t T, int64_t H,
                  int64_t Is, uint16_t* h, cudaStream_t s) {
  if (T > kPairMinRows) {
    PairParams p{};
    if (!make_gate_up_pair_map(&p.tmA, wgu, H, Is, 1) || !make_pair_b_maps(&p, xq, H, T)) return W8A8_ERR_UNSUPPORTED;
    p.num_kb = int(H / 128);
    p.n_cb = int(Is / 128);
    p.num_groups = 1;
    p.M = int(T);
    p.a_rows_per_group = int(2 * Is);
    p.n_channels = int(Is);
    p.timeout_ns = wait_timeout_ns();
    p.out = h;
    p.ldo = int(Is);
    p.row_scale = sx;
    p.col_scale = s_gu;
    p.col_scale_stride = int(2 * Is);
    p.up_offset = int(Is);
    return launch_pair<kEpiGateUp>(p, int((T + kPairNB - 1) / kPairNB) * p.n_cb, s);
  }
  GemmParams p{};
  if (!make_kmajor_map(&p.tmA, wgu, false, H, uint64_t(2 * Is), 128) ||
      !make_kmajor_map(&p.tmB, xq, false, H, T, kBBoxRows) || !make_kmajor_map(&p.tmB2, xq, false, H, T, 32))
    return W8A8_ERR_UNSUPPORTED;
  p.num_kb = int(H / 128);
  p.n_cb = int(Is / 128);
  p.num_groups = 1;
  p.M = int(T);
  p.a_rows_per_group = int(2 * Is);
  p.a_second_offset = int(Is);
  p.a_cb_step = 128;
  p.timeout_ns = wait_timeout_ns();
  p.out = h;
  p.ldo = int(Is);
  p.row_scale = sx;
  p.col_scale = s_gu;
  p.col_scale_stride = int(2 * Is);
  p.up_offset = int(Is);
  return launch_gemm<2, 32, kEpiGateUp, kKindI8>(p, int((T + 31) / 32) * p.n_cb, s);
}

// Steps 1 and 2 of the forward: routing, the grouping of the T*k assignments by expert and the
// per-token quantisation into the sorted rows, into the workspace regions of L.
int route_group_stage(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, int64_t T, int64_t H, int64_t E,
                      int k, int renorm, uint8_t* ws, const w8a8_moe_ws_layout& L, cudaStream_t s,
                      void* const* ev) {
  int* ids = reinterpret_cast<int*>(ws + L.topk_ids);
  float* w = reinterpret_cast<float*>(ws + L.topk_w);
  int* tile_counts = reinterpret_cast<int*>(ws + L.tile_counts);
  int* offsets = reinterpret_cast<int*>(ws + L.offsets);
  int* perm = reinterpret_cast<int*>(ws + L.perm);
  float* sx = reinterpret_cast<float*>(ws + L.sx);
  float* sx_sorted = reinterpret_cast<float*>(ws + L.sx_sorted);
  int8_t* xq = reinterpret_cast<int8_t*>(ws + L.xq);
  const int C = int((T + kChunk - 1) / kChunk);
  int rc;
  if (T <= kFrontMaxT && H <= kFrontMaxH) {
    // short batch: routing, grouping and quantisation in one cooperative launch
    mark(ev, 0, s);
    unsigned* sync = reinterpret_cast<unsigned*>(ws + L.sync);
    if (cudaMemsetAsync(sync, 0, sizeof(unsigned), s) != cudaSuccess) return W8A8_ERR_LAUNCH;
    rc = launch_front_small(x, wg, bias, int(T), int(H), int(E), k, renorm, reinterpret_cast<float*>(ws + L.logits),
                            sync, ids, w, tile_counts, offsets, perm, sx, sx_sorted, xq, s);
    if (rc != W8A8_OK) return rc;
    mark(ev, 1, s);
    return W8A8_OK;
  }
  // 1. router (bf16 tcgen05 GEMM + softmax / top-k epilogue, per-chunk expert histogram)
  mark(ev, 0, s);
  rc = run_router(x, wg, bias, T, H, E, k, renorm, ids, w, tile_counts, E, reinterpret_cast<float*>(ws + L.logits),
                  s);
  if (rc != W8A8_OK) return rc;
  // 2. group assignments by expert and quantise every token once into its sorted rows
  const size_t gq_smem = sizeof(int) * (2 * E + 2 * kChunk * k + 4 * E);
  mark(ev, 1, s);
  return launch_group_quant(dim3(C, group_quant_splits()), gq_smem, s, x, ids, tile_counts, int(T), int(H), int(E),
                            k, offsets, perm, sx, sx_sorted, xq);
}

// Operands of the grouped expert FFN: A sorted token rows xq [round_up(A, 128), H] with their
// scales, G groups of consecutive rows (offsets [G+1] on the device; group g uses expert g), the
// intermediates h, s_h, hq (round_up(A, 128) rows) and the output o; row_map sends sorted row r
// to output row row_map[r].
struct ExpertRows {
  const int8_t* xq;
  const float* sx;
  const int* offsets;
  uint16_t* h;
  float* s_h;
  int8_t* hq;
  uint16_t* o;
  const int* row_map;
};

// Steps 3-5 of the forward: grouped gate_up with dequant + SiLU(gate)*up, the requantisation of h,
// grouped down with dequant; the G = Ew experts are held in wgu [Ew, 2I, H] / wd [Ew, H, I].
int experts_stage(const ExpertRows& b, int64_t A, int64_t G, int64_t Ew, int64_t H, int64_t I,
                  const int8_t* wgu, const float* s_gu, const int8_t* wd, const float* s_d, cudaStream_t s,
                  void* const* ev) {
  const int64_t Ap = round_up(A > 0 ? A : 1, 128);
  int rc;
  // Few rows per group (decode): the expert GEMMs run one CTA per tile of <= 32 sorted rows;
  // otherwise CTA pairs on tiles of <= 256 rows.
  const bool small = small_token_blocks(A, G);

  // 3. grouped gate_up GEMM (weights on M, tokens on N) with the dequant + SiLU(gate)*up
  //    epilogue -> h
  if (small) {
    GemmParams p{};
    if (!make_kmajor_map(&p.tmA, wgu, false, H, uint64_t(Ew) * 2 * I, 128) ||
        !make_kmajor_map(&p.tmB, b.xq, false, H, Ap, kBBoxRows) || !make_kmajor_map(&p.tmB2, b.xq, false, H, Ap, 32))
      return W8A8_ERR_UNSUPPORTED;
    p.num_kb = int(H / 128);
    p.n_cb = int(I / 128);
    p.num_groups = int(G);
    p.group_offsets = b.offsets;
    p.a_rows_per_group = int(2 * I);
    p.a_second_offset = int(I);
    p.a_cb_step = 128;
    p.timeout_ns = wait_timeout_ns();
    p.out = b.h;
    p.ldo = int(I);
    p.row_scale = b.sx;
    p.col_scale = s_gu;
    p.col_scale_stride = int(2 * I);
    p.up_offset = int(I);
    const int tiles = max_token_blocks(A, G, 32) * p.n_cb;
    mark(ev, 2, s);
    if ((rc = launch_gemm<2, 32, kEpiGateUp, kKindI8>(p, tiles, s)) != W8A8_OK) return rc;
  } else {
    PairParams p{};
    if (!make_gate_up_pair_map(&p.tmA, wgu, H, I, Ew) || !make_pair_b_maps(&p, b.xq, H, Ap))
      return W8A8_ERR_UNSUPPORTED;
    p.num_kb = int(H / 128);
    p.n_cb = int(I / 128);
    p.num_groups = int(G);
    p.group_offsets = b.offsets;
    p.a_rows_per_group = int(2 * I);
    p.n_channels = int(I);
    p.timeout_ns = wait_timeout_ns();
    p.out = b.h;
    p.ldo = int(I);
    p.row_scale = b.sx;
    p.col_scale = s_gu;
    p.col_scale_stride = int(2 * I);
    p.up_offset = int(I);
    const int tiles = max_token_blocks(A, G, kPairNB) * p.n_cb;
    mark(ev, 2, s);
    if ((rc = launch_pair<kEpiGateUp>(p, tiles, s)) != W8A8_OK) return rc;
  }

  // 4. per-row requantisation of h: inside the down GEMM for short token lists with rows of up
  //    to 1024 values (each CTA quantises its tile's rows into shared memory), else a launch of
  //    its own
  const bool rq_in_down = small && I <= 1024;
  mark(ev, 3, s);
  if (!rq_in_down && (rc = launch_quant_rows(b.h, A, int(I), b.hq, b.s_h, s)) != W8A8_OK) return rc;

  // 5. grouped down GEMM with the dequant epilogue -> o (rows through row_map)
  if (small) {
    GemmParams p{};
    if (!make_kmajor_map(&p.tmA, wd, false, I, uint64_t(Ew) * H, 128) ||
        !make_kmajor_map(&p.tmB, b.hq, false, I, Ap, kBBoxRows) || !make_kmajor_map(&p.tmB2, b.hq, false, I, Ap, 32))
      return W8A8_ERR_UNSUPPORTED;
    p.num_kb = int(I / 128);
    p.n_cb = int((H + 255) / 256);
    p.n_channels = int(H);
    p.num_groups = int(G);
    p.group_offsets = b.offsets;
    p.a_rows_per_group = int(H);
    p.a_second_offset = 128;
    p.a_cb_step = 256;
    p.timeout_ns = wait_timeout_ns();
    p.out = b.o;
    p.ldo = int(H);
    p.row_scale = b.s_h;
    p.col_scale = s_d;
    p.col_scale_stride = int(H);
    p.row_map = b.row_map;
    const int tiles = max_token_blocks(A, G, 32) * p.n_cb;
    mark(ev, 4, s);
    if (rq_in_down) {
      p.qb_h = b.h;
      p.qb_hq = b.hq;
      p.qb_s = b.s_h;
      rc = launch_gemm<2, 32, kEpiDown, kKindI8, 8>(p, tiles, s);
    } else {
      rc = launch_gemm<2, 32, kEpiDown, kKindI8>(p, tiles, s);
    }
    return rc;
  }
  PairParams p{};
  if (!make_kmajor_map(&p.tmA, wd, false, I, uint64_t(Ew) * H, 128) || !make_pair_b_maps(&p, b.hq, I, Ap))
    return W8A8_ERR_UNSUPPORTED;
  p.num_kb = int(I / 128);
  p.n_cb = int((H + 255) / 256);
  p.n_channels = int(H);
  p.num_groups = int(G);
  p.group_offsets = b.offsets;
  p.a_rows_per_group = int(H);
  p.timeout_ns = wait_timeout_ns();
  p.out = b.o;
  p.ldo = int(H);
  p.row_scale = b.s_h;
  p.col_scale = s_d;
  p.col_scale_stride = int(H);
  p.row_map = b.row_map;
  const int tiles = max_token_blocks(A, G, kPairNB) * p.n_cb;
  mark(ev, 4, s);
  return launch_pair<kEpiDown>(p, tiles, s);
}

int moe_forward_impl(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                     const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H, int64_t E, int k,
                     int64_t I, int renorm, void* workspace, size_t workspace_bytes, w8a8_bf16* y,
                     w8a8_stream stream, void* const* ev, const SharedExpert* sh = nullptr) {
  const int st = check_moe_shape(T, H, E, k, I);
  if (st != W8A8_OK) return st;
  if (sh != nullptr && (sh->Is <= 0 || sh->Is % 128 || 2 * sh->Is * H >= (int64_t(1) << 31)))
    return sh->Is <= 0 ? W8A8_ERR_ARG : W8A8_ERR_UNSUPPORTED;
  if (T == 0) return W8A8_OK;
  if (!x || !wg || !wgu || !s_gu || !wd || !s_d || !workspace || !y) return W8A8_ERR_ARG;
  if (sh != nullptr && (!sh->wsg || !sh->wgu || !sh->s_gu || !sh->wd || !sh->s_d)) return W8A8_ERR_ARG;
  if (!aligned16(x) || !aligned16(wg) || !aligned16(wgu) || !aligned16(wd) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return W8A8_ERR_UNSUPPORTED;
  if (sh != nullptr && (!aligned16(sh->wsg) || !aligned16(sh->wgu) || !aligned16(sh->wd))) return W8A8_ERR_UNSUPPORTED;
  w8a8_moe_shared_ws_layout SL;
  if (sh != nullptr) fill_shared_layout(T, H, E, k, I, sh->Is, &SL);
  else fill_layout(T, H, E, k, I, &SL.routed);
  const w8a8_moe_ws_layout& L = SL.routed;
  if (workspace_bytes < (sh != nullptr ? SL.total : L.total)) return W8A8_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* w = reinterpret_cast<float*>(ws + L.topk_w);
  int* offsets = reinterpret_cast<int*>(ws + L.offsets);
  int* perm = reinterpret_cast<int*>(ws + L.perm);
  float* sx_sorted = reinterpret_cast<float*>(ws + L.sx_sorted);
  int8_t* xq = reinterpret_cast<int8_t*>(ws + L.xq);
  uint16_t* h = reinterpret_cast<uint16_t*>(ws + L.h);
  float* s_h = reinterpret_cast<float*>(ws + L.s_h);
  int8_t* hq = reinterpret_cast<int8_t*>(ws + L.hq);
  uint16_t* o = reinterpret_cast<uint16_t*>(ws + L.o);
  cudaStream_t s = as_stream(stream);
  const int64_t A = T * k;
  int rc = route_group_stage(x, wg, bias, T, H, E, k, renorm, ws, L, s, ev);
  if (rc != W8A8_OK) return rc;
  ExpertRows b{xq, sx_sorted, offsets, h, s_h, hq, o, perm};
  if ((rc = experts_stage(b, A, E, E, H, I, wgu, s_gu, wd, s_d, s, ev)) != W8A8_OK) return rc;

  // 5b. the shared expert (every token): its bf16 gate, per-token int8 x, the dense gate_up GEMM
  //     with the SiLU*up epilogue, the requantisation of its h, the dense down GEMM
  uint16_t* o_sh = nullptr;
  float* gate = nullptr;
  if (sh != nullptr) {
    int8_t* sxq = reinterpret_cast<int8_t*>(ws + SL.xq);
    float* ssx = reinterpret_cast<float*>(ws + SL.sx);
    uint16_t* sh_h = reinterpret_cast<uint16_t*>(ws + SL.h);
    float* sh_sh = reinterpret_cast<float*>(ws + SL.s_h);
    int8_t* sh_hq = reinterpret_cast<int8_t*>(ws + SL.hq);
    o_sh = reinterpret_cast<uint16_t*>(ws + SL.o);
    gate = reinterpret_cast<float*>(ws + SL.gate);
    if ((rc = launch_pdl(shared_gate_kernel, dim3(unsigned((T + kRowWarps - 1) / kRowWarps)), dim3(kRowWarps * 32), 0,
                         s, x, sh->wsg, int(T), int(H), gate)) != W8A8_OK)
      return rc;
    if ((rc = launch_quant_rows(x, T, int(H), sxq, ssx, s)) != W8A8_OK) return rc;
    if ((rc = dense_gate_up(sxq, ssx, sh->wgu, sh->s_gu, T, H, sh->Is, sh_h, s)) != W8A8_OK) return rc;
    if ((rc = launch_quant_rows(sh_h, T, int(sh->Is), sh_hq, sh_sh, s)) != W8A8_OK) return rc;
    if ((rc = linear_gemm(sh_hq, sh_sh, sh->wd, sh->s_d, W8A8_W_INT8_PER_CHANNEL, T, sh->Is, H, o_sh, s)) != W8A8_OK)
      return rc;
  }

  // 6. scatter-free weighted combine (and the gated shared expert after the k slots)
  mark(ev, 5, s);
  rc = launch_pdl(combine_kernel, dim3(unsigned(T)), dim3(256), 0, s, o, w, int(T), int(H), k, y,
                  static_cast<const uint16_t*>(o_sh), static_cast<const float*>(gate));
  mark(ev, 6, s);
  return rc;
}

}  // namespace
}  // namespace w8a8

extern "C" {

int w8a8_moe_shared_workspace_layout(int64_t T, int64_t H, int64_t E, int k, int64_t I, int64_t Is,
                                     w8a8_moe_shared_ws_layout* layout) {
  if (!layout) return W8A8_ERR_ARG;
  const int st = check_moe_shape(T, H, E, k, I);
  if (st != W8A8_OK) return st;
  if (Is <= 0) return W8A8_ERR_ARG;
  if (Is % 128 || 2 * Is * H >= (int64_t(1) << 31)) return W8A8_ERR_UNSUPPORTED;
  fill_shared_layout(T, H, E, k, I, Is, layout);
  return W8A8_OK;
}

size_t w8a8_moe_shared_workspace_size(int64_t T, int64_t H, int64_t E, int k, int64_t I, int64_t Is) {
  w8a8_moe_shared_ws_layout L;
  return w8a8_moe_shared_workspace_layout(T, H, E, k, I, Is, &L) == W8A8_OK ? L.total : 0;
}

int w8a8_moe_forward_shared(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                            const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H, int64_t E,
                            int k, int64_t I, int renorm, const w8a8_bf16* wsg, const int8_t* wgu_s,
                            const float* s_gu_s, const int8_t* wd_s, const float* s_d_s, int64_t Is, void* workspace,
                            size_t workspace_bytes, w8a8_bf16* y, w8a8_stream stream) {
  const SharedExpert sh{wsg, wgu_s, s_gu_s, wd_s, s_d_s, Is};
  return moe_forward_impl(x, wg, bias, wgu, s_gu, wd, s_d, T, H, E, k, I, renorm, workspace, workspace_bytes, y,
                          stream, nullptr, &sh);
}

int w8a8_moe_forward(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                     const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H, int64_t E, int k,
                     int64_t I, int renorm, void* workspace, size_t workspace_bytes, w8a8_bf16* y,
                     w8a8_stream stream) {
  return moe_forward_impl(x, wg, bias, wgu, s_gu, wd, s_d, T, H, E, k, I, renorm, workspace, workspace_bytes, y,
                          stream, nullptr);
}

// ------------------------------------------------------------------ expert-parallel building blocks
int w8a8_moe_route_group(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, int64_t T, int64_t H, int64_t E,
                         int k, int renorm, void* workspace, size_t workspace_bytes, w8a8_stream stream) {
  const int st = check_moe_shape(T, H, E, k, 128);
  if (st != W8A8_OK) return st;
  if (T == 0) return W8A8_OK;
  if (!x || !wg || !workspace) return W8A8_ERR_ARG;
  if (!aligned16(x) || !aligned16(wg) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return W8A8_ERR_UNSUPPORTED;
  w8a8_moe_ws_layout L;
  fill_layout(T, H, E, k, 128, &L);
  if (workspace_bytes < L.total) return W8A8_ERR_WORKSPACE;  // the forward's layout with I = 128
  return route_group_stage(x, wg, bias, T, H, E, k, renorm, static_cast<uint8_t*>(workspace), L,
                           as_stream(stream), nullptr);
}

// Workspace of w8a8_moe_experts: the experts' row offsets and the row map (device copies of what
// the host builds), the rows and scales regrouped by expert, then h, s_h and hq.
struct ExpertsWs {
  size_t offsets, map, xq, sx, h, s_h, hq, total;
};

ExpertsWs experts_ws(int64_t A, int64_t H, int64_t I, int64_t Ew) {
  const size_t Ap = size_t(round_up(A > 0 ? A : 1, 128));
  ExpertsWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  w.offsets = take(sizeof(int) * size_t(Ew + 1));
  w.map = take(sizeof(int) * Ap);
  w.xq = take(Ap * size_t(H));
  w.sx = take(sizeof(float) * Ap);
  w.h = take(Ap * size_t(I) * 2);
  w.s_h = take(sizeof(float) * Ap);
  w.hq = take(Ap * size_t(I));
  w.total = off;
  return w;
}

size_t w8a8_moe_experts_workspace_size(int64_t A, int64_t H, int64_t I, int64_t Ew) {
  if (A < 0 || H <= 0 || I <= 0 || Ew <= 0 || H % 128 || I % 128 || Ew > 256) return 0;
  if (A >= (int64_t(1) << 30)) return 0;
  return experts_ws(A, H, I, Ew).total;
}

int w8a8_moe_experts(const int8_t* xq, const float* sx, const int* group_offsets_host, int64_t G,
                     int64_t weight_groups, int64_t A, int64_t H, int64_t I, int64_t Ew, const int8_t* wgu,
                     const float* s_gu, const int8_t* wd, const float* s_d, void* workspace, size_t workspace_bytes,
                     w8a8_bf16* o, w8a8_stream stream) {
  if (A < 0 || H <= 0 || I <= 0 || G <= 0 || Ew <= 0 || weight_groups < 0) return W8A8_ERR_ARG;
  const size_t need = w8a8_moe_experts_workspace_size(A, H, I, Ew);
  if (need == 0 || G > kMaxGroups || Ew * 2 * I >= (int64_t(1) << 31) || Ew * H >= (int64_t(1) << 31))
    return W8A8_ERR_UNSUPPORTED;
  if (weight_groups > Ew || (weight_groups == 0 && G > Ew)) return W8A8_ERR_ARG;
  if (!group_offsets_host) return W8A8_ERR_ARG;
  if (group_offsets_host[0] != 0 || group_offsets_host[G] != A) return W8A8_ERR_ARG;
  for (int64_t g = 0; g < G; ++g)
    if (group_offsets_host[g + 1] < group_offsets_host[g]) return W8A8_ERR_ARG;
  if (A == 0) return W8A8_OK;
  if (!xq || !sx || !wgu || !s_gu || !wd || !s_d || !workspace || !o) return W8A8_ERR_ARG;
  if (workspace_bytes < need) return W8A8_ERR_WORKSPACE;
  if (!aligned16(xq) || !aligned16(wgu) || !aligned16(wd) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return W8A8_ERR_UNSUPPORTED;
  // rows regrouped by expert: expert e takes the groups g with g % weight_groups == e (or g == e)
  // in increasing g; map[r] = the input row placed at regrouped row r, which is also where the
  // down GEMM writes that row's output
  std::vector<int> exp_off(static_cast<size_t>(Ew + 1), 0);
  std::vector<int> map(static_cast<size_t>(A), 0);
  int next = 0;
  for (int64_t e = 0; e < Ew; ++e) {
    exp_off[size_t(e)] = next;
    for (int64_t g = 0; g < G; ++g) {
      if ((weight_groups > 0 ? g % weight_groups : g) != e) continue;
      for (int i = group_offsets_host[g]; i < group_offsets_host[g + 1]; ++i) map[size_t(next++)] = i;
    }
  }
  exp_off[size_t(Ew)] = next;
  if (next != A) return W8A8_ERR_ARG;  // groups past Ew experts (weight_groups 0)
  const ExpertsWs L = experts_ws(A, H, I, Ew);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* d_off = reinterpret_cast<int*>(ws + L.offsets);
  int* d_map = reinterpret_cast<int*>(ws + L.map);
  int8_t* xq_g = reinterpret_cast<int8_t*>(ws + L.xq);
  float* sx_g = reinterpret_cast<float*>(ws + L.sx);
  cudaStream_t s = as_stream(stream);
  // pageable host sources: the copies have read them when the calls return
  if (cudaMemcpyAsync(d_off, exp_off.data(), sizeof(int) * exp_off.size(), cudaMemcpyHostToDevice, s) !=
          cudaSuccess ||
      cudaMemcpyAsync(d_map, map.data(), sizeof(int) * map.size(), cudaMemcpyHostToDevice, s) != cudaSuccess)
    return W8A8_ERR_LAUNCH;
  int rc = launch_pdl(gather_rows_kernel, dim3(unsigned((A + kRowWarps - 1) / kRowWarps)), dim3(kRowWarps * 32), 0,
                      s, reinterpret_cast<const uint8_t*>(xq), sx, static_cast<const int*>(d_map), A, int(H), A,
                      reinterpret_cast<uint8_t*>(xq_g), sx_g);
  if (rc != W8A8_OK) return rc;
  ExpertRows b{xq_g, sx_g, d_off, reinterpret_cast<uint16_t*>(ws + L.h), reinterpret_cast<float*>(ws + L.s_h),
               reinterpret_cast<int8_t*>(ws + L.hq), reinterpret_cast<uint16_t*>(o), d_map};
  return experts_stage(b, A, Ew, Ew, H, I, wgu, s_gu, wd, s_d, s, nullptr);
}

int w8a8_moe_combine_sorted(const w8a8_bf16* o_sorted, const int* perm, const float* topk_w, int64_t T, int64_t H,
                            int k, w8a8_bf16* o_slots, w8a8_bf16* y, w8a8_stream stream) {
  if (T < 0 || H <= 0 || k <= 0) return W8A8_ERR_ARG;
  if (H % 128 || k > kMaxTopK || T * k >= (int64_t(1) << 31) / 2) return W8A8_ERR_UNSUPPORTED;
  if (T == 0) return W8A8_OK;
  if (!o_sorted || !perm || !topk_w || !o_slots || !y) return W8A8_ERR_ARG;
  if (!aligned16(o_sorted) || !aligned16(o_slots) || !aligned16(y)) return W8A8_ERR_UNSUPPORTED;
  const int64_t A = T * k;
  cudaStream_t s = as_stream(stream);
  int rc = launch_pdl(scatter_rows_kernel, dim3(unsigned((A + kRowWarps - 1) / kRowWarps)), dim3(kRowWarps * 32), 0,
                      s, reinterpret_cast<const uint8_t*>(o_sorted), perm, A, int(H * 2),
                      reinterpret_cast<uint8_t*>(o_slots), A);
  if (rc != W8A8_OK) return rc;
  return launch_pdl(combine_kernel, dim3(unsigned(T)), dim3(256), 0, s, reinterpret_cast<const uint16_t*>(o_slots),
                    topk_w, int(T), int(H), k, reinterpret_cast<uint16_t*>(y), static_cast<const uint16_t*>(nullptr),
                    static_cast<const float*>(nullptr));
}

// ------------------------------------------------------------------ allocation-free variant
}  // extern "C"

namespace w8a8 {
namespace {

// Device scratch for w8a8_moe_forward_noalloc. It lives in the library's module, so every GPU
// that loads the library holds these bytes until the process exits. Host code must not pass
// the symbol itself to a kernel (on the host it only names a stand-in object); the device
// address comes from cudaGetSymbolAddress, fetched once per device below.
constexpr size_t kNoallocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoallocScratchBytes];

constexpr int kNoallocMaxDevices = 64;
std::mutex g_noalloc_mu;
struct NoallocSlot {
  void* ptr;      // device address of g_noalloc_scratch
  void* context;  // the CUDA context that address belongs to
};
NoallocSlot g_noalloc_slot[kNoallocMaxDevices] = {};

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

// The calling thread's current CUDA context (nullptr if none is bound yet or the query fails).
void* current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of g_noalloc_scratch on the current device. The address is looked up with
// cudaGetSymbolAddress, with that device current, the first time a device is used, and cached
// together with the context it was found in. If the current context differs later (the device
// was reset and the library's module loaded again, possibly at another address), it is looked
// up again. Returns W8A8_OK, W8A8_ERR_UNSUPPORTED for a device index the cache does not cover,
// or W8A8_ERR_LAUNCH if the runtime cannot give the address.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return W8A8_ERR_LAUNCH;
  if (dev < 0 || dev >= kNoallocMaxDevices) return W8A8_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc_slot[dev];
  void* ctx = current_context();
  if (slot.ptr == nullptr || ctx == nullptr || ctx != slot.context) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return W8A8_ERR_LAUNCH;
    slot.ptr = p;
    slot.context = current_context();  // bound by now: the lookup made the device's context current
  }
  *out = slot.ptr;
  return W8A8_OK;
}

}  // namespace
}  // namespace w8a8

extern "C" {

int w8a8_moe_forward_noalloc(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                             const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H,
                             int64_t E, int k, int64_t I, int renorm, w8a8_bf16* y, w8a8_stream stream) {
  const int st = check_moe_shape(T, H, E, k, I);
  if (st != W8A8_OK) return st;
  if (T == 0) return W8A8_OK;
  w8a8_moe_ws_layout L;
  fill_layout(T, H, E, k, I, &L);
  if (L.total > kNoallocScratchBytes) return W8A8_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int sst = noalloc_scratch(&scratch);
  if (sst != W8A8_OK) return sst;
  return moe_forward_impl(x, wg, bias, wgu, s_gu, wd, s_d, T, H, E, k, I, renorm, scratch, kNoallocScratchBytes, y,
                          stream, nullptr);
}

int w8a8_moe_forward_profiled(const w8a8_bf16* x, const w8a8_bf16* wg, const float* bias, const int8_t* wgu,
                              const float* s_gu, const int8_t* wd, const float* s_d, int64_t T, int64_t H,
                              int64_t E, int k, int64_t I, int renorm, void* workspace, size_t workspace_bytes,
                              w8a8_bf16* y, w8a8_stream stream, void* const* stage_events) {
  return moe_forward_impl(x, wg, bias, wgu, s_gu, wd, s_d, T, H, E, k, I, renorm, workspace, workspace_bytes, y,
                          stream, stage_events);
}

size_t w8a8_linear_workspace_size(int64_t M, int64_t K, int64_t N, int w_format, int group) {
  if (M < 0 || K <= 0 || N <= 0) return 0;
  if (K % 128 || N % 128) return 0;
  if (w_format == W8A8_W_INT4_PER_GROUP && group != 128) return 0;
  if (w_format != W8A8_W_INT8_PER_CHANNEL && w_format != W8A8_W_INT4_PER_GROUP) return 0;
  const int64_t Mp = round_up(M > 0 ? M : 1, 128);
  return align256(size_t(Mp) * K) + align256(sizeof(float) * Mp) + 256;
}

}  // extern "C"

namespace w8a8 {
namespace {

// The GEMM of the dense linear on already quantised activations: xq int8 [M, K] (rows past M
// are read as zeros), sx fp32 [M]. Arguments are checked by the callers.
int linear_gemm(const int8_t* xq, const float* sx, const void* wq, const float* sw, int w_format, int64_t M,
                int64_t K, int64_t N, w8a8_bf16* y, cudaStream_t s) {
  if (w_format == W8A8_W_INT4_PER_GROUP) {
    W4A8Params q{};
    if (!make_plain_map(&q.tmW, wq, uint64_t(K / 2), uint64_t(N), 64, 128) ||
        !make_plain_map(&q.tmY, y, uint64_t(N) * 2, uint64_t(M), 256, 128) ||
        !make_kmajor_map(&q.tmX, xq, false, K, M, kBBoxRows) || !make_kmajor_map(&q.tmX2, xq, false, K, M, 128))
      return W8A8_ERR_UNSUPPORTED;
    q.num_kb = int(K / 128);
    q.n_cb = int(N / 128);
    q.M = int(M);
    q.N = int(N);
    q.sw = sw;
    q.sw_vec = (K / 128) % 4 == 0 && aligned16(sw);
    q.sx = sx;
    q.timeout_ns = wait_timeout_ns();
    using Cfg = W4Cfg<128, 4, 8>;
    auto kern = w4a8_gemm_kernel<128, 4, 8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(Cfg::kSmemBytes)) != cudaSuccess)
      return W8A8_ERR_LAUNCH;
    const int tiles = int((M + 127) / 128) * q.n_cb;
    return launch_pdl(kern, dim3(max(1, min(num_sms(), tiles))), dim3(Cfg::kThreads), Cfg::kSmemBytes, s, q);
  }
  if (M > kPairMinRows) {
    PairParams q{};
    if (!make_kmajor_map(&q.tmA, wq, false, K, N, 128) || !make_pair_b_maps(&q, xq, K, M))
      return W8A8_ERR_UNSUPPORTED;
    q.num_kb = int(K / 128);
    q.n_cb = int((N + 255) / 256);
    q.n_channels = int(N);
    q.num_groups = 1;
    q.M = int(M);
    q.timeout_ns = wait_timeout_ns();
    q.out = y;
    q.ldo = int(N);
    q.row_scale = sx;
    q.col_scale = sw;
    return launch_pair<kEpiDense>(q, int((M + kPairNB - 1) / kPairNB) * q.n_cb, s);
  }
  GemmParams p{};
  if (!make_kmajor_map(&p.tmA, wq, false, K, N, 128) || !make_kmajor_map(&p.tmB, xq, false, K, M, kBBoxRows) ||
      !make_kmajor_map(&p.tmB2, xq, false, K, M, 128))
    return W8A8_ERR_UNSUPPORTED;
  p.num_kb = int(K / 128);
  p.n_cb = int((N + 255) / 256);
  p.n_channels = int(N);
  p.num_groups = 1;
  p.M = int(M);
  p.a_second_offset = 128;
  p.a_cb_step = 256;
  p.timeout_ns = wait_timeout_ns();
  p.out = y;
  p.ldo = int(N);
  p.row_scale = sx;
  p.col_scale = sw;
  const int tiles = int((M + 127) / 128) * p.n_cb;
  return launch_gemm<2, 128, kEpiDense, kKindI8>(p, tiles, s);
}

// Host-side checks shared by the two dense-linear entry points (everything but the activations).
int check_linear(const void* wq, const float* sw, int w_format, int group, int64_t M, int64_t K, int64_t N,
                 const w8a8_bf16* y) {
  if (M < 0 || K <= 0 || N <= 0) return W8A8_ERR_ARG;
  if (w8a8_linear_workspace_size(M, K, N, w_format, group) == 0) return W8A8_ERR_UNSUPPORTED;
  if (M == 0) return W8A8_OK;
  if (!wq || !sw || !y) return W8A8_ERR_ARG;
  if (!aligned16(wq) || !aligned16(y)) return W8A8_ERR_UNSUPPORTED;
  if (w_format == W8A8_W_INT4_PER_GROUP && (K / 128) > (int64_t(1) << 20)) return W8A8_ERR_UNSUPPORTED;
  if (M >= (int64_t(1) << 30) || N * K >= (int64_t(1) << 40)) return W8A8_ERR_UNSUPPORTED;
  return W8A8_OK;
}

}  // namespace
}  // namespace w8a8

extern "C" {

int w8a8_linear(const w8a8_bf16* x, const void* wq, const float* sw, int w_format, int group, int64_t M, int64_t K,
                int64_t N, void* workspace, size_t workspace_bytes, w8a8_bf16* y, w8a8_stream stream) {
  int rc = check_linear(wq, sw, w_format, group, M, K, N, y);
  if (rc != W8A8_OK || M == 0) return rc;
  const size_t need = w8a8_linear_workspace_size(M, K, N, w_format, group);
  if (!x || !workspace) return W8A8_ERR_ARG;
  if (workspace_bytes < need) return W8A8_ERR_WORKSPACE;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return W8A8_ERR_UNSUPPORTED;
  const int64_t Mp = round_up(M, 128);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int8_t* xq = reinterpret_cast<int8_t*>(ws);
  float* sx = reinterpret_cast<float*>(ws + align256(size_t(Mp) * K));
  rc = w8a8_quant_act_per_token(x, M, K, xq, sx, stream);
  if (rc != W8A8_OK) return rc;
  return linear_gemm(xq, sx, wq, sw, w_format, M, K, N, y, as_stream(stream));
}

int w8a8_linear_prequant(const int8_t* xq, const float* sx, const void* wq, const float* sw, int w_format,
                         int group, int64_t M, int64_t K, int64_t N, w8a8_bf16* y, w8a8_stream stream) {
  const int rc = check_linear(wq, sw, w_format, group, M, K, N, y);
  if (rc != W8A8_OK || M == 0) return rc;
  if (!xq || !sx) return W8A8_ERR_ARG;
  if (!aligned16(xq)) return W8A8_ERR_UNSUPPORTED;
  return linear_gemm(xq, sx, wq, sw, w_format, M, K, N, y, as_stream(stream));
}

int w8a8_gemm_s8s8s32(const int8_t* a, const int8_t* b, int32_t* c, int64_t M, int64_t N, int64_t K,
                      w8a8_stream stream) {
  if (M < 0 || N <= 0 || K <= 0) return W8A8_ERR_ARG;
  if (K % 128 || N % 128) return W8A8_ERR_UNSUPPORTED;
  if (M == 0) return W8A8_OK;
  if (!a || !b || !c) return W8A8_ERR_ARG;
  if (!aligned16(a) || !aligned16(b) || !aligned16(c) || M >= (int64_t(1) << 30)) return W8A8_ERR_UNSUPPORTED;
  // channels (rows of b) on the MMA M side, rows of a on N
  if (M > kPairMinRows) {
    PairParams q{};
    if (!make_kmajor_map(&q.tmA, b, false, K, N, 128) || !make_pair_b_maps(&q, a, K, M))
      return W8A8_ERR_UNSUPPORTED;
    q.num_kb = int(K / 128);
    q.n_cb = int((N + 255) / 256);
    q.n_channels = int(N);
    q.num_groups = 1;
    q.M = int(M);
    q.timeout_ns = wait_timeout_ns();
    q.out = c;
    q.ldo = int(N);
    return launch_pair<kEpiRawS32>(q, int((M + kPairNB - 1) / kPairNB) * q.n_cb, as_stream(stream));
  }
  GemmParams p{};
  if (!make_kmajor_map(&p.tmA, b, false, K, N, 128) || !make_kmajor_map(&p.tmB, a, false, K, M, kBBoxRows) ||
      !make_kmajor_map(&p.tmB2, a, false, K, M, 128))
    return W8A8_ERR_UNSUPPORTED;
  p.num_kb = int(K / 128);
  p.n_cb = int((N + 255) / 256);
  p.n_channels = int(N);
  p.num_groups = 1;
  p.M = int(M);
  p.a_second_offset = 128;
  p.a_cb_step = 256;
  p.timeout_ns = wait_timeout_ns();
  p.out = c;
  p.ldo = int(N);
  const int tiles = int((M + 127) / 128) * p.n_cb;
  return launch_gemm<2, 128, kEpiRawS32, kKindI8>(p, tiles, as_stream(stream));
}

int w8a8_debug_rcp_approx_ulp(uint32_t first_bits, uint32_t count, unsigned int* max_ulp, w8a8_stream stream) {
  if (!max_ulp || count == 0) return W8A8_ERR_ARG;
  const uint64_t last = uint64_t(first_bits) + count - 1;
  // positive normal inputs whose reciprocal is normal: [2^-126, 2^126)
  if (first_bits < 0x00800000u || last >= 0x7E800000u) return W8A8_ERR_ARG;
  if (cudaMemsetAsync(max_ulp, 0, sizeof(unsigned int), as_stream(stream)) != cudaSuccess) return W8A8_ERR_LAUNCH;
  const uint64_t want = (uint64_t(count) + 255) / 256;
  const unsigned blocks = unsigned(want < 4096 ? want : 4096);
  rcp_approx_ulp_kernel<<<blocks, 256, 0, as_stream(stream)>>>(first_bits, count, max_ulp);
  return launch_status();
}

int w8a8_debug_ex2_approx_ulp(uint32_t first_bits, uint32_t count, unsigned int* max_ulp, w8a8_stream stream) {
  if (!max_ulp || count == 0) return W8A8_ERR_ARG;
  const uint64_t first = first_bits, last = first + count - 1;
  // one sign only, and 2^x a normal number: |x| < 126
  if ((first >> 31) != (last >> 31) || (first & 0x7FFFFFFFu) >= 0x42FC0000u || (last & 0x7FFFFFFFu) >= 0x42FC0000u)
    return W8A8_ERR_ARG;
  if (cudaMemsetAsync(max_ulp, 0, sizeof(unsigned int), as_stream(stream)) != cudaSuccess) return W8A8_ERR_LAUNCH;
  const uint64_t want = (uint64_t(count) + 255) / 256;
  const unsigned blocks = unsigned(want < 4096 ? want : 4096);
  ex2_approx_ulp_kernel<<<blocks, 256, 0, as_stream(stream)>>>(first_bits, count, max_ulp);
  return launch_status();
}

int w8a8_mxfp8_quantize(const w8a8_bf16* x, int64_t R, int64_t K, uint8_t* codes, uint8_t* scales,
                        w8a8_stream stream) {
  if (R < 0 || K <= 0) return W8A8_ERR_ARG;
  if (K % kMxBlock || K > (int64_t(1) << 30) || R >= (int64_t(1) << 31)) return W8A8_ERR_UNSUPPORTED;
  if (R == 0) return W8A8_OK;
  if (!x || !codes || !scales) return W8A8_ERR_ARG;
  if (!aligned16(x) || (reinterpret_cast<uintptr_t>(codes) & 7u)) return W8A8_ERR_UNSUPPORTED;
  return launch_mx_rows(x, R, int(K), codes, scales, as_stream(stream));
}

size_t w8a8_mxfp8_linear_workspace_size(int64_t M, int64_t K, int64_t N) {
  if (M < 0 || K <= 0 || N <= 0 || K % 128 || N % 128) return 0;
  if (K > (int64_t(1) << 24) || N > (int64_t(1) << 24) || M >= (int64_t(1) << 30)) return 0;
  const size_t m = size_t(M > 0 ? M : 1);
  return align256(m * K) + align256(m * K / kMxBlock);
}

int w8a8_mxfp8_linear(const w8a8_bf16* x, const uint8_t* w_codes, const uint8_t* w_scales, int64_t M, int64_t K,
                      int64_t N, void* workspace, size_t workspace_bytes, w8a8_bf16* y, w8a8_stream stream) {
  if (M < 0 || K <= 0 || N <= 0) return W8A8_ERR_ARG;
  const size_t need = w8a8_mxfp8_linear_workspace_size(M, K, N);
  if (need == 0) return W8A8_ERR_UNSUPPORTED;
  if (M == 0) return W8A8_OK;
  if (!x || !w_codes || !w_scales || !y || !workspace) return W8A8_ERR_ARG;
  if (workspace_bytes < need) return W8A8_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(y) || !aligned16(w_codes) || (reinterpret_cast<uintptr_t>(w_scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return W8A8_ERR_UNSUPPORTED;
  uint8_t* xc = static_cast<uint8_t*>(workspace);
  uint8_t* xs = xc + align256(size_t(M) * K);
  const cudaStream_t s = as_stream(stream);
  const int rc = launch_mx_rows(x, M, int(K), xc, xs, s);
  if (rc != W8A8_OK) return rc;
  return mx_gemm<kMxE4M3>(xc, xs, w_codes, w_scales, M, K, N, y, s);
}

int w8a8_mxfp8_linear_prequant(const uint8_t* x_codes, const uint8_t* x_scales, const uint8_t* w_codes,
                               const uint8_t* w_scales, int64_t M, int64_t K, int64_t N, w8a8_bf16* y,
                               w8a8_stream stream) {
  if (M < 0 || K <= 0 || N <= 0) return W8A8_ERR_ARG;
  if (w8a8_mxfp8_linear_workspace_size(M, K, N) == 0) return W8A8_ERR_UNSUPPORTED;
  if (M == 0) return W8A8_OK;
  if (!x_codes || !x_scales || !w_codes || !w_scales || !y) return W8A8_ERR_ARG;
  if (!aligned16(x_codes) || !aligned16(w_codes) || !aligned16(y) || (reinterpret_cast<uintptr_t>(x_scales) & 3u) ||
      (reinterpret_cast<uintptr_t>(w_scales) & 3u))
    return W8A8_ERR_UNSUPPORTED;
  return mx_gemm<kMxE4M3>(x_codes, x_scales, w_codes, w_scales, M, K, N, y, as_stream(stream));
}

int w8a8_mxfp4_quantize(const w8a8_bf16* w, int64_t R, int64_t K, uint8_t* packed, uint8_t* scales,
                        w8a8_stream stream) {
  if (R < 0 || K <= 0) return W8A8_ERR_ARG;
  if (K % kMxBlock || K > (int64_t(1) << 30) || R >= (int64_t(1) << 31)) return W8A8_ERR_UNSUPPORTED;
  if (R == 0) return W8A8_OK;
  if (!w || !packed || !scales) return W8A8_ERR_ARG;
  if (!aligned16(w) || (reinterpret_cast<uintptr_t>(packed) & 3u)) return W8A8_ERR_UNSUPPORTED;
  return launch_mx4_rows(w, R, int(K), packed, scales, as_stream(stream));
}

int w8a8_mxfp_a8w4_linear(const w8a8_bf16* x, const uint8_t* w_packed, const uint8_t* w_scales, int64_t M,
                          int64_t K, int64_t N, void* workspace, size_t workspace_bytes, w8a8_bf16* y,
                          w8a8_stream stream) {
  if (M < 0 || K <= 0 || N <= 0) return W8A8_ERR_ARG;
  const size_t need = w8a8_mxfp8_linear_workspace_size(M, K, N);
  if (need == 0) return W8A8_ERR_UNSUPPORTED;
  if (M == 0) return W8A8_OK;
  if (!x || !w_packed || !w_scales || !y || !workspace) return W8A8_ERR_ARG;
  if (workspace_bytes < need) return W8A8_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(y) || (reinterpret_cast<uintptr_t>(w_packed) & 31u) ||
      (reinterpret_cast<uintptr_t>(w_scales) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return W8A8_ERR_UNSUPPORTED;
  uint8_t* xc = static_cast<uint8_t*>(workspace);
  uint8_t* xs = xc + align256(size_t(M) * K);
  const cudaStream_t s = as_stream(stream);
  const int rc = launch_mx_rows(x, M, int(K), xc, xs, s);
  if (rc != W8A8_OK) return rc;
  return mx_gemm<kMxE2M1>(xc, xs, w_packed, w_scales, M, K, N, y, s);
}

int w8a8_mxfp_a8w4_linear_prequant(const uint8_t* x_codes, const uint8_t* x_scales, const uint8_t* w_packed,
                                   const uint8_t* w_scales, int64_t M, int64_t K, int64_t N, w8a8_bf16* y,
                                   w8a8_stream stream) {
  if (M < 0 || K <= 0 || N <= 0) return W8A8_ERR_ARG;
  if (w8a8_mxfp8_linear_workspace_size(M, K, N) == 0) return W8A8_ERR_UNSUPPORTED;
  if (M == 0) return W8A8_OK;
  if (!x_codes || !x_scales || !w_packed || !w_scales || !y) return W8A8_ERR_ARG;
  if (!aligned16(x_codes) || (reinterpret_cast<uintptr_t>(w_packed) & 31u) || !aligned16(y) ||
      (reinterpret_cast<uintptr_t>(x_scales) & 3u) || (reinterpret_cast<uintptr_t>(w_scales) & 3u))
    return W8A8_ERR_UNSUPPORTED;
  return mx_gemm<kMxE2M1>(x_codes, x_scales, w_packed, w_scales, M, K, N, y, as_stream(stream));
}

int w8a8_debug_wait_timeout(uint64_t timeout_ns, w8a8_stream stream) {
  if (timeout_ns == 0 || timeout_ns > 10ull * 1000 * 1000 * 1000) return W8A8_ERR_ARG;
  wait_timeout_probe_kernel<<<1, 32, 0, as_stream(stream)>>>(timeout_ns);
  return launch_status();
}

}  // extern "C"
