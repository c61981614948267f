// Routing pieces shared by the tensor-core router epilogue and the small-batch router:
// the warp-per-token top-k selection, the CUDA-core logits kernel for short batches and the
// top-k kernel that consumes its output.
#pragma once
#include "numerics.cuh"

namespace w8a8 {

constexpr int kMaxTopK = 16;

// Top-k routing of one token by one warp. Lane l holds experts l, l+32, ..., as order-preserving
// integer keys of their logits (+ bias); each of the k rounds is two warp reductions: the
// largest key, then the lowest expert holding it (equal logits go to the lower expert), and
// the winner's lane drops that entry. Softmax over the picks (renorm) or over all E experts,
// in fp32; lanes 0..k-1 store ids[j], w[j] and add to counts[e] when counts is given.
// logit(e) returns the fp32 logit of expert e < PER * 32 (only called for e < E).
template <int PER, typename Logit>
__device__ __forceinline__ void warp_topk_token(Logit logit, int E, int k, bool renorm, const float* __restrict__ bias,
                                                int* ids, float* w, int* counts) {
  const int lane = threadIdx.x & 31;
  float lv[PER];
  uint32_t key[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    float l = 0.0f;
    if (e < E) {
      l = logit(e);
      if (bias != nullptr) l += __ldg(bias + e);
    }
    lv[i] = l;
    key[i] = (e < E) ? ordered_key(l) : 0u;  // 0: below every real logit, never picked
  }
  float pick_v = 0.0f, m = 0.0f;
  int pick_e = -1;
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    uint32_t lbest = 0;
    int li = 0;
#pragma unroll
    for (int i = PER - 1; i >= 0; --i)  // downward, so the lowest expert wins among equals
      if (key[i] >= lbest) { lbest = key[i]; li = i; }
    const uint32_t wbest = warp_max_u32(lbest);
    const uint32_t cand = (wbest != 0u && lbest == wbest) ? uint32_t(lane + 32 * li) : 0xFFFFFFFFu;
    const uint32_t ebest = warp_min_u32(cand);
    if (ebest != 0xFFFFFFFFu && int(ebest & 31u) == lane) {
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (i == int(ebest >> 5)) key[i] = 0u;
    }
    const float v = from_ordered_key(wbest);
    if (j == 0) m = v;
    if (lane == j) {
      pick_v = v;
      pick_e = (ebest == 0xFFFFFFFFu) ? -1 : int(ebest);
    }
  }
  const float ev = (lane < k && pick_e >= 0) ? expf(pick_v - m) : 0.0f;
  float denom = ev;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, o);
  if (!renorm) {
    float sall = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i)
      if (lane + 32 * i < E) sall += expf(lv[i] - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sall += __shfl_xor_sync(0xffffffffu, sall, o);
    denom = sall;
  }
  if (lane < k) {
    int e = pick_e;
    if (e < 0) {  // only non-finite logits can leave a slot unfilled; report, never index
      atomicOr(&g_error_word, kErrBadIndex);
      e = lane;
    }
    ids[lane] = e;
    w[lane] = ev / denom;
    if (counts != nullptr) atomicAdd(counts + e, 1);
  }
}

// The same selection for NT tokens at once by one warp: token u's steps are exactly those of
// warp_topk_token, and the NT tokens' warp reductions are independent, so they overlap instead
// of running one dependent chain after another. logit(u, e) for u < nt; token u's outputs at
// ids + u * ld_out, w + u * ld_out.
template <int PER, int NT, typename Logit>
__device__ __forceinline__ void warp_topk_tokens(Logit logit, int nt, int E, int k, bool renorm,
                                                 const float* __restrict__ bias, int* ids, float* w, int ld_out,
                                                 int* counts) {
  const int lane = threadIdx.x & 31;
  float lv[NT][PER];
  uint32_t key[NT][PER];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane + 32 * i;
      const bool valid = e < E && u < nt;
      float l = 0.0f;
      if (valid) {
        l = logit(u, e);
        if (bias != nullptr) l += __ldg(bias + e);
      }
      lv[u][i] = l;
      key[u][i] = valid ? ordered_key(l) : 0u;
    }
  }
  float pick_v[NT], m[NT];
  int pick_e[NT];
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    pick_v[u] = 0.0f;
    m[u] = 0.0f;
    pick_e[u] = -1;
  }
#pragma unroll 1
  for (int j = 0; j < k; ++j) {
    uint32_t lbest[NT], wbest[NT], ebest[NT];
    int li[NT];
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      lbest[u] = 0;
      li[u] = 0;
#pragma unroll
      for (int i = PER - 1; i >= 0; --i)
        if (key[u][i] >= lbest[u]) { lbest[u] = key[u][i]; li[u] = i; }
    }
#pragma unroll
    for (int u = 0; u < NT; ++u) wbest[u] = warp_max_u32(lbest[u]);
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      const uint32_t cand = (wbest[u] != 0u && lbest[u] == wbest[u]) ? uint32_t(lane + 32 * li[u]) : 0xFFFFFFFFu;
      ebest[u] = warp_min_u32(cand);
    }
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      if (ebest[u] != 0xFFFFFFFFu && int(ebest[u] & 31u) == lane) {
#pragma unroll
        for (int i = 0; i < PER; ++i)
          if (i == int(ebest[u] >> 5)) key[u][i] = 0u;
      }
      const float v = from_ordered_key(wbest[u]);
      if (j == 0) m[u] = v;
      if (lane == j) {
        pick_v[u] = v;
        pick_e[u] = (ebest[u] == 0xFFFFFFFFu) ? -1 : int(ebest[u]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < NT; ++u) {
    const float ev = (lane < k && pick_e[u] >= 0) ? expf(pick_v[u] - m[u]) : 0.0f;
    float denom = ev;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) denom += __shfl_xor_sync(0xffffffffu, denom, o);
    if (!renorm) {
      float sall = 0.0f;
#pragma unroll
      for (int i = 0; i < PER; ++i)
        if (lane + 32 * i < E) sall += expf(lv[u][i] - m[u]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sall += __shfl_xor_sync(0xffffffffu, sall, o);
      denom = sall;
    }
    if (u < nt && lane < k) {
      int e = pick_e[u];
      if (e < 0) {
        atomicOr(&g_error_word, kErrBadIndex);
        e = lane;
      }
      ids[u * ld_out + lane] = e;
      w[u * ld_out + lane] = ev / denom;
      if (counts != nullptr) atomicAdd(counts + e, 1);
    }
  }
}

// Router logits on the CUDA cores for short batches: logits[t, e] = sum_h x[t, h] * wg[e, h] in
// fp32 (bf16 inputs). A work item is 8 experts x kSmallRouterTokens tokens for 8 warps: warp w8
// takes expert eg * 8 + w8 and tokens tg * kSmallRouterTokens .. + kSmallRouterTokens - 1, with
// its 1/32 of the expert's row (H <= 256 * RU) in registers and one accumulator per token and
// vector slot. The item's token rows sit in shared memory (xs: [kSmallRouterTokens][H] bf16, rows
// past T zero), read from global memory once per item instead of once per warp. Two steps:
// router_item_weights loads the warp's expert row (issue it before staging the token rows, so
// that both loads are in flight together); router_logits_item_xs computes and stores the logits.
constexpr int kSmallRouterTokens = 4;

template <int RU>
__device__ __forceinline__ void router_item_weights(const uint16_t* __restrict__ wg, int H, int E, int eg, int w8,
                                                    uint4 (&wv)[RU]) {
  const int lane = threadIdx.x & 31;
  const int e = eg * 8 + w8;
#pragma unroll
  for (int u = 0; u < RU; ++u) {
    const int i = lane * 8 + u * 256;
    wv[u] = (i < H && e < E) ? __ldg(reinterpret_cast<const uint4*>(wg + size_t(e) * H + i)) : make_uint4(0, 0, 0, 0);
  }
}
template <int RU>
__device__ __forceinline__ void router_logits_item_xs(const uint16_t* __restrict__ xs, const uint4 (&wv)[RU], int T,
                                                      int H, int E, float* __restrict__ logits, int eg, int tg,
                                                      int w8) {
  constexpr int TT = kSmallRouterTokens;
  const int lane = threadIdx.x & 31;
  const int e = eg * 8 + w8;
  if (e >= E) return;
  const int t0 = tg * TT;
  float acc[TT];
#pragma unroll
  for (int t = 0; t < TT; ++t) {
    float part[RU];
#pragma unroll
    for (int u = 0; u < RU; ++u) {
      const int i = lane * 8 + u * 256;
      const uint4 xv = (i < H) ? *reinterpret_cast<const uint4*>(xs + t * H + i) : make_uint4(0, 0, 0, 0);
      const uint32_t a[4] = {xv.x, xv.y, xv.z, xv.w};
      const uint32_t b[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
      float s2 = 0.0f;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        s2 = fmaf(bf16_lo(a[j]), bf16_lo(b[j]), s2);
        s2 = fmaf(bf16_hi(a[j]), bf16_hi(b[j]), s2);
      }
      part[u] = s2;
    }
    float sum = 0.0f;
#pragma unroll
    for (int u = 0; u < RU; ++u) sum += part[u];
    acc[t] = sum;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
#pragma unroll
    for (int t = 0; t < TT; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
  if (lane < TT && t0 + lane < T) {
    float v = acc[0];
#pragma unroll
    for (int t = 1; t < TT; ++t) v = (lane == t) ? acc[t] : v;
    logits[size_t(t0 + lane) * E + e] = v;
  }
}

// The item's token rows into shared memory by the 256 threads of one item (thread index it),
// zero rows past T.
__device__ __forceinline__ void stage_router_rows(const uint16_t* __restrict__ x, int T, int H, int tg, int it,
                                                  uint16_t* xs) {
  const int t0 = tg * kSmallRouterTokens;
  const int vec_per_row = H / 8;
  for (int v = it; v < kSmallRouterTokens * vec_per_row; v += 256) {
    const int t = v / vec_per_row, i = (v - t * vec_per_row) * 8;
    *reinterpret_cast<uint4*>(xs + t * H + i) =
        (t0 + t < T) ? __ldg(reinterpret_cast<const uint4*>(x + size_t(t0 + t) * H + i)) : make_uint4(0, 0, 0, 0);
  }
}

template <int RU>
__global__ void __launch_bounds__(256) router_logits_small_kernel(const uint16_t* __restrict__ x,
                                                                  const uint16_t* __restrict__ wg, int T, int H,
                                                                  int E, float* __restrict__ logits) {
  extern __shared__ __align__(16) uint16_t xs_dyn[];  // [kSmallRouterTokens][H]
  pdl_wait();
  pdl_launch_dependents();
  uint4 wv[RU];
  router_item_weights<RU>(wg, H, E, blockIdx.x, threadIdx.x >> 5, wv);
  stage_router_rows(x, T, H, blockIdx.y, threadIdx.x, xs_dyn);
  __syncthreads();
  router_logits_item_xs<RU>(xs_dyn, wv, T, H, E, logits, blockIdx.x, blockIdx.y, threadIdx.x >> 5);
}

// Top-k over precomputed logits [T, E]: one warp per token. counts has one row of E per
// 128-token chunk (count_stride = E) or a single row (count_stride = 0).
template <int PER>
__global__ void __launch_bounds__(256) router_topk_kernel(const float* __restrict__ logits, const float* bias, int T,
                                                          int E, int k, int renorm, int* ids, float* w, int* counts,
                                                          int count_stride) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + size_t(t) * E;
  int* crow = counts != nullptr ? counts + size_t(t / 128) * count_stride : nullptr;
  warp_topk_token<PER>([&](int e) { return __ldg(row + e); }, E, k, renorm != 0, bias, ids + size_t(t) * k,
                       w + size_t(t) * k, crow);
}

}  // namespace w8a8
