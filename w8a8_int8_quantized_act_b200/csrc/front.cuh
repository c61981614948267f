// Front end of the MoE forward for short batches (at most one 128-token chunk, the decode
// case): router logits, softmax / top-k, the stable grouping of the T*k assignments by expert
// and the per-token activation quantisation into the sorted rows, in one cooperative launch
// instead of three latency-bound ones:
//   phase 1  logits [T, E] in fp32: the short-batch router's work items, two per CTA at a time
//            (each half of the CTA stages its item's token rows in shared memory once);
//   barrier
//   phase 2  top-k of token t by one warp (warp t / G of CTA t % G); ids and weights to the
//            workspace;
//   barrier
//   phase 3  every CTA reads the T*k expert ids and builds the counting sort by expert (stable
//            by token) in shared memory; CTA 0 stores offsets, perm and the expert histogram;
//   phase 4  token t is quantised by CTA t (all its warps; the row maximum through shared
//            memory) and its codes written to its k sorted rows.
// Both barriers are bounded: a CTA that waits too long raises the error word and returns. The
// arithmetic is that of the short-batch router, warp_topk_token and the symmetric quantiser (a
// maximum does not depend on the order it is taken in), so the results are those of the
// separate kernels bit for bit.
#pragma once
#include "elementwise.cuh"
#include "routing.cuh"

namespace w8a8 {

constexpr int kFrontMaxT = 128;
constexpr int kFrontMaxH = 2048;  // token row length the front end takes (its phase-1 staging)
constexpr int kFrontThreads = 512;
constexpr int kFrontWarps = kFrontThreads / 32;

// Arrival number `round` (1, 2, ...) of every CTA on *count (zeroed before the launch): waits
// until all `nctas` CTAs have arrived `round` times. Needs every CTA resident at once (a
// cooperative launch). Bounded: a CTA that has waited longer than `timeout_ns` raises the error
// word and returns false.
__device__ __forceinline__ bool grid_barrier(unsigned* count, unsigned nctas, unsigned round, uint64_t timeout_ns,
                                             int* ok_smem) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(count, 1u);
    const uint64_t deadline = globaltimer_ns() + timeout_ns;
    int ok = 1;
    while (true) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(count) : "memory");
      if (v >= nctas * round) break;
      if (globaltimer_ns() > deadline) {
        atomicOr(&g_error_word, kErrWaitTimeout);
        ok = 0;
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
    *ok_smem = ok;
  }
  __syncthreads();
  return *ok_smem != 0;
}

template <int RU, int PER>
__global__ void __launch_bounds__(kFrontThreads) front_small_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ wg, const float* __restrict__ bias, int T, int H,
    int E, int k, int renorm, float* __restrict__ logits, unsigned* sync_count, uint64_t timeout_ns,
    int* __restrict__ ids, float* __restrict__ w, int* __restrict__ tile_counts, int* __restrict__ offsets,
    int* __restrict__ perm, float* __restrict__ sx, float* __restrict__ sx_sorted, int8_t* __restrict__ xq) {
  __shared__ int dest[kFrontMaxT * kMaxTopK];   // sorted row of assignment t*k + j
  __shared__ int cnt[256], base[256];
  __shared__ uint32_t mask[256 * 4];            // per expert: which tokens chose it
  __shared__ float red[kFrontWarps];
  __shared__ int ok_smem;
  __shared__ __align__(16) uint16_t xrows[2][kSmallRouterTokens * kFrontMaxH];  // phase 1, per half

  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x;

  // phase 1: logits; the two halves of the CTA take one work item each (a half syncs on its
  // own named barrier, 1 or 2: the halves may run different numbers of items)
  const int neg = (E + 7) / 8, ntg = (T + kSmallRouterTokens - 1) / kSmallRouterTokens;
  const int hf = warp >> 3;
  for (int item = 2 * blockIdx.x + hf; item < neg * ntg; item += 2 * G) {
    const int tg = item / neg;
    uint4 wv[RU];
    router_item_weights<RU>(wg, H, E, item - tg * neg, warp & 7, wv);
    stage_router_rows(x, T, H, tg, threadIdx.x & 255, xrows[hf]);
    asm volatile("bar.sync %0, 256;" ::"r"(1 + hf) : "memory");
    router_logits_item_xs<RU>(xrows[hf], wv, T, H, E, logits, item - tg * neg, tg, warp & 7);
    asm volatile("bar.sync %0, 256;" ::"r"(1 + hf) : "memory");  // the rows are rewritten by the next item
  }
  if (!grid_barrier(sync_count, unsigned(G), 1u, timeout_ns, &ok_smem)) return;

  // phase 2: top-k, one warp per token, spread over the CTAs first (token t on warp t / G of
  // CTA t % G), so that no SM sub-partition interleaves several tokens' selections (logits
  // written by other CTAs: read through L2)
  for (int t = warp * G + blockIdx.x; t < T; t += G * kFrontWarps) {
    const float* row = logits + size_t(t) * E;
    warp_topk_token<PER>([&](int e) { return __ldcg(row + e); }, E, k, renorm != 0, bias, ids + size_t(t) * k,
                         w + size_t(t) * k, nullptr);
  }
  if (!grid_barrier(sync_count, unsigned(G), 2u, timeout_ns, &ok_smem)) return;

  // phase 3: counting sort by expert, stable by token, in every CTA
  for (int i = threadIdx.x; i < 4 * E; i += kFrontThreads) mask[i] = 0u;
  for (int i = threadIdx.x; i < E; i += kFrontThreads) cnt[i] = 0;
  __syncthreads();
  const int A = T * k;
  for (int i = threadIdx.x; i < A; i += kFrontThreads) {
    const int e = __ldcg(ids + i), t = i / k;
    dest[i] = e;
    atomicOr(mask + 4 * e + (t >> 5), 1u << (t & 31));
    atomicAdd(cnt + e, 1);
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the expert counts
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int v = (e < E) ? cnt[e] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (e < E) base[e] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < A; i += kFrontThreads) {
    const int e = dest[i], t = i / k;
    const uint32_t* mk = mask + 4 * e;
    int rank = __popc(mk[t >> 5] & ((1u << (t & 31)) - 1u));
    for (int q = 0; q < (t >> 5); ++q) rank += __popc(mk[q]);
    const int d = base[e] + rank;
    dest[i] = d;
    if (blockIdx.x == 0) perm[d] = i;
  }
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e < E; e += kFrontThreads) {
      offsets[e] = base[e];
      tile_counts[e] = cnt[e];
    }
    if (threadIdx.x == 0) offsets[E] = A;
  }
  __syncthreads();

  // phase 4: token t by CTA t; thread i holds the 8-value vectors i, i + 512, ... of the row
  constexpr int kVec = (RU * 256 + kFrontThreads * 8 - 1) / (kFrontThreads * 8);
  for (int t = blockIdx.x; t < T; t += G) {
    const uint16_t* src = x + size_t(t) * H;
    uint4 v[kVec];
    float amax = 0.0f;
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int i = (threadIdx.x + u * kFrontThreads) * 8;
      v[u] = (i < H) ? __ldg(reinterpret_cast<const uint4*>(src + i)) : make_uint4(0, 0, 0, 0);
      amax = fmaxf(amax, amax8(v[u]));
    }
    amax = warp_max(amax);
    if (lane == 0) red[warp] = amax;
    __syncthreads();
    amax = red[0];
#pragma unroll
    for (int i = 1; i < kFrontWarps; ++i) amax = fmaxf(amax, red[i]);
    const float s = sym_scale(amax, kQMaxInt8);
    const float inv = __frcp_rn(s);
    const int* drow = dest + t * k;
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      const int i = (threadIdx.x + u * kFrontThreads) * 8;
      if (i < H) {
        const uint2 q = quant8(v[u], s, inv);
        for (int j = 0; j < k; ++j) *reinterpret_cast<uint2*>(xq + size_t(drow[j]) * H + i) = q;
      }
    }
    if (threadIdx.x == 0) sx[t] = s;
    if (threadIdx.x < k) sx_sorted[drow[threadIdx.x]] = s;
    __syncthreads();  // red[] is reused by the CTA's next token
  }
}

}  // namespace w8a8
