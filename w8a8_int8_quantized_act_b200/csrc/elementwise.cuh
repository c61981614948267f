// Memory-bound kernels of the path: per-row symmetric quantisation (activations per token,
// weights per output channel, h per assignment row), the int4 per-group weight packer, the
// grouping of assignments by expert fused with the activation quantisation, and the
// scatter-free weighted combine. All use 16-byte vector loads and one warp per row.
#pragma once
#include "numerics.cuh"

namespace w8a8 {

constexpr int kRowWarps = 8;  // warps per CTA for one-warp-per-row kernels

// q[r, :] = codes of src[r, :], scale[r] = amax / 127, for rows r < R (row length K).
template <int U>
__global__ void __launch_bounds__(kRowWarps * 32) quant_rows_kernel(const uint16_t* __restrict__ src,
                                                                    int64_t R, int K, int8_t* __restrict__ q,
                                                                    float* __restrict__ scale) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t r = int64_t(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (r >= R) return;
  int8_t* dst = q + r * K;
  const float s = quant_row_warp<U>(src + r * K, K, [&](int i, uint2 v) {
    *reinterpret_cast<uint2*>(dst + i) = v;
  });
  if ((threadIdx.x & 31) == 0) scale[r] = s;
}

// The same quantisation (U > 0) with a grid of resident CTAs: each warp walks rows r, r + stride,
// ... and loads its next row while it quantises the current one, so every warp keeps a row's
// loads in flight instead of waiting for them once per row.
template <int U>
__device__ __forceinline__ void load_row8(const uint16_t* __restrict__ src, int64_t R, int K, int64_t r, int lane,
                                          uint4 (&v)[U]) {
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int i = lane * 8 + u * 256;
    v[u] = (r < R && i < K) ? __ldg(reinterpret_cast<const uint4*>(src + r * K + i)) : make_uint4(0, 0, 0, 0);
  }
}

template <int U>
__global__ void __launch_bounds__(kRowWarps * 32) quant_rows_stream_kernel(const uint16_t* __restrict__ src,
                                                                           int64_t R, int K, int8_t* __restrict__ q,
                                                                           float* __restrict__ scale) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t stride = int64_t(gridDim.x) * kRowWarps;
  int64_t r = int64_t(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  uint4 cur[U], nxt[U];
  load_row8<U>(src, R, K, r, lane, cur);
  for (; r < R; r += stride) {
    load_row8<U>(src, R, K, r + stride, lane, nxt);
    float amax = 0.0f;
#pragma unroll
    for (int u = 0; u < U; ++u) amax = fmaxf(amax, amax8(cur[u]));
    amax = warp_max(amax);
    const float s = sym_scale(amax, kQMaxInt8);
    const float inv = __frcp_rn(s);
    int8_t* dst = q + r * K;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = lane * 8 + u * 256;
      if (i < K) *reinterpret_cast<uint2*>(dst + i) = quant8(cur[u], s, inv);
    }
    if (lane == 0) scale[r] = s;
#pragma unroll
    for (int u = 0; u < U; ++u) cur[u] = nxt[u];
  }
}

// Symmetric int4 per group of 128 along K: one warp per (row, group), 4 values per lane.
// Byte i of a row holds code 2i (low nibble) and code 2i+1 (high nibble).
__global__ void __launch_bounds__(kRowWarps * 32) quant_int4_group128_kernel(
    const uint16_t* __restrict__ w, int64_t N, int K, uint8_t* __restrict__ packed, float* __restrict__ scale) {
  const int groups = K / 128;
  const int64_t item = int64_t(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (item >= N * groups) return;
  const int64_t n = item / groups;
  const int g = int(item - n * groups);
  const int lane = threadIdx.x & 31;
  const uint2 v = __ldg(reinterpret_cast<const uint2*>(w + n * K + g * 128 + lane * 4));
  const float f[4] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y)};
  float amax = fmaxf(fmaxf(fabsf(f[0]), fabsf(f[1])), fmaxf(fabsf(f[2]), fabsf(f[3])));
  amax = warp_max(amax);
  const float s = sym_scale(amax, kQMaxInt4);
  uint32_t nib[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) nib[j] = uint32_t(sym_code(f[j], s, 7)) & 0xFu;
  const uint16_t bytes = uint16_t((nib[0] | (nib[1] << 4)) | ((nib[2] | (nib[3] << 4)) << 8));
  *reinterpret_cast<uint16_t*>(packed + n * (K / 2) + g * 64 + lane * 2) = bytes;
  if (lane == 0) scale[n * groups + g] = s;
}

// Groups the T*k assignments by expert (stable by token) and quantises each token once,
// writing its codes to every sorted row that it feeds.
//   tile_counts [C, E]: assignments per (128-token chunk, expert) (from the router)
//   offsets [E+1], perm [A] (sorted row -> t*k + j), sx [T], sx_sorted [A], xq_sorted [A, H]
// Grid (chunk, split): the CTAs of one 128-token chunk each derive the chunk's write positions
// (only split 0 stores perm/offsets) and quantise every split-th token. Inside a chunk, the
// rank of assignment (t, e) among the chunk's rows of expert e is the number of earlier tokens
// of the chunk that chose e: a popcount over a 128-bit token mask per expert.
constexpr int kPermThreads = 256;
constexpr int kChunk = 128;

template <int U>
__global__ void __launch_bounds__(kPermThreads) group_quant_kernel(
    const uint16_t* __restrict__ x, const int* __restrict__ ids, const int* __restrict__ tile_counts, int T,
    int H, int E, int k, int* __restrict__ offsets, int* __restrict__ perm, float* __restrict__ sx,
    float* __restrict__ sx_sorted, int8_t* __restrict__ xq_sorted) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ int sm[];
  int* base = sm;                                   // [E]  first sorted row of the chunk's rows of e
  int* before = sm + E;                             // [E]  rows of e in earlier chunks
  int* dest = sm + 2 * E;                           // [kChunk * k]
  int* cid = dest + kChunk * k;                     // [kChunk * k] the chunk's expert ids
  uint32_t* mask = reinterpret_cast<uint32_t*>(cid + kChunk * k);  // [E][4] token masks
  const int C = (T + kChunk - 1) / kChunk;
  const int A = T * k;
  const int chunk = blockIdx.x;
  const int split = blockIdx.y, nsplit = gridDim.y;
  const int t0 = chunk * kChunk;
  const int nt = min(kChunk, T - t0);
  const int na = nt * k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // per-expert totals and this chunk's prefix over earlier chunks; the chunk's ids; clear masks
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int total = 0, prior = 0;
    for (int c = 0; c < C; ++c) {
      const int v = __ldg(tile_counts + size_t(c) * E + e);
      total += v;
      if (c < chunk) prior += v;
    }
    base[e] = total;  // temporarily: totals
    before[e] = prior;
  }
  for (int i = threadIdx.x; i < 4 * E; i += blockDim.x) mask[i] = 0u;
  for (int i = threadIdx.x; i < kChunk * k; i += blockDim.x) {
    dest[i] = -1;
    int e = (i < na) ? __ldg(ids + size_t(t0) * k + i) : -1;
    if (i < na && (e < 0 || e >= E)) {
      if (split == 0) atomicOr(&g_error_word, kErrBadIndex);
      e = -1;  // an invalid id gets no row
    }
    cid[i] = e;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of totals over experts (one warp)
    int carry = 0;
    for (int e0 = 0; e0 < E; e0 += 32) {
      const int e = e0 + lane;
      const int v = (e < E) ? base[e] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (e < E) {
        const int excl = carry + incl - v;
        if (chunk == 0 && split == 0) offsets[e] = excl;
        base[e] = excl + before[e];
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (chunk == 0 && split == 0 && lane == 0) offsets[E] = carry;
  } else {
    for (int i = threadIdx.x - 32; i < na; i += blockDim.x - 32) {
      const int e = cid[i];
      const int tl = i / k;
      if (e >= 0) atomicOr(mask + 4 * e + (tl >> 5), 1u << (tl & 31));
    }
  }
  __syncthreads();
  // every assignment's sorted row, in parallel
  for (int i = threadIdx.x; i < na; i += blockDim.x) {
    const int e = cid[i];
    if (e < 0) continue;
    const int tl = i / k;
    const uint32_t* mk = mask + 4 * e;
    int rank = __popc(mk[tl >> 5] & ((1u << (tl & 31)) - 1u));
    for (int w = 0; w < (tl >> 5); ++w) rank += __popc(mk[w]);
    const int d = base[e] + rank;
    if (d >= 0 && d < A) {
      if (split == 0) perm[d] = t0 * k + i;
      dest[i] = d;
    } else if (split == 0) {
      atomicOr(&g_error_word, kErrBadIndex);  // ids inconsistent with the per-chunk counts
    }
  }
  __syncthreads();
  // quantise each token once, write its codes to its k sorted rows
  for (int tl = split + nsplit * warp; tl < nt; tl += nsplit * (kPermThreads / 32)) {
    const int t = t0 + tl;
    const int* drow = dest + tl * k;
    const float s = quant_row_warp<U>(x + size_t(t) * H, H, [&](int i, uint2 v) {
      for (int j = 0; j < k; ++j)
        if (drow[j] >= 0) *reinterpret_cast<uint2*>(xq_sorted + size_t(drow[j]) * H + i) = v;
    });
    if (lane == 0) sx[t] = s;
    for (int j = lane; j < k; j += 32)
      if (drow[j] >= 0) sx_sorted[drow[j]] = s;
  }
}

// dst[map[r], :] = src[r, :] for r < R, rows of `row_bytes` bytes (a multiple of 16, both buffers
// 16-byte aligned): one warp per row. A map value outside [0, dst_rows) sets the bad-index bit of
// the device error word and the row is skipped.
__global__ void __launch_bounds__(kRowWarps * 32) scatter_rows_kernel(const uint8_t* __restrict__ src,
                                                                      const int* __restrict__ map, int64_t R,
                                                                      int row_bytes, uint8_t* __restrict__ dst,
                                                                      int64_t dst_rows) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t r = int64_t(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (r >= R) return;
  const int d = __ldg(map + r);
  if (d < 0 || d >= dst_rows) {
    if ((threadIdx.x & 31) == 0) atomicOr(&g_error_word, kErrBadIndex);
    return;
  }
  const uint4* s4 = reinterpret_cast<const uint4*>(src + r * row_bytes);
  uint4* d4 = reinterpret_cast<uint4*>(dst + int64_t(d) * row_bytes);
  for (int i = threadIdx.x & 31; i < row_bytes / 16; i += 32) d4[i] = __ldg(s4 + i);
}

// dst[r, :] = src[map[r], :] for r < R, rows of `row_bytes` bytes (a multiple of 16, both buffers
// 16-byte aligned), and dst_s[r] = src_s[map[r]] (one fp32 per row): one warp per row. A map
// value outside [0, src_rows) sets the bad-index bit of the device error word and the row is left.
__global__ void __launch_bounds__(kRowWarps * 32) gather_rows_kernel(const uint8_t* __restrict__ src,
                                                                     const float* __restrict__ src_s,
                                                                     const int* __restrict__ map, int64_t R,
                                                                     int row_bytes, int64_t src_rows,
                                                                     uint8_t* __restrict__ dst,
                                                                     float* __restrict__ dst_s) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t r = int64_t(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (r >= R) return;
  const int m = __ldg(map + r);
  if (m < 0 || m >= src_rows) {
    if ((threadIdx.x & 31) == 0) atomicOr(&g_error_word, kErrBadIndex);
    return;
  }
  const uint4* s4 = reinterpret_cast<const uint4*>(src + int64_t(m) * row_bytes);
  uint4* d4 = reinterpret_cast<uint4*>(dst + r * row_bytes);
  for (int i = threadIdx.x & 31; i < row_bytes / 16; i += 32) d4[i] = __ldg(s4 + i);
  if ((threadIdx.x & 31) == 0) dst_s[r] = __ldg(src_s + m);
}

// y[t, :] = bf16(sum_j w[t, j] * o[t, j, :]): fp32 fused multiply-adds in slot order from 0.
// With a shared expert (o_shared != nullptr) one more fused multiply-add follows the k slots:
// acc = fma(g[t], o_shared[t, :], acc).
// One CTA per token, 8 columns per thread, no atomics: every y element has one writer.
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ o, const float* __restrict__ w,
                                                      int T, int H, int k, uint16_t* __restrict__ y,
                                                      const uint16_t* __restrict__ o_shared,
                                                      const float* __restrict__ g) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = blockIdx.x;
  if (t >= T) return;
  for (int c = threadIdx.x * 8; c < H; c += blockDim.x * 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j = 0; j < k; ++j) {
      const float wj = __ldg(w + size_t(t) * k + j);
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(o + (size_t(t) * k + j) * H + c));
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fmaf_rn(wj, bf16_lo(u[i]), acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(wj, bf16_hi(u[i]), acc[2 * i + 1]);
      }
    }
    if (o_shared != nullptr) {
      const float gt = __ldg(g + t);
      const uint4 v = __ldg(reinterpret_cast<const uint4*>(o_shared + size_t(t) * H + c));
      const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] = __fmaf_rn(gt, bf16_lo(u[i]), acc[2 * i]);
        acc[2 * i + 1] = __fmaf_rn(gt, bf16_hi(u[i]), acc[2 * i + 1]);
      }
    }
    uint4 out;
    out.x = pack_bf16(acc[0], acc[1]);
    out.y = pack_bf16(acc[2], acc[3]);
    out.z = pack_bf16(acc[4], acc[5]);
    out.w = pack_bf16(acc[6], acc[7]);
    *reinterpret_cast<uint4*>(y + size_t(t) * H + c) = out;
  }
}

// Gate of the shared expert (bf16 shared_expert_gate, never quantised): g[t] = sigmoid(z),
// z = sum_h x[t, h] * w_sg[h] in fp32 (bf16 inputs; each lane fma-accumulates its 8-value vectors,
// then a warp butterfly sum), sigmoid(z) = 1 / (1 + exp(-z)) with the layer's exponential and a
// true divide. One warp per token; H a multiple of 8.
__global__ void __launch_bounds__(kRowWarps * 32) shared_gate_kernel(const uint16_t* __restrict__ x,
                                                                     const uint16_t* __restrict__ wsg, int T, int H,
                                                                     float* __restrict__ g) {
  pdl_wait();
  pdl_launch_dependents();
  const int t = int(blockIdx.x) * kRowWarps + (threadIdx.x >> 5);
  if (t >= T) return;
  const int lane = threadIdx.x & 31;
  float z = 0.0f;
  for (int i = lane * 8; i < H; i += 256) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(x + size_t(t) * H + i));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(wsg + i));
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      z = __fmaf_rn(bf16_lo(av[j]), bf16_lo(bv[j]), z);
      z = __fmaf_rn(bf16_hi(av[j]), bf16_hi(bv[j]), z);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z = __fadd_rn(z, __shfl_xor_sync(0xffffffffu, z, o));
  if (lane == 0) g[t] = __fdiv_rn(1.0f, __fadd_rn(1.0f, exp_cw(-z)));
}

// Largest distance, in units in the last place, between rcp.approx.ftz.f32(d) and the correctly
// rounded reciprocal of d, over the fp32 bit patterns first .. first + count - 1 (positive normal
// d with a normal reciprocal). The certified SiLU evaluation assumes this is at most 2.
__global__ void rcp_approx_ulp_kernel(uint32_t first, uint32_t count, unsigned int* max_ulp) {
  unsigned int worst = 0;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x) {
    const float d = __uint_as_float(first + i);
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    const int diff = int(__float_as_uint(r)) - int(__float_as_uint(__frcp_rn(d)));
    worst = max(worst, unsigned(diff < 0 ? -diff : diff));
  }
  worst = warp_max_u32(worst);
  if ((threadIdx.x & 31) == 0) atomicMax(max_ulp, worst);
}

// Largest distance, in units in the last place, between ex2.approx.ftz.f32(x) and 2^x computed
// in double and rounded to fp32, over the fp32 bit patterns first .. first + count - 1 (finite x
// whose 2^x is a normal fp32). The certified SiLU evaluation assumes this is at most 3.
__global__ void ex2_approx_ulp_kernel(uint32_t first, uint32_t count, unsigned int* max_ulp) {
  unsigned int worst = 0;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x) {
    const float x = __uint_as_float(first + i);
    float a;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(a) : "f"(x));
    const float ref = __double2float_rn(exp2(double(x)));
    const int diff = int(__float_as_uint(a)) - int(__float_as_uint(ref));
    worst = max(worst, unsigned(diff < 0 ? -diff : diff));
  }
  worst = warp_max_u32(worst);
  if ((threadIdx.x & 31) == 0) atomicMax(max_ulp, worst);
}

// Host-visible probe of the bounded-wait machinery: waits on an mbarrier phase that nothing
// completes, so the wait must run out after `timeout_ns` and raise the error word.
__global__ void wait_timeout_probe_kernel(uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const WaitCtx wc{&abort_flag, timeout_ns};
    mbar_wait(&bar, 0, wc);
  }
}

}  // namespace w8a8
