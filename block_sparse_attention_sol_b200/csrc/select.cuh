// Block selection ("preparation" of the sparse attention, which the Sol-H3
// runtime made 76.4% faster: ai-feiten.nl, "Videomodel MiniMax-H3 rendert
// sneller dan afspelen", section "Waar de snelheidswinst vandaan komt").
//
//   pool:   qbar[b,h,i,:] = mean of q[b,n,h,:] over the valid tokens n of block i
//           (same for k).  HBM-bound: one CTA per (b, block, tensor) streams the
//           block's rows (all heads, contiguous) with 16-byte loads.
//   score:  s[b,h,i,j] = qbar[b,h,i,:] . kbar[b,h,j,:]  in fp32 (register-tiled
//           SIMT; a tensor-core score would round the scores and move the top-k
//           boundary).
//   top-k:  per row, the k largest scores, exact ties to the lower j, written in
//           ascending j.  A warp finds the k-th largest order-preserving key by a
//           most-significant-bit-first search of the 32-bit key space, then
//           compacts the winners in ascending j with ballots.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace sol {
namespace select {

// ------------------------------------------------------------------ pooling
template <typename T> struct PoolVec;
template <> struct PoolVec<float> { static constexpr int n = 4; };
template <> struct PoolVec<__nv_bfloat16> { static constexpr int n = 8; };

__device__ __forceinline__ void acc_vec(const float* p, float (&a)[4]) {
  const float4 v = __ldcs(reinterpret_cast<const float4*>(p));
  a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
}
__device__ __forceinline__ void acc_vec(const __nv_bfloat16* p, float (&a)[8]) {
  const uint4 v = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a[2 * i] += __uint_as_float(w[i] << 16);
    a[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// grid (nb, B, 2): blockIdx.z = 0 pools q, 1 pools k.  out: [B, H, nb, D] fp32.
template <typename T>
__global__ void __launch_bounds__(256) block_pool_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                         float* __restrict__ qbar, float* __restrict__ kbar, int N,
                                                         int H, int D, int block, int nb) {
  constexpr int V = PoolVec<T>::n;
  const int i = blockIdx.x, b = blockIdx.y;
  const T* src = blockIdx.z == 0 ? q : k;
  float* dst = blockIdx.z == 0 ? qbar : kbar;
  const int HD = H * D;
  const int n0 = i * block;
  const int cnt = min(block, N - n0);
  const float inv = 1.0f / static_cast<float>(cnt);
  for (int c = threadIdx.x; c < HD / V; c += blockDim.x) {
    float a[V];
#pragma unroll
    for (int e = 0; e < V; ++e) a[e] = 0.f;
    const T* base = src + (static_cast<size_t>(b) * N + n0) * HD + c * V;
    int n = 0;
    for (; n + 8 <= cnt; n += 8) {
#pragma unroll
      for (int u = 0; u < 8; ++u) acc_vec(base + static_cast<size_t>(n + u) * HD, a);
    }
    for (; n < cnt; ++n) acc_vec(base + static_cast<size_t>(n) * HD, a);
    const int h = (c * V) / D, d0 = (c * V) % D;
    float* o = dst + ((static_cast<size_t>(b) * H + h) * nb + i) * D + d0;
#pragma unroll
    for (int e = 0; e < V; e += 4) *reinterpret_cast<float4*>(o + e) = make_float4(a[e] * inv, a[e + 1] * inv, a[e + 2] * inv, a[e + 3] * inv);
  }
}

// ------------------------------------------------------------------ scores + top-k
constexpr int kRows = 16;        // query blocks per CTA
constexpr int kKeys = 64;        // key blocks per shared-memory chunk
constexpr int kThreads = 256;

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0 so equal scores get equal keys
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Dynamic shared memory: qs[kRows][D+4] | ks[kKeys][D+4] | sc[kRows][nb]
// grid (ceil(nb / kRows), B * H).
template <int D>
__global__ void __launch_bounds__(kThreads) score_topk_kernel(const float* __restrict__ qbar,
                                                              const float* __restrict__ kbar,
                                                              int32_t* __restrict__ idx, float* __restrict__ scores_out,
                                                              int nb, int topk) {
  extern __shared__ float smem[];
  constexpr int P = D + 4;
  float* qs = smem;
  float* ks = qs + kRows * P;
  float* sc = ks + kKeys * P;
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * kRows;
  const int nrows = min(kRows, nb - r0);
  const float* qb = qbar + static_cast<size_t>(bh) * nb * D;
  const float* kb = kbar + static_cast<size_t>(bh) * nb * D;

  for (int e = threadIdx.x; e < kRows * (D / 4); e += kThreads) {
    const int r = e / (D / 4), d = (e % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nrows) v = *reinterpret_cast<const float4*>(qb + static_cast<size_t>(r0 + r) * D + d);
    *reinterpret_cast<float4*>(qs + r * P + d) = v;
  }
  // thread -> (4 rows, 1 key) of a 16 x 64 chunk
  const int kj = threadIdx.x % kKeys;
  const int rg = (threadIdx.x / kKeys) * 4;
  for (int j0 = 0; j0 < nb; j0 += kKeys) {
    __syncthreads();
    for (int e = threadIdx.x; e < kKeys * (D / 4); e += kThreads) {
      const int j = e / (D / 4), d = (e % (D / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (j0 + j < nb) v = *reinterpret_cast<const float4*>(kb + static_cast<size_t>(j0 + j) * D + d);
      *reinterpret_cast<float4*>(ks + j * P + d) = v;
    }
    __syncthreads();
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
    for (int d = 0; d < D; d += 4) {
      const float4 kv = *reinterpret_cast<const float4*>(ks + kj * P + d);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 qv = *reinterpret_cast<const float4*>(qs + (rg + r) * P + d);
        acc[r] = fmaf(qv.x, kv.x, acc[r]);
        acc[r] = fmaf(qv.y, kv.y, acc[r]);
        acc[r] = fmaf(qv.z, kv.z, acc[r]);
        acc[r] = fmaf(qv.w, kv.w, acc[r]);
      }
    }
    if (j0 + kj < nb) {
#pragma unroll
      for (int r = 0; r < 4; ++r) sc[(rg + r) * nb + j0 + kj] = acc[r];
    }
  }
  __syncthreads();

  if (scores_out != nullptr) {
    for (int e = threadIdx.x; e < nrows * nb; e += kThreads) {
      const int r = e / nb, j = e % nb;
      scores_out[(static_cast<size_t>(bh) * nb + r0 + r) * nb + j] = sc[r * nb + j];
    }
  }

  __syncthreads();   // the dump above reads rows the key conversion below rewrites

  // top-k: one warp per row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int r = warp; r < nrows; r += kThreads / 32) {
    uint32_t* keys = reinterpret_cast<uint32_t*>(sc + r * nb);
    for (int j = lane; j < nb; j += 32) keys[j] = order_key(sc[r * nb + j]);
    __syncwarp();
    // largest T with count(key >= T) >= topk, i.e. the k-th largest key
    uint32_t prefix = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = prefix | (1u << bit);
      int cnt = 0;
      for (int j = lane; j < nb; j += 32) cnt += keys[j] >= cand ? 1 : 0;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
      if (cnt >= topk) prefix = cand;
    }
    int gt = 0;
    for (int j = lane; j < nb; j += 32) gt += keys[j] > prefix ? 1 : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) gt += __shfl_xor_sync(0xffffffffu, gt, off);
    const int need_eq = topk - gt;
    int32_t* out = idx + (static_cast<size_t>(bh) * nb + r0 + r) * topk;
    int written = 0, eq_seen = 0;
    for (int j0 = 0; j0 < nb; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t key = j < nb ? keys[j] : 0u;
      const bool is_gt = j < nb && key > prefix;
      const bool is_eq = j < nb && key == prefix;
      const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
      const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
      const bool sel = is_gt || (is_eq && eq_rank < need_eq);
      const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
      if (sel) out[written + __popc(sel_mask & lt_mask)] = j;
      written += __popc(sel_mask);
      eq_seen += __popc(eq_mask);
    }
  }
}

}  // namespace select
}  // namespace sol
