// Backward pass of the block-sparse attention (CUDA cores, fp32 arithmetic).
//
// Sol-Attn is used for inference (ai-feiten.nl, "Videomodel MiniMax-H3 rendert
// sneller dan afspelen", section "Waar de snelheidswinst vandaan komt"); the
// gradients are provided for completeness.  With P the softmax of
// scale * q k^T over the kept keys (recomputed from the forward's LSE),
//     delta_n = do_n . o_n
//     dS_nm   = P_nm (do_n . v_m - delta_n)
//     dq_n    = scale * sum_m dS_nm k_m
//     dk_m    = scale * sum_n dS_nm q_n,     dv_m = sum_n P_nm do_n
// where the sums over n run over the queries of every query block that kept
// m's block.  Kernels:
//   bwd_delta_kernel   one warp per (b, h, n): delta.
//   bwd_dq_kernel      one warp per query row over its kept keys.
//   bwd_invert_kernel  one thread per (b, h, key block j): the query blocks
//                      that kept j, in ascending order (deterministic, no atomics).
//   bwd_dkdv_kernel    one warp per key row over the queries of those blocks.
// Each lane holds D / 32 channels; dot products are warp reductions.  Blocks are
// runs of `block` consecutive tokens (the last may be short).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "sm100_ptx.cuh"

namespace sol {
namespace attnbwd {

constexpr int kWarps = 8;   // rows per CTA

__device__ __forceinline__ float ld(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

struct Shape {
  int B, N, H, block, nb, topk;
};

__device__ __forceinline__ int row_count(const int32_t* counts, size_t rowi, int topk) {
  return counts == nullptr ? topk : min(max(__ldg(counts + rowi), 1), topk);
}

// delta [B, H, N] = do . o
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_delta_kernel(const T* __restrict__ o, const T* __restrict__ dout,
                                                                float* __restrict__ delta, Shape s) {
  constexpr int C = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);   // over B * H * N
  if (row >= static_cast<long long>(s.B) * s.H * s.N) return;
  const int n = static_cast<int>(row % s.N);
  const int h = static_cast<int>((row / s.N) % s.H);
  const int b = static_cast<int>(row / (static_cast<long long>(s.N) * s.H));
  const size_t off = ((static_cast<size_t>(b) * s.N + n) * s.H + h) * D;
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < C; ++c) acc = fmaf(ld(dout + off + lane + 32 * c), ld(o + off + lane + 32 * c), acc);
  acc = warp_sum(acc);
  if (lane == 0) delta[row] = acc;
}

// dq [B, N, H, D] fp32: one warp per query row.
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                             const T* __restrict__ v, const T* __restrict__ dout,
                                                             const float* __restrict__ lse,
                                                             const float* __restrict__ delta,
                                                             const int32_t* __restrict__ idx,
                                                             const int32_t* __restrict__ counts, float* __restrict__ dq,
                                                             Shape s, float scale) {
  constexpr int C = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);   // over B * H * N
  if (row >= static_cast<long long>(s.B) * s.H * s.N) return;
  const int n = static_cast<int>(row % s.N);
  const int h = static_cast<int>((row / s.N) % s.H);
  const int b = static_cast<int>(row / (static_cast<long long>(s.N) * s.H));
  const size_t rs = static_cast<size_t>(s.H) * D;
  const size_t qoff = (static_cast<size_t>(b) * s.N + n) * rs + h * D;
  float qr[C], dor[C], acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) {
    qr[c] = ld(q + qoff + lane + 32 * c);
    dor[c] = ld(dout + qoff + lane + 32 * c);
    acc[c] = 0.f;
  }
  const float l = lse[row], dl = delta[row];
  const size_t rowi = static_cast<size_t>(b * s.H + h) * s.nb + n / s.block;
  const int32_t* list = idx + rowi * s.topk;
  const int kt = row_count(counts, rowi, s.topk);
  for (int j = 0; j < kt; ++j) {
    const int blk = __ldg(list + j);
    if (static_cast<unsigned>(blk) >= static_cast<unsigned>(s.nb)) {   // unusable id: skipped, reported
      if (lane == 0) raise_bad_arg();
      continue;
    }
    const int m0 = blk * s.block, m1 = min(s.N, m0 + s.block);
    for (int m = m0; m < m1; ++m) {
      const size_t koff = (static_cast<size_t>(b) * s.N + m) * rs + h * D;
      float sd = 0.f, pd = 0.f;
#pragma unroll
      for (int c = 0; c < C; ++c) {
        sd = fmaf(qr[c], ld(k + koff + lane + 32 * c), sd);
        pd = fmaf(dor[c], ld(v + koff + lane + 32 * c), pd);
      }
      sd = warp_sum(sd);
      pd = warp_sum(pd);
      const float p = expf(scale * sd - l);
      const float ds = p * (pd - dl) * scale;
#pragma unroll
      for (int c = 0; c < C; ++c) acc[c] = fmaf(ds, ld(k + koff + lane + 32 * c), acc[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < C; ++c) dq[qoff + lane + 32 * c] = acc[c];
}

// inv [B, H, nb, nb]: for key block j, the query blocks i that kept it, ascending; inv_cnt [B, H, nb].
__global__ void __launch_bounds__(256) bwd_invert_kernel(const int32_t* __restrict__ idx,
                                                         const int32_t* __restrict__ counts, int32_t* __restrict__ inv,
                                                         int32_t* __restrict__ inv_cnt, Shape s) {
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;   // over B * H * nb
  if (t >= static_cast<long long>(s.B) * s.H * s.nb) return;
  const int j = static_cast<int>(t % s.nb);
  const long long bh = t / s.nb;
  // Every entry of every row is read, so that an id outside [0, nb) or an id a
  // row repeats (which this index cannot represent) is reported, once, by the
  // thread of key block 0 or of the repeated block.
  int c = 0;
  bool bad = false;
  for (int i = 0; i < s.nb; ++i) {
    const size_t rowi = static_cast<size_t>(bh) * s.nb + i;
    const int32_t* list = idx + rowi * s.topk;
    const int kt = row_count(counts, rowi, s.topk);
    int hits = 0;
    for (int e = 0; e < kt; ++e) {
      const int id = __ldg(list + e);
      hits += id == j ? 1 : 0;
      bad |= j == 0 && static_cast<unsigned>(id) >= static_cast<unsigned>(s.nb);
    }
    if (hits > 0) inv[static_cast<size_t>(t) * s.nb + c++] = i;
    bad |= hits > 1;
  }
  inv_cnt[t] = c;
  if (bad) raise_bad_arg();
}

// dk, dv [B, N, H, D] fp32: one warp per key row.
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) bwd_dkdv_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                               const T* __restrict__ v, const T* __restrict__ dout,
                                                               const float* __restrict__ lse,
                                                               const float* __restrict__ delta,
                                                               const int32_t* __restrict__ inv,
                                                               const int32_t* __restrict__ inv_cnt,
                                                               float* __restrict__ dk, float* __restrict__ dv, Shape s,
                                                               float scale) {
  constexpr int C = D / 32;
  const int lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + (threadIdx.x >> 5);   // over B * H * N
  if (row >= static_cast<long long>(s.B) * s.H * s.N) return;
  const int m = static_cast<int>(row % s.N);
  const int h = static_cast<int>((row / s.N) % s.H);
  const int b = static_cast<int>(row / (static_cast<long long>(s.N) * s.H));
  const size_t rs = static_cast<size_t>(s.H) * D;
  const size_t koff = (static_cast<size_t>(b) * s.N + m) * rs + h * D;
  float kr[C], vr[C], ak[C], av[C];
#pragma unroll
  for (int c = 0; c < C; ++c) {
    kr[c] = ld(k + koff + lane + 32 * c);
    vr[c] = ld(v + koff + lane + 32 * c);
    ak[c] = 0.f;
    av[c] = 0.f;
  }
  const size_t ti = static_cast<size_t>(b * s.H + h) * s.nb + m / s.block;
  const int cnt = __ldg(inv_cnt + ti);
  const float* lse_bh = lse + static_cast<size_t>(b * s.H + h) * s.N;
  const float* delta_bh = delta + static_cast<size_t>(b * s.H + h) * s.N;
  for (int e = 0; e < cnt; ++e) {
    const int i = __ldg(inv + ti * s.nb + e);
    const int n0 = i * s.block, n1 = min(s.N, n0 + s.block);
    for (int n = n0; n < n1; ++n) {
      const size_t qoff = (static_cast<size_t>(b) * s.N + n) * rs + h * D;
      float sd = 0.f, pd = 0.f;
#pragma unroll
      for (int c = 0; c < C; ++c) {
        sd = fmaf(ld(q + qoff + lane + 32 * c), kr[c], sd);
        pd = fmaf(ld(dout + qoff + lane + 32 * c), vr[c], pd);
      }
      sd = warp_sum(sd);
      pd = warp_sum(pd);
      const float p = expf(scale * sd - __ldg(lse_bh + n));
      const float ds = p * (pd - __ldg(delta_bh + n)) * scale;
#pragma unroll
      for (int c = 0; c < C; ++c) {
        av[c] = fmaf(p, ld(dout + qoff + lane + 32 * c), av[c]);
        ak[c] = fmaf(ds, ld(q + qoff + lane + 32 * c), ak[c]);
      }
    }
  }
#pragma unroll
  for (int c = 0; c < C; ++c) {
    dk[koff + lane + 32 * c] = ak[c];
    dv[koff + lane + 32 * c] = av[c];
  }
}

}  // namespace attnbwd
}  // namespace sol
