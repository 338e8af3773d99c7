// Block-sparse attention forward in fp32 on the CUDA cores.
//
// Same definition as the tensor-core kernel (exact softmax over the keys of
// the kept blocks, returning O and the natural-log LSE), for fp32 inputs where
// a relative error near 1e-5 is required: tf32 tensor cores cannot reach that.
// One warp owns one query row; each lane holds D/32 channels of q and of the
// running output, so a logit is a lane-partial dot product reduced with
// shuffles.  Online softmax with exact expf, fp32 throughout.
#pragma once
#include <cstdint>
#include "blocks.cuh"
#include "sm100_ptx.cuh"

namespace sol {
namespace attnf32 {

constexpr int kWarps = 8;   // query rows per CTA

template <int D>
__global__ void __launch_bounds__(kWarps * 32) sparse_attn_fwd_f32_kernel(
    const float* __restrict__ q, const float* __restrict__ k, const float* __restrict__ v,
    const int32_t* __restrict__ idx, const int32_t* __restrict__ counts, float* __restrict__ o,
    float* __restrict__ lse, int B, int N, int H, const BlockMap bm, int nb, int topk, float scale) {
  constexpr int C = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * kWarps + warp;   // over B * H * N
  if (row >= static_cast<long long>(B) * H * N) return;
  const int n = static_cast<int>(row % N);
  const int h = static_cast<int>((row / N) % H);
  const int b = static_cast<int>(row / (static_cast<long long>(N) * H));
  const size_t rs = static_cast<size_t>(H) * D;   // token stride
  const float* qp = q + (static_cast<size_t>(b) * N + n) * rs + h * D;
  float qr[C], acc[C];
#pragma unroll
  for (int c = 0; c < C; ++c) { qr[c] = qp[lane + 32 * c] * scale; acc[c] = 0.f; }
  const size_t rowi = static_cast<size_t>(b * H + h) * nb + token_block(bm, n);   // row of idx / counts
  const int32_t* list = idx + rowi * topk;
  const int kt = counts == nullptr ? topk : min(max(counts[rowi], 1), topk);
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < kt; ++j) {
    const int blk = list[j];
    if (static_cast<unsigned>(blk) >= static_cast<unsigned>(nb)) {   // unusable id: skipped, reported
      if (lane == 0) raise_bad_arg();
      continue;
    }
    const int len = bm.tw == 0 ? min(bm.block, N - blk * bm.block) : bm.block;
    for (int u = 0; u < len; ++u) {
      const int mk = block_token(bm, blk, u);
      const float* kp = k + (static_cast<size_t>(b) * N + mk) * rs + h * D;
      float part = 0.f;
#pragma unroll
      for (int c = 0; c < C; ++c) part = fmaf(qr[c], kp[lane + 32 * c], part);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      const float m_new = fmaxf(m, part);
      const float alpha = expf(m - m_new);
      const float pexp = expf(part - m_new);
      l = l * alpha + pexp;
      const float* vp = v + (static_cast<size_t>(b) * N + mk) * rs + h * D;
#pragma unroll
      for (int c = 0; c < C; ++c) acc[c] = fmaf(pexp, vp[lane + 32 * c], acc[c] * alpha);
      m = m_new;
    }
  }
  float* op = o + (static_cast<size_t>(b) * N + n) * rs + h * D;
  const float inv = 1.0f / l;
#pragma unroll
  for (int c = 0; c < C; ++c) op[lane + 32 * c] = acc[c] * inv;
  if (lane == 0) lse[(static_cast<size_t>(b) * H + h) * N + n] = m + logf(l);
}

}  // namespace attnf32
}  // namespace sol
