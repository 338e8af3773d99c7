// Quantised exchange buffers for sequence-parallel Sol-Attn.
//
// Multi-GPU runs of the Sol-H3 runtime move Q, K and V between GPUs as INT8 and
// the attention output as FP8, halving the inter-GPU bytes (ai-feiten.nl,
// "Videomodel MiniMax-H3 rendert sneller dan afspelen", section "Waar de
// snelheidswinst vandaan komt").  Here a row is the D channels of one
// (batch, token, head); each row gets one fp32 scale s = max|x| / L
// (L = 127 for INT8, 448 for e4m3) and codes x * (L / max|x|) rounded to
// nearest even (INT8 clamped to +-127, e4m3 saturating), all decided in fp32:
// one division per row, one product per value (a division per value made the
// kernel issue-bound on the XU pipe).
//
//   quant_pack:     bf16 rows [B, N, H, D] -> codes + scales packed by
//                   destination rank g: [G][B][Nc][Hc][D] and [G][B][Nc][Hc].
//                   Split heads (token shard -> head shards): Hc = H / G,
//                   Nc = N, g = h / Hc.  Split tokens (head shard -> token
//                   shards): Nc = N / G, Hc = H, g = n / Nc.
//   dequant_unpack: codes + scales [G][B][Nc][Hc] received from G ranks ->
//                   bf16 bf16_rn(code * s), concatenated along tokens (the
//                   slices were head shards of token shards) or along heads.
// Both are HBM streams: D / 8 lanes per row, 16-byte bf16 loads / stores and
// 8-byte code stores / loads, one CTA per token (pack) or received row group
// (unpack) so that the index arithmetic is a few 32-bit operations per CTA.  Slice g starts g * g_stride rows into the
// buffers, so several tensors can share one exchange buffer.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>

namespace sol {
namespace quant {

enum : int { kSplitHeads = 0, kSplitTokens = 1 };
enum : int { kInt8 = 0, kE4M3 = 1 };

__device__ __forceinline__ void bf16x8_to_f32(const uint4 w, float (&v)[8]) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(u[i] << 16);
    v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

// Codes of 8 values q (already multiplied by the reciprocal scale), low byte first.
template <int CODE>
__device__ __forceinline__ uint2 encode8(const float (&q)[8]) {
  uint32_t w[2];
  if constexpr (CODE == kInt8) {
    // q + 1.5 * 2^23 rounds q to an integer (nearest even) in the sum's low mantissa
    // bits, exactly for |q| < 2^22; its low byte is the two's complement code.
    uint32_t b[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = __float_as_uint(fminf(fmaxf(q[e], -127.0f), 127.0f) + 12582912.0f);
    w[0] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
    w[1] = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
  } else {
    uint32_t p[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      p[i] = __nv_cvt_float2_to_fp8x2(make_float2(q[2 * i], q[2 * i + 1]), __NV_SATFINITE, __NV_E4M3);
    w[0] = p[0] | (p[1] << 16);
    w[1] = p[2] | (p[3] << 16);
  }
  return make_uint2(w[0], w[1]);
}

// Two codes (low byte first) of a 16-bit word as fp32, exactly.
template <int CODE>
__device__ __forceinline__ float2 decode2(uint32_t w16) {
  if constexpr (CODE == kInt8) {
    // 2^23 + (c + 128) is exact in fp32: subtract 2^23 + 128 (no conversion instruction)
    const uint32_t u = w16 ^ 0x8080u;
    return make_float2(__uint_as_float(0x4B000000u | (u & 0xFFu)) - 8388736.0f,
                       __uint_as_float(0x4B000000u | ((u >> 8) & 0xFFu)) - 8388736.0f);
  } else {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w16), __NV_E4M3);
    return __half22float2(__half2(h));
  }
}

// One row's share (8 channels) of the pack: scale from the L-lane group's max,
// codes from the reciprocal scale.
template <int L, int CODE>
__device__ __forceinline__ void pack_row(const float (&v)[8], unsigned seg, uint8_t* code_dst, float* scale_dst,
                                         bool write_scale) {
  const float levels = CODE == kInt8 ? 127.0f : 448.0f;
  float a = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[e]));
#pragma unroll
  for (int o = L / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(seg, a, o));
  const float s = __fdiv_rn(a, levels);
  const float rcp = __fdiv_rn(levels, a > 0.f ? a : 1.0f);
  float q[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) q[e] = s > 0.f ? __fmul_rn(v[e], rcp) : 0.f;
  __stcs(reinterpret_cast<uint2*>(code_dst), encode8<CODE>(q));
  if (write_scale) *scale_dst = s;
}

// CTA c handles tokens (b, n) = c, c + gridDim, ... of x; thread t handles
// channels 8 (t % L) .. +7 (L = D / 8 lanes per row) of heads h = t / L + k S,
// S = blockDim / L, two heads per pass with both loads issued first.  Index
// arithmetic is 32-bit and per token: B * N * H < 2^31 (checked on the host).
template <int D, int CODE>
__global__ void __launch_bounds__(512) quant_pack_kernel(const __nv_bfloat16* __restrict__ x,
                                                         uint8_t* __restrict__ codes, float* __restrict__ scales,
                                                         int B, int N, int H, int G, int split, long long g_stride) {
  constexpr int L = D / 8;
  const int li = threadIdx.x % L;
  const int S = blockDim.x / L;
  const unsigned lane = threadIdx.x & 31u;
  const unsigned seg = (L == 32) ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~static_cast<unsigned>(L - 1)));
  const int Nc = split == kSplitHeads ? N : N / G;
  const int Hc = split == kSplitHeads ? H / G : H;
  for (int tok = blockIdx.x; tok < B * N; tok += gridDim.x) {   // tok = b * N + n
    const int b = tok / N, n = tok - b * N;
    const int g_tok = split == kSplitHeads ? 0 : n / Nc;          // split tokens: one destination per token
    const int nc = n - g_tok * Nc;
    const __nv_bfloat16* src = x + static_cast<long long>(tok) * H * D + li * 8;
    for (int h = threadIdx.x / L; h < H; h += 2 * S) {
      const int h2 = h + S;
      const bool two = h2 < H;
      const uint4 r1 = __ldcs(reinterpret_cast<const uint4*>(src + static_cast<long long>(h) * D));
      const uint4 r2 = two ? __ldcs(reinterpret_cast<const uint4*>(src + static_cast<long long>(h2) * D)) : r1;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u == 1 && !two) break;
        const int hh = u ? h2 : h;
        float v[8];
        bf16x8_to_f32(u ? r2 : r1, v);
        int g = g_tok, hc = hh;
        if (split == kSplitHeads) { g = hh / Hc; hc = hh - g * Hc; }
        const long long drow = g * g_stride + (static_cast<long long>(b) * Nc + nc) * Hc + hc;
        pack_row<L, CODE>(v, seg, codes + drow * D + li * 8, scales + drow, li == 0);
      }
    }
  }
}

// CTA c handles received row groups (g, b, nc) = c, c + gridDim, ...; thread t
// handles channels 8 (t % L) .. +7 of heads hc = t / L + k S, two per pass.
template <int D, int CODE>
__global__ void __launch_bounds__(512) dequant_unpack_kernel(const uint8_t* __restrict__ codes,
                                                             const float* __restrict__ scales,
                                                             __nv_bfloat16* __restrict__ out, int B, int Nc, int Hc,
                                                             int G, int split, long long g_stride) {
  constexpr int L = D / 8;
  const int li = threadIdx.x % L;
  const int S = blockDim.x / L;
  for (int blk = blockIdx.x; blk < G * B * Nc; blk += gridDim.x) {   // blk = (g * B + b) * Nc + nc
    const int gb = blk / Nc, nc = blk - gb * Nc;
    const int g = gb / B, b = gb - g * B;
    const long long rbase = g * g_stride + (static_cast<long long>(b) * Nc + nc) * Hc;
    long long obase;   // output row of hc = 0
    if (split == kSplitHeads) obase = (static_cast<long long>(b) * G * Nc + static_cast<long long>(g) * Nc + nc) * Hc;
    else obase = (static_cast<long long>(b) * Nc + nc) * (static_cast<long long>(G) * Hc) + static_cast<long long>(g) * Hc;
    for (int hc = threadIdx.x / L; hc < Hc; hc += 2 * S) {
      const int hc2 = hc + S;
      const bool two = hc2 < Hc;
      const uint2 c1 = __ldcs(reinterpret_cast<const uint2*>(codes + (rbase + hc) * D + li * 8));
      const uint2 c2 = two ? __ldcs(reinterpret_cast<const uint2*>(codes + (rbase + hc2) * D + li * 8)) : c1;
      const float s1 = __ldg(scales + rbase + hc);
      const float s2 = two ? __ldg(scales + rbase + hc2) : s1;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u == 1 && !two) break;
        const uint2 c = u ? c2 : c1;
        const float s = u ? s2 : s1;
        const uint32_t cw[2] = {c.x, c.y};
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = decode2<CODE>((cw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
          const __nv_bfloat162 p = __floats2bfloat162_rn(__fmul_rn(f.x, s), __fmul_rn(f.y, s));
          o[i] = *reinterpret_cast<const uint32_t*>(&p);
        }
        __stcs(reinterpret_cast<uint4*>(out + (obase + (u ? hc2 : hc)) * D + li * 8),
               make_uint4(o[0], o[1], o[2], o[3]));
      }
    }
  }
}

}  // namespace quant
}  // namespace sol
