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

template <int CODE>
__device__ __forceinline__ uint8_t encode(float q) {
  if constexpr (CODE == kInt8) {
    const int c = min(max(__float2int_rn(q), -127), 127);
    return static_cast<uint8_t>(static_cast<int8_t>(c));
  } else {
    return static_cast<uint8_t>(__nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3));
  }
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

// CTA c handles tokens (b, n) = c, c + gridDim, ... of x; thread t handles
// channels 8 (t % L) .. +7 of heads t / L, t / L + blockDim / L, ... (L = D / 8
// lanes per row).  Index arithmetic is 32-bit and per token: B * N * H < 2^31
// (checked on the host).
template <int D, int CODE>
__global__ void __launch_bounds__(1024) quant_pack_kernel(const __nv_bfloat16* __restrict__ x,
                                                          uint8_t* __restrict__ codes, float* __restrict__ scales,
                                                          int B, int N, int H, int G, int split, long long g_stride) {
  constexpr int L = D / 8;
  const int li = threadIdx.x % L;
  const unsigned lane = threadIdx.x & 31u;
  const unsigned seg = (L == 32) ? 0xffffffffu : (((1u << L) - 1u) << (lane & ~static_cast<unsigned>(L - 1)));
  const float levels = CODE == kInt8 ? 127.0f : 448.0f;
  const int Nc = split == kSplitHeads ? N : N / G;
  const int Hc = split == kSplitHeads ? H / G : H;
  for (int tok = blockIdx.x; tok < B * N; tok += gridDim.x) {   // tok = b * N + n
  const int b = tok / N, n = tok - b * N;
  const int g_tok = split == kSplitHeads ? 0 : n / Nc;          // split tokens: one destination per token
  const int nc = n - g_tok * Nc;
  for (int h = threadIdx.x / L; h < H; h += blockDim.x / L) {
    float v[8];
    bf16x8_to_f32(__ldcs(reinterpret_cast<const uint4*>(x + (static_cast<long long>(tok) * H + h) * D + li * 8)), v);
    float a = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) a = fmaxf(a, fabsf(v[e]));
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(seg, a, o));
    const float s = __fdiv_rn(a, levels);
    const float rcp = __fdiv_rn(levels, a > 0.f ? a : 1.0f);
    int g = g_tok, hc = h;
    if (split == kSplitHeads) { g = h / Hc; hc = h - g * Hc; }
    const long long drow = g * g_stride + (static_cast<long long>(b) * Nc + nc) * Hc + hc;
    uint32_t w[2] = {0u, 0u};
    if (s > 0.f) {
#pragma unroll
      for (int e = 0; e < 8; ++e)
        w[e >> 2] |= static_cast<uint32_t>(encode<CODE>(__fmul_rn(v[e], rcp))) << (8 * (e & 3));
    }
    __stcs(reinterpret_cast<uint2*>(codes + drow * D + li * 8), make_uint2(w[0], w[1]));
    if (li == 0) scales[drow] = s;
  }
  }
}

// CTA c handles received row groups (g, b, nc) = c, c + gridDim, ...; thread t
// handles channels 8 (t % L) .. +7 of heads hc = t / L, t / L + blockDim / L, ...
template <int D, int CODE>
__global__ void __launch_bounds__(1024) dequant_unpack_kernel(const uint8_t* __restrict__ codes,
                                                              const float* __restrict__ scales,
                                                              __nv_bfloat16* __restrict__ out, int B, int Nc, int Hc,
                                                              int G, int split, long long g_stride) {
  constexpr int L = D / 8;
  const int li = threadIdx.x % L;
  for (int blk = blockIdx.x; blk < G * B * Nc; blk += gridDim.x) {   // blk = (g * B + b) * Nc + nc
  const int gb = blk / Nc, nc = blk - gb * Nc;
  const int g = gb / B, b = gb - g * B;
  const long long rbase = g * g_stride + (static_cast<long long>(b) * Nc + nc) * Hc;
  long long obase;   // output row of hc = 0
  if (split == kSplitHeads) obase = (static_cast<long long>(b) * G * Nc + static_cast<long long>(g) * Nc + nc) * Hc;
  else obase = (static_cast<long long>(b) * Nc + nc) * (static_cast<long long>(G) * Hc) + static_cast<long long>(g) * Hc;
  for (int hc = threadIdx.x / L; hc < Hc; hc += blockDim.x / L) {
    const long long srow = rbase + hc;
    const float s = __ldg(scales + srow);
    const uint2 c = __ldcs(reinterpret_cast<const uint2*>(codes + srow * D + li * 8));
    const uint32_t cw[2] = {c.x, c.y};
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 c2 = decode2<CODE>((cw[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
      const __nv_bfloat162 p = __floats2bfloat162_rn(__fmul_rn(c2.x, s), __fmul_rn(c2.y, s));
      o[i] = *reinterpret_cast<const uint32_t*>(&p);
    }
    __stcs(reinterpret_cast<uint4*>(out + (obase + hc) * D + li * 8), make_uint4(o[0], o[1], o[2], o[3]));
  }
  }
}

}  // namespace quant
}  // namespace sol
