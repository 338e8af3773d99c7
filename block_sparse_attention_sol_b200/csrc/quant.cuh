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
// Both are HBM streams: D / 16 lanes per row, each with 16 channels (32 bytes of
// bf16, 16 bytes of codes), packed fp32x2 arithmetic, and each CTA walks a
// contiguous run of tokens with counters instead of per-element index division.  Slice g starts g * g_stride rows into the
// buffers, so several tensors can share one exchange buffer.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cstdint>
#include "sm100_ptx.cuh"

namespace sol {
namespace quant {

enum : int { kSplitHeads = 0, kSplitTokens = 1 };
enum : int { kInt8 = 0, kE4M3 = 1 };

// One row's share of a pack: 16 channels of one thread, L lanes per row.
template <int L, int CODE>
__device__ __forceinline__ uint4 encode16(const uint32_t (&w)[8], unsigned seg, float* scale_out) {
  const float levels = CODE == kInt8 ? 127.0f : 448.0f;
  float a = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    a = fmaxf(a, fmaxf(fabsf(__uint_as_float(w[i] << 16)), fabsf(__uint_as_float(w[i] & 0xFFFF0000u))));
#pragma unroll
  for (int o = L / 2; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(seg, a, o));
  const float s = __fdiv_rn(a, levels);
  *scale_out = s;
  if (!(s > 0.f)) return make_uint4(0u, 0u, 0u, 0u);
  const float rcp = __fdiv_rn(levels, a);
  const uint64_t rcp2 = f2_pack(rcp, rcp);
  uint32_t out[4];
  if constexpr (CODE == kInt8) {
    // |x * rcp| <= 127 (1 + 2^-23): no clamp needed.  q + 1.5 * 2^23 rounds q to
    // the nearest (even) integer, held in the sum's low mantissa bits: its low
    // byte is the two's complement code.  The product must be rounded before the
    // add (a fused multiply-add rounds ties such as 63.5 the other way), so the
    // add is a scalar __fadd_rn, which is never contracted.
    uint32_t b[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float lo, hi;
      f2_unpack(f2_mul(f2_pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u)), rcp2), lo, hi);
      b[2 * i] = __float_as_uint(__fadd_rn(lo, 12582912.0f));
      b[2 * i + 1] = __float_as_uint(__fadd_rn(hi, 12582912.0f));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
      out[k] = __byte_perm(__byte_perm(b[4 * k], b[4 * k + 1], 0x0040), __byte_perm(b[4 * k + 2], b[4 * k + 3], 0x0040),
                           0x5410);
  } else {
    uint32_t p[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float lo, hi;
      f2_unpack(f2_mul(f2_pack(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u)), rcp2), lo, hi);
      p[i] = __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) out[k] = p[2 * k] | (p[2 * k + 1] << 16);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// 16 codes (one 16-byte word) times s, as 8 bf16 pairs.
template <int CODE>
__device__ __forceinline__ void decode16(const uint4 c, float s, uint32_t (&o)[8]) {
  const uint64_t s2 = f2_pack(s, s);
  const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
  if constexpr (CODE == kInt8) {
    // byte c ^ 0x80 into the low mantissa of 2^23: the float is 2^23 + c + 128 exactly
    const uint64_t bias2 = f2_pack(-8388736.0f, -8388736.0f);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t u = cw[j] ^ 0x80808080u;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float f0 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540 | (2 * k)));
        const float f1 = __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7540 | (2 * k + 1)));
        float lo, hi;
        f2_unpack(f2_mul(f2_add(f2_pack(f0, f1), bias2), s2), lo, hi);
        const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
        o[2 * j + k] = *reinterpret_cast<const uint32_t*>(&p);
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(cw[j] >> (16 * k)),
                                                         __NV_E4M3);
        const float2 f = __half22float2(__half2(h));
        float lo, hi;
        f2_unpack(f2_mul(f2_pack(f.x, f.y), s2), lo, hi);
        const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
        o[2 * j + k] = *reinterpret_cast<const uint32_t*>(&p);
      }
    }
  }
}

// A CTA handles a contiguous run of tokens (b, n) of x; thread t handles channels
// 16 (t % L) .. +15 (L = D / 16 lanes per row) of heads h = t / L + k S,
// S = blockDim / L, two heads per pass with all four loads issued first.  Index
// arithmetic is 32-bit: B * N * H < 2^31 (checked on the host); one division per
// CTA, then counters.
template <int D, int CODE>
__global__ void __launch_bounds__(512) quant_pack_kernel(const __nv_bfloat16* __restrict__ x,
                                                         uint8_t* __restrict__ codes, float* __restrict__ scales,
                                                         int B, int N, int H, int G, int split, long long g_stride) {
  constexpr int L = D / 16;
  const int li = threadIdx.x % L;
  const int S = blockDim.x / L;
  const unsigned lane = threadIdx.x & 31u;
  const unsigned seg = (((1u << L) - 1u) << (lane & ~static_cast<unsigned>(L - 1)));
  const int Nc = split == kSplitHeads ? N : N / G;
  const int Hc = split == kSplitHeads ? H / G : H;
  const int total = B * N;
  const int chunk = (total + gridDim.x - 1) / gridDim.x;
  const int t0 = blockIdx.x * chunk, t1 = min(total, t0 + chunk);
  if (t0 >= t1) return;
  int b = t0 / N, n = t0 - b * N;
  int g_tok = split == kSplitHeads ? 0 : n / Nc;   // split tokens: one destination per token
  int nc = n - g_tok * Nc;
  for (int tok = t0; tok < t1; ++tok) {
    const __nv_bfloat16* src = x + static_cast<long long>(tok) * H * D + li * 16;
    for (int h = threadIdx.x / L; h < H; h += 2 * S) {
      const int h2 = h + S;
      const bool two = h2 < H;
      uint4 r[4];
      r[0] = __ldcs(reinterpret_cast<const uint4*>(src + static_cast<long long>(h) * D));
      r[1] = __ldcs(reinterpret_cast<const uint4*>(src + static_cast<long long>(h) * D + 8));
      if (two) {
        r[2] = __ldcs(reinterpret_cast<const uint4*>(src + static_cast<long long>(h2) * D));
        r[3] = __ldcs(reinterpret_cast<const uint4*>(src + static_cast<long long>(h2) * D + 8));
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        if (u == 1 && !two) break;
        const int hh = u ? h2 : h;
        const uint32_t w[8] = {r[2 * u].x, r[2 * u].y, r[2 * u].z, r[2 * u].w,
                               r[2 * u + 1].x, r[2 * u + 1].y, r[2 * u + 1].z, r[2 * u + 1].w};
        int g = g_tok, hc = hh;
        if (split == kSplitHeads) { g = hh / Hc; hc = hh - g * Hc; }
        const long long drow = g * g_stride + (static_cast<long long>(b) * Nc + nc) * Hc + hc;
        float s;
        const uint4 cw = encode16<L, CODE>(w, seg, &s);
        __stcs(reinterpret_cast<uint4*>(codes + drow * D + li * 16), cw);
        if (li == 0) scales[drow] = s;
      }
    }
    ++n;
    ++nc;
    if (nc == Nc) { nc = 0; ++g_tok; }
    if (n == N) { n = 0; nc = 0; g_tok = 0; ++b; }
  }
}

// A CTA handles a contiguous run of received row groups (g, b, nc); thread t
// handles channels 16 (t % L) .. +15 of heads hc = t / L + k S, kUnpackRows per
// pass with all their loads issued first (four cost occupancy and ran slower).
constexpr int kUnpackRows = 2;

template <int D, int CODE>
__global__ void __launch_bounds__(512) dequant_unpack_kernel(const uint8_t* __restrict__ codes,
                                                             const float* __restrict__ scales,
                                                             __nv_bfloat16* __restrict__ out, int B, int Nc, int Hc,
                                                             int G, int split, long long g_stride) {
  constexpr int L = D / 16;
  const int li = threadIdx.x % L;
  const int S = blockDim.x / L;
  const int total = G * B * Nc;
  const int chunk = (total + gridDim.x - 1) / gridDim.x;
  const int t0 = blockIdx.x * chunk, t1 = min(total, t0 + chunk);
  if (t0 >= t1) return;
  int gb = t0 / Nc, nc = t0 - gb * Nc;
  int g = gb / B, b = gb - g * B;
  for (int blk = t0; blk < t1; ++blk) {   // blk = (g * B + b) * Nc + nc
    const long long rbase = g * g_stride + (static_cast<long long>(b) * Nc + nc) * Hc;
    long long obase;   // output row of hc = 0
    if (split == kSplitHeads) obase = (static_cast<long long>(b) * G * Nc + static_cast<long long>(g) * Nc + nc) * Hc;
    else obase = (static_cast<long long>(b) * Nc + nc) * (static_cast<long long>(G) * Hc) + static_cast<long long>(g) * Hc;
    for (int hc = threadIdx.x / L; hc < Hc; hc += kUnpackRows * S) {
      uint4 c[kUnpackRows];
      float sc[kUnpackRows];
#pragma unroll
      for (int u = 0; u < kUnpackRows; ++u) {
        const int hu = hc + u * S;
        if (hu < Hc) {
          c[u] = __ldcs(reinterpret_cast<const uint4*>(codes + (rbase + hu) * D + li * 16));
          sc[u] = __ldg(scales + rbase + hu);
        }
      }
#pragma unroll
      for (int u = 0; u < kUnpackRows; ++u) {
        const int hu = hc + u * S;
        if (hu >= Hc) break;
        uint32_t o[8];
        decode16<CODE>(c[u], sc[u], o);
        uint4* dst = reinterpret_cast<uint4*>(out + (obase + hu) * D + li * 16);
        __stcs(dst, make_uint4(o[0], o[1], o[2], o[3]));
        __stcs(dst + 1, make_uint4(o[4], o[5], o[6], o[7]));
      }
    }
    if (++nc == Nc) {
      nc = 0;
      if (++b == B) { b = 0; ++g; }
    }
  }
}

}  // namespace quant
}  // namespace sol
