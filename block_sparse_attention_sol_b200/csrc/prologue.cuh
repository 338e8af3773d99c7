// Fused QK-RMSNorm + 3D RoPE prologue.
//
// The Sol-H3 runtime merged normalisation and RoPE into single kernels
// (ai-feiten.nl, "Videomodel MiniMax-H3 rendert sneller dan afspelen",
// section "Waar de snelheidswinst vandaan komt").  Per (b, n, h) row of D
// channels, for Q and for K:
//     y_d = x_d / sqrt(mean_d x_d^2 + eps) * gamma[h*D + d]
//     (y_2p, y_2p+1) <- rotation by pos_axis(p)(n) * theta^(-2i/d_axis)
// with the first dt/2 pairs on the frame axis t, the next dh/2 on the row axis
// y and the last dw/2 on the column axis x; i is the pair index within its axis.
//
// HBM-bound streaming kernel.  A group of D/VEC lanes owns one row and moves it
// with 16-byte loads and stores; the sum of squares is reduced with shuffles
// inside the group.  The grid holds a multiple of H groups, so every group keeps
// one head for its whole life: its gains and its channel -> (axis, pair) map sit
// in registers, and the loop advances by whole tokens with 32-bit indices.  Two
// tokens are in flight per iteration.  The per-axis cos/sin tables (a few KB)
// are built once per CTA in shared memory from double-precision angles, so the
// rotation carries no angle error beyond rounding the table to fp32.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include "blocks.cuh"
#include "sm100_ptx.cuh"

namespace sol {
namespace prologue {

struct Params {
  const void* q_in;
  const void* k_in;
  void* q_out;
  void* k_out;
  const float* gamma_q;
  const float* gamma_k;
  int tokens;            // B * N
  int N, H;
  int gt, gh, gw;        // latent grid (T, Hg, Wg)
  int dt, dh, dw;        // rotary channels per axis
  double log2_theta;
  float eps;
  int tab_t, tab_h;      // offsets (in float2) of the y and x tables in shared memory
  int tab_total;
};

template <typename T> struct Vec;
template <> struct Vec<float> { static constexpr int n = 4; };
template <> struct Vec<__nv_bfloat16> { static constexpr int n = 8; };

__device__ __forceinline__ void load_vec(const float* p, float (&x)[4]) {
  const float4 v = __ldcs(reinterpret_cast<const float4*>(p));
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 v = __ldcs(reinterpret_cast<const uint4*>(p));
  x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
  x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  x[4] = __uint_as_float(v.z << 16); x[5] = __uint_as_float(v.z & 0xFFFF0000u);
  x[6] = __uint_as_float(v.w << 16); x[7] = __uint_as_float(v.w & 0xFFFF0000u);
}
__device__ __forceinline__ void store_vec(float* p, const float (&y)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(y[0], y[1], y[2], y[3]);
}
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float (&y)[8]) {
  *reinterpret_cast<uint4*>(p) =
      make_uint4(bf16x2_bits(y[0], y[1]), bf16x2_bits(y[2], y[3]), bf16x2_bits(y[4], y[5]), bf16x2_bits(y[6], y[7]));
}

// Normalise, scale by the gains, rotate the V/2 channel pairs this lane owns.
template <int V, int L>
__device__ __forceinline__ void norm_rotate(float (&x)[V], const float (&g)[V], const float2 (&cs)[V / 2],
                                            unsigned seg, int D, float eps) {
  // packed fp32x2 sum of squares, rsqrt on MUFU (relative error ~2^-22, far inside
  // the prologue's 2^-17 bound), packed gain products
  uint64_t ss2 = 0ull;
#pragma unroll
  for (int e = 0; e < V; e += 2) {
    const uint64_t xe = f2_pack(x[e], x[e + 1]);
    ss2 = f2_fma(xe, xe, ss2);
  }
  float sa, sb;
  f2_unpack(ss2, sa, sb);
  float ss = sa + sb;
#pragma unroll
  for (int off = L / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(seg, ss, off, L);
  const float r = rsqrtf(ss / static_cast<float>(D) + eps);
  const uint64_t r2 = f2_pack(r, r);
#pragma unroll
  for (int e = 0; e < V; e += 2) {
    float y0, y1;
    f2_unpack(f2_mul(f2_mul(f2_pack(x[e], x[e + 1]), r2), f2_pack(g[e], g[e + 1])), y0, y1);
    x[e] = y0 * cs[e / 2].x - y1 * cs[e / 2].y;
    x[e + 1] = y0 * cs[e / 2].y + y1 * cs[e / 2].x;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256, sizeof(T) == 2 ? 2 : 4) qk_prologue_kernel(const Params p) {
  extern __shared__ float2 tab[];   // [gt * dt/2 | gh * dh/2 | gw * dw/2] of (cos, sin)
  const int pt = p.dt / 2, ph = p.dh / 2, pw = p.dw / 2;
  for (int i = threadIdx.x; i < p.tab_total; i += blockDim.x) {
    int pos, pair, d_axis;
    if (i < p.tab_t) { pos = i / pt; pair = i % pt; d_axis = p.dt; }
    else if (i < p.tab_h) { pos = (i - p.tab_t) / ph; pair = (i - p.tab_t) % ph; d_axis = p.dh; }
    else { pos = (i - p.tab_h) / pw; pair = (i - p.tab_h) % pw; d_axis = p.dw; }
    const double angle = static_cast<double>(pos) * exp2(-p.log2_theta * (2.0 * pair) / d_axis);
    double s, c;
    sincos(angle, &s, &c);
    tab[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
  __syncthreads();

  constexpr int V = Vec<T>::n;
  constexpr int L = D / V;            // lanes per row
  constexpr int GPC = 256 / L;        // row groups per CTA
  const int lane_in_row = threadIdx.x % L;
  const unsigned lane = threadIdx.x & 31u;
  const unsigned seg = (L == 32) ? 0xffffffffu : (((1u << (L & 31)) - 1u) << (lane & ~(unsigned)(L - 1)));
  const int grp = blockIdx.x * GPC + threadIdx.x / L;
  const int groups = gridDim.x * GPC;          // a multiple of H (host guarantees)
  const int h = grp % p.H;
  const int tok_step = groups / p.H;

  // per-lane constants: gains and the table slot (axis, pair) of each owned channel pair
  float gq[V], gk[V];
#pragma unroll
  for (int e = 0; e < V; ++e) {
    gq[e] = __ldg(p.gamma_q + h * D + lane_in_row * V + e);
    gk[e] = __ldg(p.gamma_k + h * D + lane_in_row * V + e);
  }
  int axis[V / 2], slot[V / 2];
#pragma unroll
  for (int e = 0; e < V / 2; ++e) {
    const int c = lane_in_row * V + 2 * e;
    if (c < p.dt) { axis[e] = 0; slot[e] = c / 2; }
    else if (c < p.dt + p.dh) { axis[e] = 1; slot[e] = p.tab_t + (c - p.dt) / 2; }
    else { axis[e] = 2; slot[e] = p.tab_h + (c - p.dt - p.dh) / 2; }
  }

  const T* qi = static_cast<const T*>(p.q_in);
  const T* ki = static_cast<const T*>(p.k_in);
  T* qo = static_cast<T*>(p.q_out);
  T* ko = static_cast<T*>(p.k_out);
  const int hw = p.gh * p.gw;

  auto angles = [&](int tok, float2 (&cs)[V / 2]) {
    const int n = tok % p.N;
    const int t = n / hw, y = (n / p.gw) % p.gh, x = n % p.gw;
    const int st = t * pt, sy = y * ph, sx = x * pw;
#pragma unroll
    for (int e = 0; e < V / 2; ++e) cs[e] = tab[slot[e] + (axis[e] == 0 ? st : (axis[e] == 1 ? sy : sx))];
  };

  int tok = grp / p.H;
  for (; tok + tok_step < p.tokens; tok += 2 * tok_step) {
    const int tok2 = tok + tok_step;
    const size_t o1 = (static_cast<size_t>(tok) * p.H + h) * D + lane_in_row * V;
    const size_t o2 = (static_cast<size_t>(tok2) * p.H + h) * D + lane_in_row * V;
    float xq1[V], xk1[V], xq2[V], xk2[V];
    load_vec(qi + o1, xq1);
    load_vec(ki + o1, xk1);
    load_vec(qi + o2, xq2);
    load_vec(ki + o2, xk2);
    float2 cs1[V / 2], cs2[V / 2];
    angles(tok, cs1);
    angles(tok2, cs2);
    norm_rotate<V, L>(xq1, gq, cs1, seg, D, p.eps);
    norm_rotate<V, L>(xk1, gk, cs1, seg, D, p.eps);
    norm_rotate<V, L>(xq2, gq, cs2, seg, D, p.eps);
    norm_rotate<V, L>(xk2, gk, cs2, seg, D, p.eps);
    store_vec(qo + o1, xq1);
    store_vec(ko + o1, xk1);
    store_vec(qo + o2, xq2);
    store_vec(ko + o2, xk2);
  }
  if (tok < p.tokens) {
    const size_t o1 = (static_cast<size_t>(tok) * p.H + h) * D + lane_in_row * V;
    float xq[V], xk[V];
    load_vec(qi + o1, xq);
    load_vec(ki + o1, xk);
    float2 cs[V / 2];
    angles(tok, cs);
    norm_rotate<V, L>(xq, gq, cs, seg, D, p.eps);
    norm_rotate<V, L>(xk, gk, cs, seg, D, p.eps);
    store_vec(qo + o1, xq);
    store_vec(ko + o1, xk);
  }
}

// ------------------------------------------------------------------ prologue + block pooling
// The same prologue, organised by key block so that the pooled means of the
// selection come out of the same pass over Q and K: one CTA per (b, block i)
// takes the block's tokens for every head.  Row group g works on heads g, g +
// GPC, ... (consecutive groups on consecutive heads, so a warp moves 512
// contiguous bytes per token); for each head it writes the block's output rows
// and then the fp32 mean over the block's valid tokens of the stored (rounded)
// outputs, which is what the selection pools.
__device__ __forceinline__ void store_vec_acc(float* p, const float (&y)[4], float (&acc)[4]) {
  store_vec(p, y);
#pragma unroll
  for (int e = 0; e < 4; ++e) acc[e] += y[e];
}
__device__ __forceinline__ void store_vec_acc(__nv_bfloat16* p, const float (&y)[8], float (&acc)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    w[e] = bf16x2_bits(y[2 * e], y[2 * e + 1]);
    acc[2 * e] += __uint_as_float(w[e] << 16);             // the stored (rounded) values
    acc[2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// grid (nb, B); qbar, kbar: fp32 [B, H, nb, D].  Block bi holds the tokens
// block_token(bm, bi, l), l = 0 .. its length - 1, summed in that order.
template <typename T, int D>
__global__ void __launch_bounds__(256) qk_prologue_pool_kernel(const Params p, const BlockMap bm, int nb, float* qbar,
                                                               float* kbar) {
  extern __shared__ float2 tab[];   // [gt * dt/2 | gh * dh/2 | gw * dw/2] of (cos, sin)
  const int pt = p.dt / 2, ph = p.dh / 2, pw = p.dw / 2;
  for (int i = threadIdx.x; i < p.tab_total; i += blockDim.x) {
    int pos, pair, d_axis;
    if (i < p.tab_t) { pos = i / pt; pair = i % pt; d_axis = p.dt; }
    else if (i < p.tab_h) { pos = (i - p.tab_t) / ph; pair = (i - p.tab_t) % ph; d_axis = p.dh; }
    else { pos = (i - p.tab_h) / pw; pair = (i - p.tab_h) % pw; d_axis = p.dw; }
    const double angle = static_cast<double>(pos) * exp2(-p.log2_theta * (2.0 * pair) / d_axis);
    double s, c;
    sincos(angle, &s, &c);
    tab[i] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
  __syncthreads();

  constexpr int V = Vec<T>::n;
  constexpr int L = D / V;            // lanes per row
  constexpr int GPC = 256 / L;        // row groups per CTA
  const int lane_in_row = threadIdx.x % L;
  const unsigned lane = threadIdx.x & 31u;
  const unsigned seg = (L == 32) ? 0xffffffffu : (((1u << (L & 31)) - 1u) << (lane & ~(unsigned)(L - 1)));
  const int grp = threadIdx.x / L;
  const int bi = blockIdx.x, b = blockIdx.y;
  const int cnt = bm.tw == 0 ? min(bm.block, p.N - bi * bm.block) : bm.block;   // tokens of this block
  const float inv = 1.0f / static_cast<float>(cnt);

  int axis[V / 2], slot[V / 2];
#pragma unroll
  for (int e = 0; e < V / 2; ++e) {
    const int c = lane_in_row * V + 2 * e;
    if (c < p.dt) { axis[e] = 0; slot[e] = c / 2; }
    else if (c < p.dt + p.dh) { axis[e] = 1; slot[e] = p.tab_t + (c - p.dt) / 2; }
    else { axis[e] = 2; slot[e] = p.tab_h + (c - p.dt - p.dh) / 2; }
  }
  const T* qi = static_cast<const T*>(p.q_in);
  const T* ki = static_cast<const T*>(p.k_in);
  T* qo = static_cast<T*>(p.q_out);
  T* ko = static_cast<T*>(p.k_out);
  const int hw = p.gh * p.gw;
  auto angles = [&](int n, float2 (&cs)[V / 2]) {
    const int t = n / hw, y = (n / p.gw) % p.gh, x = n % p.gw;
    const int st = t * pt, sy = y * ph, sx = x * pw;
#pragma unroll
    for (int e = 0; e < V / 2; ++e) cs[e] = tab[slot[e] + (axis[e] == 0 ? st : (axis[e] == 1 ? sy : sx))];
  };

  for (int h = grp; h < p.H; h += GPC) {
    float gq[V], gk[V], aq[V], ak[V];
#pragma unroll
    for (int e = 0; e < V; ++e) {
      gq[e] = __ldg(p.gamma_q + h * D + lane_in_row * V + e);
      gk[e] = __ldg(p.gamma_k + h * D + lane_in_row * V + e);
      aq[e] = 0.f;
      ak[e] = 0.f;
    }
    const size_t base = (static_cast<size_t>(b) * p.N * p.H + h) * D + lane_in_row * V;
    const size_t tstride = static_cast<size_t>(p.H) * D;
    int l = 0;
    for (; l + 1 < cnt; l += 2) {   // two tokens in flight
      const int n = block_token(bm, bi, l), n2 = block_token(bm, bi, l + 1);
      const size_t o1 = base + static_cast<size_t>(n) * tstride, o2 = base + static_cast<size_t>(n2) * tstride;
      float xq1[V], xk1[V], xq2[V], xk2[V];
      load_vec(qi + o1, xq1);
      load_vec(ki + o1, xk1);
      load_vec(qi + o2, xq2);
      load_vec(ki + o2, xk2);
      float2 cs1[V / 2], cs2[V / 2];
      angles(n, cs1);
      angles(n2, cs2);
      norm_rotate<V, L>(xq1, gq, cs1, seg, D, p.eps);
      norm_rotate<V, L>(xk1, gk, cs1, seg, D, p.eps);
      norm_rotate<V, L>(xq2, gq, cs2, seg, D, p.eps);
      norm_rotate<V, L>(xk2, gk, cs2, seg, D, p.eps);
      store_vec_acc(qo + o1, xq1, aq);
      store_vec_acc(ko + o1, xk1, ak);
      store_vec_acc(qo + o2, xq2, aq);
      store_vec_acc(ko + o2, xk2, ak);
    }
    if (l < cnt) {
      const int n = block_token(bm, bi, l);
      const size_t o1 = base + static_cast<size_t>(n) * tstride;
      float xq[V], xk[V];
      load_vec(qi + o1, xq);
      load_vec(ki + o1, xk);
      float2 cs[V / 2];
      angles(n, cs);
      norm_rotate<V, L>(xq, gq, cs, seg, D, p.eps);
      norm_rotate<V, L>(xk, gk, cs, seg, D, p.eps);
      store_vec_acc(qo + o1, xq, aq);
      store_vec_acc(ko + o1, xk, ak);
    }
    float* dq = qbar + ((static_cast<size_t>(b) * p.H + h) * nb + bi) * D + lane_in_row * V;
    float* dk = kbar + ((static_cast<size_t>(b) * p.H + h) * nb + bi) * D + lane_in_row * V;
#pragma unroll
    for (int e = 0; e < V; e += 4) {
      *reinterpret_cast<float4*>(dq + e) = make_float4(aq[e] * inv, aq[e + 1] * inv, aq[e + 2] * inv, aq[e + 3] * inv);
      *reinterpret_cast<float4*>(dk + e) = make_float4(ak[e] * inv, ak[e + 1] * inv, ak[e + 2] * inv, ak[e + 3] * inv);
    }
  }
}

// ------------------------------------------------------------------ staged prologue + block pooling
// bf16, D = 128: the arithmetic of qk_prologue_pool_kernel (same norm_rotate,
// same per-block summation order, so the same bits), with the data movement
// organised for HBM.  One persistent CTA per SM walks the (b, block) units
// blockIdx.x, blockIdx.x + gridDim.x, ...; a producer warp copies each token's
// whole Q and K rows (all heads: H * 256 contiguous bytes each in [B, N, H, D])
// into a ring of shared-memory stages with bulk async copies, so that up to
// `stages` tokens per SM are in flight without holding registers, and writes
// the token's rotary table offsets beside them.  Sixteen consumer warps (32
// groups of 16 lanes; group g owns heads g + 32 i, i < HPG) normalise, rotate and
// store from shared memory, accumulate the block means in registers, and hand
// each stage back once read.  Every wait is bounded.
namespace staged {
constexpr int kConsumerWarps = 16;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kGroups = kConsumerWarps * 2;
constexpr int kMaxStages = 16;
constexpr int kHeaderBytes = 1024;   // full[16] | empty[16] | meta[16] (int4) | abort flag
enum : unsigned { kSiteStageFull = 33, kSiteStageFree, kSiteStageTail };
// Shared-memory offset of the stage ring (after the header and the rotary table).
__host__ __device__ constexpr int stage_offset(int tab_total) {
  return (kHeaderBytes + tab_total * 8 + 127) / 128 * 128;
}
}  // namespace staged

__device__ __forceinline__ void load_vec_smem(const unsigned char* p, float (&x)[8]) {
  const uint4 v = *reinterpret_cast<const uint4*>(p);
  x[0] = __uint_as_float(v.x << 16); x[1] = __uint_as_float(v.x & 0xFFFF0000u);
  x[2] = __uint_as_float(v.y << 16); x[3] = __uint_as_float(v.y & 0xFFFF0000u);
  x[4] = __uint_as_float(v.z << 16); x[5] = __uint_as_float(v.z & 0xFFFF0000u);
  x[6] = __uint_as_float(v.w << 16); x[7] = __uint_as_float(v.w & 0xFFFF0000u);
}

// grid: min(B * nb, SMs); stages in [2, kMaxStages], each 2 * H * 256 bytes.
// kPool = false: the plain prologue (no means; qbar, kbar unused), walked in
// runs of bm.block consecutive tokens.
template <int HPG, bool kPool>
__global__ void __launch_bounds__(staged::kThreads, 1)
    qk_prologue_pool_staged_kernel(const Params p, const BlockMap bm, int nb, int stages, float* qbar, float* kbar) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  constexpr int D = 128, V = 8, L = 16;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw);
  uint64_t* empty = full + staged::kMaxStages;
  int4* meta = reinterpret_cast<int4*>(empty + staged::kMaxStages);   // (n, t*pt, y*ph, x*pw) per stage
  volatile int* abort_flag = reinterpret_cast<volatile int*>(meta + staged::kMaxStages);
  float2* tab = reinterpret_cast<float2*>(smem_raw + staged::kHeaderBytes);
  unsigned char* ring = smem_raw + staged::stage_offset(p.tab_total);
  const uint32_t row_bytes = static_cast<uint32_t>(p.H) * D * 2;
  const uint32_t stage_bytes = 2 * row_bytes;
  const int pt = p.dt / 2, ph = p.dh / 2, pw = p.dw / 2;
  if (threadIdx.x == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], staged::kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < p.tab_total; i += blockDim.x) {
    int pos, pair, d_axis;
    if (i < p.tab_t) { pos = i / pt; pair = i % pt; d_axis = p.dt; }
    else if (i < p.tab_h) { pos = (i - p.tab_t) / ph; pair = (i - p.tab_t) % ph; d_axis = p.dh; }
    else { pos = (i - p.tab_h) / pw; pair = (i - p.tab_h) % pw; d_axis = p.dw; }
    const double angle = static_cast<double>(pos) * exp2(-p.log2_theta * (2.0 * pair) / d_axis);
    double sn, cn;
    sincos(angle, &sn, &cn);
    tab[i] = make_float2(static_cast<float>(cn), static_cast<float>(sn));
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = (p.tokens / p.N) * nb;
  const int hw = p.gh * p.gw;
  auto unit_tokens = [&](int bi) { return bm.tw == 0 ? min(bm.block, p.N - bi * bm.block) : bm.block; };

  if (warp == staged::kConsumerWarps) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      uint32_t s = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int b = u / nb, bi = u - b * nb;
        const int cnt = unit_tokens(bi);
        for (int l = 0; l < cnt; ++l, ++s) {
          const int st = static_cast<int>(s % stages);
          if (s >= static_cast<uint32_t>(stages) &&
              !mbar_wait(&empty[st], (s / stages - 1) & 1, abort_flag, staged::kSiteStageFree)) {
            ok = false;
            break;
          }
          const int n = block_token(bm, bi, l);
          meta[st] = make_int4(n, (n / hw) * pt, ((n / p.gw) % p.gh) * ph, (n % p.gw) * pw);
          const size_t off = (static_cast<size_t>(b) * p.N + n) * row_bytes;
          unsigned char* dst = ring + static_cast<size_t>(st) * stage_bytes;
          mbar_arrive_expect_tx(&full[st], stage_bytes);
          bulk_load(dst, static_cast<const unsigned char*>(p.q_in) + off, row_bytes, &full[st]);
          bulk_load(dst + row_bytes, static_cast<const unsigned char*>(p.k_in) + off, row_bytes, &full[st]);
        }
      }
      // every copy issued completes before the CTA exits (on the abort path too)
      const uint32_t first = s > static_cast<uint32_t>(stages) ? s - stages : 0u;
      for (uint32_t i = first; i < s; ++i)
        mbar_wait(&full[i % stages], (i / stages) & 1, abort_flag, staged::kSiteStageTail, SOL_WAIT_LIMIT_NS, false);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int grp = threadIdx.x / L;               // 0 .. kGroups - 1
  const int lane_in_row = threadIdx.x % L;
  const unsigned seg = 0xffffu << (lane & 16);
  float gq[HPG][V], gk[HPG][V];
#pragma unroll
  for (int i = 0; i < HPG; ++i) {
    const int h = min(grp + staged::kGroups * i, p.H - 1);
#pragma unroll
    for (int e = 0; e < V; ++e) {
      gq[i][e] = __ldg(p.gamma_q + h * D + lane_in_row * V + e);
      gk[i][e] = __ldg(p.gamma_k + h * D + lane_in_row * V + e);
    }
  }
  int axis[V / 2], slot[V / 2];
#pragma unroll
  for (int e = 0; e < V / 2; ++e) {
    const int c = lane_in_row * V + 2 * e;
    if (c < p.dt) { axis[e] = 0; slot[e] = c / 2; }
    else if (c < p.dt + p.dh) { axis[e] = 1; slot[e] = p.tab_t + (c - p.dt) / 2; }
    else { axis[e] = 2; slot[e] = p.tab_h + (c - p.dt - p.dh) / 2; }
  }
  __nv_bfloat16* qo = static_cast<__nv_bfloat16*>(p.q_out);
  __nv_bfloat16* ko = static_cast<__nv_bfloat16*>(p.k_out);
  uint32_t s = 0;
  bool ok = true;
  for (int u = blockIdx.x; u < units; u += gridDim.x) {
    const int b = u / nb, bi = u - b * nb;
    const int cnt = unit_tokens(bi);
    const float inv = 1.0f / static_cast<float>(cnt);
    float aq[HPG][V], ak[HPG][V];
#pragma unroll
    for (int i = 0; i < HPG; ++i)
#pragma unroll
      for (int e = 0; e < V; ++e) {
        aq[i][e] = 0.f;
        ak[i][e] = 0.f;
      }
    for (int l = 0; l < cnt; ++l, ++s) {
      const int st = static_cast<int>(s % stages);
      ok = mbar_wait(&full[st], (s / stages) & 1, abort_flag, staged::kSiteStageFull);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      const int4 m = meta[st];
      float2 cs[V / 2];
#pragma unroll
      for (int e = 0; e < V / 2; ++e) cs[e] = tab[slot[e] + (axis[e] == 0 ? m.y : (axis[e] == 1 ? m.z : m.w))];
      const unsigned char* src = ring + static_cast<size_t>(st) * stage_bytes + lane_in_row * V * 2;
      const size_t obase = (static_cast<size_t>(b) * p.N + m.x) * p.H * D + lane_in_row * V;
#pragma unroll
      for (int i = 0; i < HPG; ++i) {
        const int h = grp + staged::kGroups * i;
        if (h < p.H) {
          float xq[V], xk[V];
          load_vec_smem(src + h * D * 2, xq);
          load_vec_smem(src + row_bytes + h * D * 2, xk);
          norm_rotate<V, L>(xq, gq[i], cs, seg, D, p.eps);
          norm_rotate<V, L>(xk, gk[i], cs, seg, D, p.eps);
          if constexpr (kPool) {
            store_vec_acc(qo + obase + h * D, xq, aq[i]);
            store_vec_acc(ko + obase + h * D, xk, ak[i]);
          } else {
            store_vec(qo + obase + h * D, xq);
            store_vec(ko + obase + h * D, xk);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
    if (!ok) break;
    if constexpr (!kPool) continue;
#pragma unroll
    for (int i = 0; i < HPG; ++i) {
      const int h = grp + staged::kGroups * i;
      if (h < p.H) {
        float* dq = qbar + ((static_cast<size_t>(b) * p.H + h) * nb + bi) * D + lane_in_row * V;
        float* dk = kbar + ((static_cast<size_t>(b) * p.H + h) * nb + bi) * D + lane_in_row * V;
#pragma unroll
        for (int e = 0; e < V; e += 4) {
          *reinterpret_cast<float4*>(dq + e) =
              make_float4(aq[i][e] * inv, aq[i][e + 1] * inv, aq[i][e + 2] * inv, aq[i][e + 3] * inv);
          *reinterpret_cast<float4*>(dk + e) =
              make_float4(ak[i][e] * inv, ak[i][e + 1] * inv, ak[i][e + 2] * inv, ak[i][e + 3] * inv);
        }
      }
    }
  }
}

}  // namespace prologue
}  // namespace sol
