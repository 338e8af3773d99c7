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
// HBM-bound streaming kernel: each group of D/VEC lanes owns one row and moves
// it with 16-byte vector loads and stores; the sum of squares is reduced with
// warp shuffles inside the group.  The per-axis cos/sin tables (a few KB) are
// built once per CTA in shared memory, so the trigonometry is amortised over all
// heads and tokens the CTA streams.  Arithmetic in fp32.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace sol {
namespace prologue {

struct Params {
  const void* q_in;
  const void* k_in;
  void* q_out;
  void* k_out;
  const float* gamma_q;
  const float* gamma_k;
  long long rows;        // B * N * H
  int N, H;
  int gt, gh, gw;        // latent grid (T, Hg, Wg)
  int dt, dh, dw;        // rotary channels per axis
  float log2_theta;
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
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void store_vec(float* p, const float (&y)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(y[0], y[1], y[2], y[3]);
}
__device__ __forceinline__ void store_vec(__nv_bfloat16* p, const float (&y)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);   // .x = low half
    w[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// One row: normalise, scale by gamma, rotate.  `lane_in_row` owns channels
// [lane_in_row*V, lane_in_row*V + V).
template <typename T, int D>
__device__ __forceinline__ void process_row(const T* in, T* out, const float* gamma, int h, const float2* tab_t,
                                            const float2* tab_y, const float2* tab_x, int dt, int dh, float eps,
                                            int lane_in_row) {
  constexpr int V = Vec<T>::n;
  constexpr int L = D / V;   // lanes per row
  float x[V];
  load_vec(in + lane_in_row * V, x);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < V; ++e) ss = fmaf(x[e], x[e], ss);
  // only the L lanes of this row's group take part (rows may run out unevenly in a warp)
  const unsigned lane = threadIdx.x & 31u;
  const unsigned seg = (L == 32) ? 0xffffffffu : (((1u << (L & 31)) - 1u) << (lane & ~(unsigned)(L - 1)));
#pragma unroll
  for (int off = L / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(seg, ss, off, L);
  const float r = 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
  const float* g = gamma + h * D + lane_in_row * V;
  float y[V];
#pragma unroll
  for (int e = 0; e < V; e += 2) {
    const float y0 = x[e] * r * __ldg(g + e);
    const float y1 = x[e + 1] * r * __ldg(g + e + 1);
    const int c = lane_in_row * V + e;   // even channel index
    float2 cs;
    if (c < dt) cs = tab_t[c >> 1];
    else if (c < dt + dh) cs = tab_y[(c - dt) >> 1];
    else cs = tab_x[(c - dt - dh) >> 1];
    y[e] = y0 * cs.x - y1 * cs.y;
    y[e + 1] = y0 * cs.y + y1 * cs.x;
  }
  store_vec(out + lane_in_row * V, y);
}

// Grid-stride over rows; both Q and K rows are handled in the same iteration.
template <typename T, int D>
__global__ void __launch_bounds__(256) qk_prologue_kernel(const Params p) {
  extern __shared__ float2 tab[];   // [gt * dt/2 | gh * dh/2 | gw * dw/2] of (cos, sin)
  const int pt = p.dt / 2, ph = p.dh / 2, pw = p.dw / 2;
  for (int i = threadIdx.x; i < p.tab_total; i += blockDim.x) {
    int pos, pair, d_axis;
    if (i < p.tab_t) { pos = i / pt; pair = i % pt; d_axis = p.dt; }
    else if (i < p.tab_h) { pos = (i - p.tab_t) / ph; pair = (i - p.tab_t) % ph; d_axis = p.dh; }
    else { pos = (i - p.tab_h) / pw; pair = (i - p.tab_h) % pw; d_axis = p.dw; }
    const float inv_freq = exp2f(-p.log2_theta * (2.0f * pair) / static_cast<float>(d_axis));
    float s, c;
    sincosf(static_cast<float>(pos) * inv_freq, &s, &c);
    tab[i] = make_float2(c, s);
  }
  __syncthreads();

  constexpr int V = Vec<T>::n;
  constexpr int L = D / V;
  const int lane_in_row = threadIdx.x % L;
  const long long group = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / L;
  const long long groups = static_cast<long long>(gridDim.x) * blockDim.x / L;
  const T* qi = static_cast<const T*>(p.q_in);
  const T* ki = static_cast<const T*>(p.k_in);
  T* qo = static_cast<T*>(p.q_out);
  T* ko = static_cast<T*>(p.k_out);
  const int hw = p.gh * p.gw;
  for (long long row = group; row < p.rows; row += groups) {
    const int h = static_cast<int>(row % p.H);
    const int n = static_cast<int>((row / p.H) % p.N);
    const int t = n / hw, y = (n / p.gw) % p.gh, x = n % p.gw;
    const float2* tt = tab + t * pt;
    const float2* ty = tab + p.tab_t + y * ph;
    const float2* tx = tab + p.tab_h + x * pw;
    const size_t off = static_cast<size_t>(row) * D;
    process_row<T, D>(qi + off, qo + off, p.gamma_q, h, tt, ty, tx, p.dt, p.dh, p.eps, lane_in_row);
    process_row<T, D>(ki + off, ko + off, p.gamma_k, h, tt, ty, tx, p.dt, p.dh, p.eps, lane_in_row);
  }
}

}  // namespace prologue
}  // namespace sol
