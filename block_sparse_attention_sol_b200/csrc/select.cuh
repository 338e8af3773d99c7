// Block selection ("preparation" of the sparse attention, which the Sol-H3
// runtime made 76.4% faster: ai-feiten.nl, "Videomodel MiniMax-H3 rendert
// sneller dan afspelen", section "Waar de snelheidswinst vandaan komt").
//
//   pool:   qbar[b,h,i,:] = mean of q[b,n,h,:] over the valid tokens n of block i
//           (same for k).  HBM-bound: one CTA per (b, block, tensor) streams the
//           block's rows (all heads, contiguous) with 16-byte loads.
//   score:  s[b,h,i,j] = qbar[b,h,i,:] . kbar[b,h,j,:]  in fp32 (SIMT FMA; a
//           tensor-core score would round the scores and move the top-k
//           boundary).  A CTA keeps 32 (or 16) rows' scores in shared memory;
//           each thread computes 4 rows x 4 keys of a 128-key chunk: 16-byte
//           shared loads, rows broadcast across the warp, keys 32 apart.
//   top-k:  per row, the k largest scores, exact ties to the lower j, written in
//           ascending j.  A warp holds four rows' order-preserving keys in
//           registers (two for nb > 1024), finds each row's threshold by a
//           most-significant-bit-first search of the 32-bit key space (the
//           searches interleaved; a row stops once exactly k keys pass), then
//           compacts the winners in ascending j with ballots.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>
#include <cmath>

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
// A CTA scores 8 * RPW query blocks (RPW rows per warp: 4, or 2 when 32 rows of
// scores do not fit in shared memory) against all key blocks, in chunks of kKeys.
constexpr int kKeys = 128;       // key blocks per shared-memory chunk
constexpr int kThreads = 256;    // warp w: rows RPW w .. +RPW-1; lane l: keys l + {0, 32, 64, 96} of a chunk
constexpr int kMaxNb = 2048;

__host__ __device__ constexpr size_t score_topk_smem_bytes(int D, int rows, int nb) {
  return (static_cast<size_t>(D + 4) * (rows + kKeys) + static_cast<size_t>(rows) * nb) * sizeof(float);
}

__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.0f);   // -0 -> +0 so equal scores get equal keys
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// A threshold T for each of NR rows held as KPL keys per lane (key j at lane
// j % 32, slot j / 32; 0 pads, below every real key) such that the row's topk
// largest keys are those above T plus the first ones equal to T, in id order:
// built most significant bit first as the largest T with count(key >= T) >=
// topk (the k-th largest key), except that a row stops early at the first
// candidate T with count(key >= T) == topk exactly, whose set {key >= T} is
// already the row's top-k.  The NR searches share one bit loop, so their
// counts and warp reductions overlap; a lane counts in four partial sums.
template <int KPL, int NR>
__device__ __forceinline__ void kth_largest(const uint32_t (&key)[NR][KPL], int topk, uint32_t (&prefix)[NR]) {
  bool done[NR];
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    prefix[r] = 0u;
    done[r] = false;
  }
#pragma unroll 1
  for (int bit = 31; bit >= 0; --bit) {
    uint32_t cnt[NR];
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const uint32_t cand = prefix[r] | (1u << bit);
      uint32_t c[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int q = 0; q < KPL; ++q) c[q & 3] += key[r][q] >= cand ? 1u : 0u;
      cnt[r] = (c[0] + c[1]) + (c[2] + c[3]);
    }
    bool all_done = true;
#pragma unroll
    for (int r = 0; r < NR; ++r) {
      const int total = static_cast<int>(__reduce_add_sync(0xffffffffu, cnt[r]));
      if (!done[r] && total >= topk) {
        prefix[r] |= 1u << bit;
        done[r] = total == topk;
      }
      all_done = all_done && done[r];
    }
    if (all_done) break;   // warp-uniform: the totals are
  }
}

// The row's ids with key above `kth`, plus the first (topk - count above) with
// key equal to it, written in ascending j.
template <int KPL>
__device__ __forceinline__ void compact_row(const uint32_t (&key)[KPL], uint32_t kth, int nb, int topk, int32_t* out,
                                            int lane) {
  uint32_t gt = 0;
#pragma unroll
  for (int q = 0; q < KPL; ++q) gt += key[q] > kth ? 1u : 0u;
  const int need_eq = topk - static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
  const uint32_t lt_mask = (1u << lane) - 1u;
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int q = 0; q < KPL; ++q) {
    if (q * 32 >= nb) break;
    const int j = q * 32 + lane;
    const bool is_gt = key[q] > kth;
    const bool is_eq = key[q] == kth;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, is_eq);
    const int eq_rank = eq_seen + __popc(eq_mask & lt_mask);
    const bool sel = is_gt || (is_eq && eq_rank < need_eq);
    const uint32_t sel_mask = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(sel_mask & lt_mask)] = j;
    written += __popc(sel_mask);
    eq_seen += __popc(eq_mask);
  }
}

// Selection variants, all optional (zero / null: plain top-k):
//  - kForceDiagonal keeps the query's own key block, kForceFirstFrame the key
//    blocks 0 .. n_first - 1 (those holding tokens of the first latent frame),
//    ahead of every scored block (forced blocks beyond the row's k: lowest ids);
//  - head_k[h] (device, clamped to [1, topk]) replaces topk for head h;
//  - kTopP keeps, instead of a fixed k, the shortest prefix of the row's order
//    (forced blocks first, then descending score, ties to the lower id) whose
//    softmax mass, softmax_j(scale s_ij) over all key blocks, reaches top_p;
//    at least the forced blocks and one block, at most the row's k.
//  A row's ids beyond its count are set to -1; counts (nullable) receives the count.
enum : unsigned { kForceDiagonal = 1u, kForceFirstFrame = 2u, kTopP = 4u };

struct SelectArgs {
  int32_t* idx;            // [B, H, nb, topk]
  float* scores;           // nullable [B, H, nb, nb]
  int32_t* counts;         // nullable [B, H, nb]
  const int32_t* head_k;   // nullable [H]
  int nb, topk, H;
  unsigned flags;
  int n_first;
  float top_p;             // in (0, 1] with kTopP
  float scale_log2;        // softmax scale * log2(e) with kTopP
};

// Dynamic shared memory: qs[rows][D+4] | ks[kKeys][D+4] | sc[rows][nb].  The 4-float row
// padding puts the 16-byte loads of 8 consecutive rows on distinct banks.
// Scores of rows r0 .. r0 + nrows - 1 of (b, h) = bh against all key blocks, left in sc.
template <int D, int RPW>
__device__ __forceinline__ void score_rows(const float* __restrict__ qbar, const float* __restrict__ kbar, float* smem,
                                           int bh, int r0, int nrows, int nb, float* __restrict__ scores_out) {
  constexpr int P = D + 4;
  constexpr int kRows = 8 * RPW;
  float* qs = smem;
  float* ks = qs + kRows * P;
  float* sc = ks + kKeys * P;
  const float* qb = qbar + static_cast<size_t>(bh) * nb * D;
  const float* kb = kbar + static_cast<size_t>(bh) * nb * D;

  for (int e = threadIdx.x; e < kRows * (D / 4); e += kThreads) {
    const int r = e / (D / 4), d = (e % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < nrows) v = __ldg(reinterpret_cast<const float4*>(qb + static_cast<size_t>(r0 + r) * D + d));
    *reinterpret_cast<float4*>(qs + r * P + d) = v;
  }
  const int lane = threadIdx.x & 31;
  const int rg = (threadIdx.x >> 5) * RPW;   // this warp's rows
  // Key chunks are double-buffered through registers: the next chunk's global
  // loads are in flight while the current chunk's FMAs run.
  constexpr int kPre = kKeys * (D / 4) / kThreads;   // float4 per thread per chunk
  float4 pre[kPre];
  auto load_chunk = [&](int j0) {
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
      const int e = threadIdx.x + u * kThreads;
      const int j = e / (D / 4), d = (e % (D / 4)) * 4;
      pre[u] = j0 + j < nb ? __ldg(reinterpret_cast<const float4*>(kb + static_cast<size_t>(j0 + j) * D + d))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  load_chunk(0);
  for (int j0 = 0; j0 < nb; j0 += kKeys) {
    __syncthreads();   // previous chunk fully consumed (and qs written, the first time)
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
      const int e = threadIdx.x + u * kThreads;
      const int j = e / (D / 4), d = (e % (D / 4)) * 4;
      *reinterpret_cast<float4*>(ks + j * P + d) = pre[u];
    }
    __syncthreads();
    if (j0 + kKeys < nb) load_chunk(j0 + kKeys);
    float acc[RPW][4];   // [row][key lane + 32 c]
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 4
    for (int d = 0; d < D; d += 4) {   // channels in ascending order: one fixed fp32 rounding sequence per score
      float4 qv[RPW], kv[4];
#pragma unroll
      for (int r = 0; r < RPW; ++r) qv[r] = *reinterpret_cast<const float4*>(qs + (rg + r) * P + d);
#pragma unroll
      for (int c = 0; c < 4; ++c) kv[c] = *reinterpret_cast<const float4*>(ks + (lane + 32 * c) * P + d);
#pragma unroll
      for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[r][c] = fmaf(qv[r].x, kv[c].x, acc[r][c]);
          acc[r][c] = fmaf(qv[r].y, kv[c].y, acc[r][c]);
          acc[r][c] = fmaf(qv[r].z, kv[c].z, acc[r][c]);
          acc[r][c] = fmaf(qv[r].w, kv[c].w, acc[r][c]);
        }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = j0 + lane + 32 * c;
      if (j < nb) {
#pragma unroll
        for (int r = 0; r < RPW; ++r) sc[(rg + r) * nb + j] = acc[r][c];
      }
    }
  }
  __syncthreads();

  if (scores_out != nullptr) {
    for (int e = threadIdx.x; e < nrows * nb; e += kThreads) {
      const int r = e / nb, j = e % nb;
      scores_out[(static_cast<size_t>(bh) * nb + r0 + r) * nb + j] = sc[r * nb + j];
    }
  }
}

// Order-preserving key of score j of a row, or the largest key for a forced block
// (order_key of a finite score never reaches it), 0 for padding j >= nb.
__device__ __forceinline__ uint32_t select_key(const float* row_scores, int j, int i, const SelectArgs& a) {
  if (j >= a.nb) return 0u;
  const bool forced = ((a.flags & kForceDiagonal) && j == i) || ((a.flags & kForceFirstFrame) && j < a.n_first);
  return forced ? 0xffffffffu : order_key(row_scores[j]);
}

// Writes the row's ids beyond its count as -1 and the count itself.
__device__ __forceinline__ void finish_row(const SelectArgs& a, size_t row, int count, int lane) {
  for (int e = count + lane; e < a.topk; e += 32) a.idx[row * a.topk + e] = -1;
  if (a.counts != nullptr && lane == 0) a.counts[row] = count;
}

__device__ __forceinline__ float warp_sum(float v) {
  // xor butterfly: every lane ends with the same sum, added in the same order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Softmax mass of the keys >= t (each lane adds its own in slot order, then the warp sums).
template <int KPL>
__device__ __forceinline__ float mass_at_least(const uint32_t (&key)[KPL], const float (&e)[KPL], uint32_t t) {
  float m = 0.f;
#pragma unroll
  for (int q = 0; q < KPL; ++q) m += key[q] >= t ? e[q] : 0.f;
  return warp_sum(m);
}

// grid (ceil(nb / (8 RPW)), B * H).  KPL = keys per lane in the top-k, nb <= 32 * KPL.
template <int D, int RPW, int KPL>
__global__ void __launch_bounds__(kThreads, 1) score_topk_kernel(const float* __restrict__ qbar,
                                                                 const float* __restrict__ kbar, SelectArgs a) {
  extern __shared__ float smem[];
  constexpr int kRows = 8 * RPW;
  const int nb = a.nb;
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * kRows;
  const int nrows = min(kRows, nb - r0);
  score_rows<D, RPW>(qbar, kbar, smem, bh, r0, nrows, nb, a.scores);
  const float* sc = smem + (kRows + kKeys) * (D + 4);

  // top-k: each warp searches NT rows of its share together (rows r, r + 8, ...,
  // their keys in registers; NT = 2 for the widest rows, whose keys take 64
  // registers each); slots past the CTA's last row repeat the pass's first row
  constexpr int kWarps = kThreads / 32;
  constexpr int NT = (KPL >= 64 ? 2 : 4) < kRows / kWarps ? (KPL >= 64 ? 2 : 4) : kRows / kWarps;
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int kr = a.head_k == nullptr ? a.topk : min(max(__ldg(a.head_k + bh % a.H), 1), a.topk);
  for (int r1 = warp; r1 < nrows; r1 += NT * kWarps) {
    int rr[NT];
#pragma unroll
    for (int u = 0; u < NT; ++u) rr[u] = r1 + u * kWarps < nrows ? r1 + u * kWarps : r1;
    uint32_t key[NT][KPL];
#pragma unroll
    for (int q = 0; q < KPL; ++q)
#pragma unroll
      for (int u = 0; u < NT; ++u) key[u][q] = select_key(sc + rr[u] * nb, q * 32 + lane, r0 + rr[u], a);
    uint32_t kth[NT];
    kth_largest<KPL, NT>(key, kr, kth);
#pragma unroll
    for (int u = 0; u < NT; ++u) {
      if (u > 0 && rr[u] == r1) break;
      const size_t row = static_cast<size_t>(bh) * nb + r0 + rr[u];
      compact_row<KPL>(key[u], kth[u], nb, kr, a.idx + row * a.topk, lane);
      finish_row(a, row, kr, lane);
    }
  }
}

// Top-p selection (kTopP): one warp per row, keys and softmax terms in registers.
// The cut is found as the largest key T whose mass(key >= T) reaches top_p times
// the row's total, by the same most-significant-bit-first search as the top-k;
// blocks tied at T are then taken in id order until the mass is reached.
template <int D, int RPW, int KPL>
__global__ void __launch_bounds__(kThreads, 1) score_topp_kernel(const float* __restrict__ qbar,
                                                                 const float* __restrict__ kbar, SelectArgs a) {
  extern __shared__ float smem[];
  constexpr int kRows = 8 * RPW;
  const int nb = a.nb;
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * kRows;
  const int nrows = min(kRows, nb - r0);
  score_rows<D, RPW>(qbar, kbar, smem, bh, r0, nrows, nb, a.scores);
  const float* sc = smem + (kRows + kKeys) * (D + 4);

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int kcap = a.head_k == nullptr ? a.topk : min(max(__ldg(a.head_k + bh % a.H), 1), a.topk);
  for (int r = warp; r < nrows; r += kThreads / 32) {
    const float* row_sc = sc + r * nb;
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < KPL; ++q)
      if (q * 32 + lane < nb) mx = fmaxf(mx, row_sc[q * 32 + lane]);
    mx = warp_max(mx);
    uint32_t key[KPL];
    float e[KPL];
    uint32_t nf = 0;
#pragma unroll
    for (int q = 0; q < KPL; ++q) {
      const int j = q * 32 + lane;
      key[q] = select_key(row_sc, j, r0 + r, a);
      e[q] = j < nb ? exp2f((row_sc[j] - mx) * a.scale_log2) : 0.f;
      nf += key[q] == 0xffffffffu ? 1u : 0u;
    }
    const int n_forced = static_cast<int>(__reduce_add_sync(0xffffffffu, nf));
    const float target = a.top_p * mass_at_least<KPL>(key, e, 0u);
    uint32_t t = 0u;
#pragma unroll 1
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = t | (1u << bit);
      if (mass_at_least<KPL>(key, e, cand) >= target) t = cand;
    }
    int count = n_forced;
    if (t != 0xffffffffu) {
      uint32_t gt = 0, eq = 0;
      float et = 0.f;
#pragma unroll
      for (int q = 0; q < KPL; ++q) {
        gt += key[q] > t ? 1u : 0u;
        eq += key[q] == t ? 1u : 0u;
        if (key[q] == t) et = e[q];   // tied keys are equal scores: equal terms
      }
      const int n_gt = static_cast<int>(__reduce_add_sync(0xffffffffu, gt));
      const int n_eq = static_cast<int>(__reduce_add_sync(0xffffffffu, eq));
      et = warp_max(et);
      const float need = target - mass_at_least<KPL>(key, e, t + 1u);
      const float take = et > 0.f ? fminf(ceilf(need / et), static_cast<float>(n_eq)) : static_cast<float>(n_eq);
      count = max(count, n_gt + max(static_cast<int>(take), 1));
    }
    count = min(max(count, 1), kcap);
    uint32_t keys1[1][KPL];
#pragma unroll
    for (int q = 0; q < KPL; ++q) keys1[0][q] = key[q];
    uint32_t kth[1];
    kth_largest<KPL, 1>(keys1, count, kth);
    const size_t row = static_cast<size_t>(bh) * nb + r0 + r;
    compact_row<KPL>(keys1[0], kth[0], nb, count, a.idx + row * a.topk, lane);
    finish_row(a, row, count, lane);
  }
}

}  // namespace select
}  // namespace sol
