// Block-sparse attention forward on sm_100a tensor cores (bf16 in, fp32 accumulate).
//
// Sol-Attn keeps, per query block, only the key blocks that matter and runs
// exact softmax attention over them (ai-feiten.nl, "Videomodel MiniMax-H3
// rendert sneller dan afspelen", section "Waar de snelheidswinst vandaan
// komt").  For every (b, h, query block i) this kernel computes, over the keys
// m < N of the blocks idx[b,h,i,0..k-1]:
//     l_m = scale * q_n . k_m,   O_n = sum_m softmax(l)_m v_m,   LSE_n = ln sum_m exp(l_m)
//
// Design (one CTA per SM, persistent over 128-query tiles in head-major order so
// that the K/V of the head being processed stays hot in L2):
//   warp 0      TMA producer: Q tile, then K_j / V_j gathered by block id
//               (coordinate = id * 128), 128-byte swizzled, K one step ahead of V.
//   warp 1      TMEM owner + single-thread MMA issuer:
//                 S_j = Q K_j^T  (SS, both K-major)  into S[j % 2]
//                 O  += P_j V_j  (TS, P from TMEM, V MN-major)
//   warps 2..5  softmax: one thread per query row (TMEM lane), online softmax in
//               the exp2 domain with a lazy rescale (O is only rescaled when the
//               running max grows by more than 2^8), P written to TMEM as bf16;
//               epilogue O / l -> bf16 and LSE.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P0 [384,448) P1 [448,512).
// Shared memory: Q 32 KB, K 3 x 32 KB, V 2 x 32 KB.
#pragma once
#include <cuda.h>
#include "sm100_ptx.cuh"

namespace sol {
namespace attn100 {

constexpr int kBlock = 128;            // tokens per query / key block
constexpr int kHeadDim = 128;
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kTileBytes = kBlock * kHeadDim * 2;   // 32 KB bf16 tile
constexpr int kHalfBytes = kTileBytes / 2;          // one 64-column swizzled box
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
constexpr float kRescaleLog2 = 8.0f;   // lazy-rescale threshold (log2 units)

struct __align__(1024) Smem {
  uint8_t q[kTileBytes];
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  const int32_t* idx;     // [B, H, nb, topk]
  __nv_bfloat16* o;       // [B, N, H, D]
  float* lse;             // [B, H, N]
  int B, N, H, nb, topk;
  int num_tiles;
  float scale_log2;       // softmax scale * log2(e)
};

// Wait-site ids reported in the error info word.
enum : unsigned { kSiteQEmpty = 1, kSiteKEmpty, kSiteVEmpty, kSiteQFull, kSiteKFull, kSiteVFull, kSitePFull,
                  kSiteOFree, kSiteSFull, kSitePvDone, kSiteDrain, kSiteTail };

__device__ __forceinline__ void decode_tile(const Params& p, int t, int& b, int& h, int& qb) {
  qb = t % p.nb;
  const int bh = t / p.nb;
  h = bh % p.H;
  b = bh / p.H;
}

__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kKStages; ++s) { mbar_init(&sm.k_full[s], 1); mbar_init(&sm.k_empty[s], 1); }
    for (int s = 0; s < kVStages; ++s) { mbar_init(&sm.v_full[s], 1); mbar_init(&sm.v_empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&sm.s_full[s], 1); mbar_init(&sm.p_full[s], 128); }
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.o_free, 128);
    mbar_init(&sm.drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t g = 0;          // global key-block counter (same sequence as the MMA issuer)
      uint32_t kq = 0, vq = 0; // K / V loads issued so far
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
        int b, h, qb;
        decode_tile(p, t, b, h, qb);
        if (it > 0 && !(ok = mbar_wait(&sm.q_empty, (it - 1) & 1, abort_flag, kSiteQEmpty))) break;
        mbar_arrive_expect_tx(&sm.q_full, kTileBytes);
        tma_load_4d(sm.q, &tm_q, &sm.q_full, 0, h, qb * kBlock, b);
        tma_load_4d(sm.q + kHalfBytes, &tm_q, &sm.q_full, 64, h, qb * kBlock, b);
        const int32_t* list = p.idx + (static_cast<size_t>(b * p.H + h) * p.nb + qb) * p.topk;
        // order: K0, K1, V0, K2, V1, ..., V_{k-1}
        for (int j = 0; j <= p.topk && ok; ++j) {
          if (j < p.topk) {
            const int blk = __ldg(list + j);
            const uint32_t st = kq % kKStages, use = kq / kKStages;
            if (use > 0 && !(ok = mbar_wait(&sm.k_empty[st], (use - 1) & 1, abort_flag, kSiteKEmpty))) break;
            mbar_arrive_expect_tx(&sm.k_full[st], kTileBytes);
            tma_load_4d(sm.k[st], &tm_k, &sm.k_full[st], 0, h, blk * kBlock, b);
            tma_load_4d(sm.k[st] + kHalfBytes, &tm_k, &sm.k_full[st], 64, h, blk * kBlock, b);
            ++kq;
          }
          if (j >= 1) {
            const int blk = __ldg(list + j - 1);
            const uint32_t st = vq % kVStages, use = vq / kVStages;
            if (use > 0 && !(ok = mbar_wait(&sm.v_empty[st], (use - 1) & 1, abort_flag, kSiteVEmpty))) break;
            mbar_arrive_expect_tx(&sm.v_full[st], kTileBytes);
            tma_load_4d(sm.v[st], &tm_v, &sm.v_full[st], 0, h, blk * kBlock, b);
            tma_load_4d(sm.v[st] + kHalfBytes, &tm_v, &sm.v_full[st], 64, h, blk * kBlock, b);
            ++vq;
          }
        }
        g += p.topk;
      }
      // Before the CTA exits, every load issued must have landed (stage s
      // received loads s, s + stages, ...; wait for the phase of its last one).
      for (uint32_t s = 0; s < kKStages; ++s) {
        if (s < kq) {
          const uint32_t uses = (kq - s + kKStages - 1) / kKStages;          // loads issued into stage s
          mbar_wait(&sm.k_full[s], (uses - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
        }
      }
      for (uint32_t s = 0; s < kVStages; ++s) {
        if (s < vq) {
          const uint32_t uses = (vq - s + kVStages - 1) / kVStages;
          mbar_wait(&sm.v_full[s], (uses - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
        }
      }
      if (it > 0) mbar_wait(&sm.q_full, (it - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, true);
      const uint32_t q_base = smem_addr(sm.q);
      uint32_t g = 0;
      int it = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t gg) -> bool {
        const uint32_t st = gg % kKStages;
        if (!mbar_wait(&sm.k_full[st], (gg / kKStages) & 1, abort_flag, kSiteKFull)) return false;
        tc_fence_after();
        const uint32_t k_base = smem_addr(sm.k[st]);
        const uint32_t d = tmem + kColS + (gg & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(d, smem_desc_sw128(q_base + off, 16, 1024), smem_desc_sw128(k_base + off, 16, 1024), kIdescS,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(&sm.k_empty[st]);
        tc_commit(&sm.s_full[gg & 1]);
        return true;
      };
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
        if (!(ok = mbar_wait(&sm.q_full, it & 1, abort_flag, kSiteQFull))) break;
        tc_fence_after();
        if (!(ok = issue_s(g))) break;
        for (int j = 0; j < p.topk; ++j) {
          const uint32_t gg = g + j;
          if (j + 1 < p.topk) {
            if (!(ok = issue_s(gg + 1))) break;
          } else {
            tc_commit(&sm.q_empty);   // every S MMA of this tile has been issued
          }
          if (!(ok = mbar_wait(&sm.p_full[gg & 1], (gg >> 1) & 1, abort_flag, kSitePFull))) break;
          if (j == 0 && it > 0 && !(ok = mbar_wait(&sm.o_free, (it - 1) & 1, abort_flag, kSiteOFree))) break;
          const uint32_t vs = gg % kVStages;
          if (!(ok = mbar_wait(&sm.v_full[vs], (gg / kVStages) & 1, abort_flag, kSiteVFull))) break;
          tc_fence_after();
          const uint32_t v_base = smem_addr(sm.v[vs]);
          const uint32_t a_tm = tmem + kColP + (gg & 1) * 64;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // 16 keys per step: P columns kk*8.., V rows kk*16.. (2 KB of the swizzled tile)
            mma_ts(tmem + kColO, a_tm + kk * 8, smem_desc_sw128(v_base + kk * 2048, kHalfBytes, 1024), kIdescPV,
                   (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&sm.v_empty[vs]);
          tc_commit(&sm.pv_done);
        }
        g += p.topk;
      }
      // Drain: every MMA issued must complete before TMEM is released.
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, abort_flag, kSiteDrain, 200000000ull, false);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;          // query row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int tail_valid = p.N - (p.nb - 1) * kBlock;   // valid keys in the last block
    uint32_t g = 0;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
      int b, h, qb;
      decode_tile(p, t, b, h, qb);
      const int32_t* list = p.idx + (static_cast<size_t>(b * p.H + h) * p.nb + qb) * p.topk;
      float m = -INFINITY;   // running max in log2 units (possibly stale by < 2^8)
      float l = 0.f;         // running sum of exp2(x - m)
      for (int j = 0; j < p.topk; ++j) {
        const uint32_t gg = g + j;
        const uint32_t buf = gg & 1;
        ok = mbar_wait(&sm.s_full[buf], (gg >> 1) & 1, abort_flag, kSiteSFull);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128_wait(tmem + lane_off + kColS + buf * 128, sr);
        const int blk = __ldg(list + j);
        if (blk == p.nb - 1 && tail_valid < kBlock) {
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e >= tail_valid) sr[e] = __float_as_uint(-INFINITY);
        }
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 128; ++e) mx = fmaxf(mx, __uint_as_float(sr[e]));
        mx *= p.scale_log2;
        const bool rescale = mx > m + kRescaleLog2;
        const float m_use = rescale ? mx : m;
        float rowsum = 0.f;
        const uint32_t p_addr = tmem + lane_off + kColP + buf * 64;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pk[32];
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int c = half * 2 + c2;
              const float p0 = ex2_approx(fmaf(__uint_as_float(sr[c * 32 + e]), p.scale_log2, -m_use));
              const float p1 = ex2_approx(fmaf(__uint_as_float(sr[c * 32 + e + 1]), p.scale_log2, -m_use));
              rowsum += p0 + p1;
              pk[c2 * 16 + (e >> 1)] = pack_bf16x2(p0, p1);
            }
          tmem_st32(p_addr + half * 32, pk);   // P_j as bf16 pairs: 64 columns per row
        }
        if (j > 0) {
          // PV of the previous step must be done before O may be rescaled, and is
          // waited every step so this thread tracks every phase of pv_done.
          ok = mbar_wait(&sm.pv_done, (gg - 1) & 1, abort_flag, kSitePvDone);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            const float alpha = rescale ? ex2_approx(m - m_use) : 1.f;
            const uint32_t o_addr = tmem + lane_off + kColO;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t orr[32];
              tmem_ld32_wait(o_addr + c * 32, orr);
#pragma unroll
              for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
              tmem_st32(o_addr + c * 32, orr);
            }
            l *= alpha;
          }
        }
        m = m_use;
        l += rowsum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sm.p_full[buf]);
      }
      if (!ok) break;
      // epilogue: O / l and LSE
      const uint32_t gl = g + p.topk - 1;
      ok = mbar_wait(&sm.pv_done, gl & 1, abort_flag, kSitePvDone);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t orr[128];
      tmem_ld128_wait(tmem + lane_off + kColO, orr);
      tc_fence_before();
      mbar_arrive(&sm.o_free);
      const int n = qb * kBlock + row;
      if (n < p.N) {
        const float inv = 1.f / l;
        uint4* dst = reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kHeadDim);
#pragma unroll
        for (int e = 0; e < 128; e += 8) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(orr[e + 0]) * inv, __uint_as_float(orr[e + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(orr[e + 2]) * inv, __uint_as_float(orr[e + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(orr[e + 4]) * inv, __uint_as_float(orr[e + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(orr[e + 6]) * inv, __uint_as_float(orr[e + 7]) * inv);
          dst[e / 8] = w;
        }
        p.lse[(static_cast<size_t>(b) * p.H + h) * p.N + n] = (m + __log2f(l)) * 0.69314718055994531f;
      }
      g += p.topk;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace attn100
}  // namespace sol
