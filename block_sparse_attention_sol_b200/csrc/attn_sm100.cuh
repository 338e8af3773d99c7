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
//   warp 0      TMA producer: K_j / V_j gathered by block id (coordinate = id * 128),
//               128-byte swizzled, K one step ahead of V.
//   warp 1      TMEM owner + single-thread MMA issuer, both MMAs with A in TMEM:
//                 S_j = Q K_j^T  into S[j % 2]     (Q from TMEM, K from shared memory)
//                 O  += P_j V_j                    (P from TMEM, V from shared memory)
//               Keeping Q in TMEM halves the shared-memory operand traffic of the
//               S MMAs, which would otherwise saturate the tensor core's 128 B/clk
//               shared-memory read path at N = 128.
//   warps 2..5  softmax + epilogue: one thread per query row (its TMEM lane).
//               Each tile starts by loading the thread's Q row from global
//               memory into TMEM.  Online softmax in the exp2 domain with a lazy
//               rescale (O is rescaled only when the running max grows by more
//               than 2^8); P is written to TMEM as bf16 once PV of the previous
//               step has completed (single P buffer); epilogue O / l -> bf16, LSE.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P [384,448) Q [448,512).
// Shared memory: K 3 x 32 KB, V 3 x 32 KB.
//
// Descriptor note: the MMA descriptors are built once per call and each K-step
// adds a compile-time offset; building them per instruction measurably slows
// tcgen05.mma issue.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"

namespace sol {
namespace attn100 {

constexpr int kBlock = 128;            // tokens per query / key block
constexpr int kHeadDim = 128;
constexpr int kKStages = 3;
constexpr int kVStages = 3;
constexpr int kTileBytes = kBlock * kHeadDim * 2;   // 32 KB bf16 tile
constexpr int kHalfBytes = kTileBytes / 2;          // one 64-column swizzled box
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384, kColQ = 448;
constexpr float kRescaleLog2 = 8.0f;   // lazy-rescale threshold (log2 units)
// Of every 8 exponential pairs, this many run as a polynomial on the FMA pipe
// instead of on MUFU (16 results per clock per SM).
constexpr int kPolyPairsPer8 = 0;

struct __align__(1024) Smem {
  uint8_t k[kKStages][kTileBytes];
  uint8_t v[kVStages][kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full;
  uint64_t pv_done, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  const __nv_bfloat16* q; // [B, N, H, D]
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

// K-step offsets (16-byte units) inside a 128-byte-swizzled K-major tile: 16
// channels = 32 bytes per step, the second 64-channel box 16 KB further.
__device__ __forceinline__ constexpr uint32_t kstep_off(int kk) {
  return static_cast<uint32_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
}

__device__ __forceinline__ void decode_tile(const Params& p, int t, int& b, int& h, int& qb) {
  qb = t % p.nb;
  const int bh = t / p.nb;
  h = bh % p.H;
  b = bh / p.H;
}

__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_fwd_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                       const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    mbar_init(&sm.q_full, 4);            // one arrival per softmax warp
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kKStages; ++s) { mbar_init(&sm.k_full[s], 1); mbar_init(&sm.k_empty[s], 1); }
    for (int s = 0; s < kVStages; ++s) { mbar_init(&sm.v_full[s], 1); mbar_init(&sm.v_empty[s], 1); }
    mbar_init(&sm.s_full[0], 1);
    mbar_init(&sm.s_full[1], 1);
    mbar_init(&sm.p_full, 4);
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.o_free, 4);
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
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t kq = 0, vq = 0;   // K / V loads issued so far
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int b, h, qb;
        decode_tile(p, t, b, h, qb);
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
      }
      // Before the CTA exits, every load issued must have landed (stage s
      // received loads s, s + stages, ...; wait for the phase of its last one).
      for (uint32_t s = 0; s < kKStages; ++s)
        if (s < kq) {
          const uint32_t uses = (kq - s + kKStages - 1) / kKStages;
          mbar_wait(&sm.k_full[s], (uses - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
        }
      for (uint32_t s = 0; s < kVStages; ++s)
        if (s < vq) {
          const uint32_t uses = (vq - s + kVStages - 1) / kVStages;
          mbar_wait(&sm.v_full[s], (uses - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, true);
      const uint32_t q_tm = tmem + kColQ;
      const uint32_t p_tm = tmem + kColP;
      const uint32_t o_tm = tmem + kColO;
      uint32_t g = 0;
      int it = 0;
      bool ok = true;
      // S(gg) = Q K^T into S[gg % 2]
      auto issue_s = [&](uint32_t gg) -> bool {
        const uint32_t st = gg % kKStages;
        if (!mbar_wait(&sm.k_full[st], (gg / kKStages) & 1, abort_flag, kSiteKFull)) return false;
        tc_fence_after();
        const uint64_t kd = smem_desc_sw128(smem_addr(sm.k[st]), 16, 1024);
        const uint32_t d = tmem + kColS + (gg & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ts(d, q_tm + kk * 8, kd + kstep_off(kk), kIdescS, kk > 0 ? 1u : 0u);
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
          if (!(ok = mbar_wait(&sm.p_full, gg & 1, abort_flag, kSitePFull))) break;
          if (j == 0 && it > 0 && !(ok = mbar_wait(&sm.o_free, (it - 1) & 1, abort_flag, kSiteOFree))) break;
          const uint32_t vs = gg % kVStages;
          if (!(ok = mbar_wait(&sm.v_full[vs], (gg / kVStages) & 1, abort_flag, kSiteVFull))) break;
          tc_fence_after();
          const uint64_t vd = smem_desc_sw128(smem_addr(sm.v[vs]), kHalfBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: P columns kk*8.., V rows kk*16.. (2 KB)
            mma_ts(o_tm, p_tm + kk * 8, vd + static_cast<uint32_t>(kk * 128), kIdescPV,
                   (j > 0 || kk > 0) ? 1u : 0u);
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
    const uint32_t q_addr = tmem + lane_off + kColQ;
    const uint32_t p_addr = tmem + lane_off + kColP;
    const uint32_t o_addr = tmem + lane_off + kColO;
    const int tail_valid = p.N - (p.nb - 1) * kBlock;   // valid keys in the last block
    uint32_t g = 0;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
      int b, h, qb;
      decode_tile(p, t, b, h, qb);
      const int32_t* list = p.idx + (static_cast<size_t>(b * p.H + h) * p.nb + qb) * p.topk;
      const int n = qb * kBlock + row;
      // ---- Q row into TMEM (A operand of the S MMAs: lane = row, 2 bf16 per column)
      if (it > 0) {
        ok = mbar_wait(&sm.q_empty, (it - 1) & 1, abort_flag, kSiteQEmpty);   // previous tile's S MMAs done
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
      }
      {
        uint32_t q0[32], q1[32];
        if (n < p.N) {
          const uint4* src =
              reinterpret_cast<const uint4*>(p.q + ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kHeadDim);
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 w0 = __ldg(src + c), w1 = __ldg(src + 8 + c);
            q0[4 * c] = w0.x; q0[4 * c + 1] = w0.y; q0[4 * c + 2] = w0.z; q0[4 * c + 3] = w0.w;
            q1[4 * c] = w1.x; q1[4 * c + 1] = w1.y; q1[4 * c + 2] = w1.z; q1[4 * c + 3] = w1.w;
          }
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) { q0[c] = 0u; q1[c] = 0u; }
        }
        tmem_st32(q_addr, q0);
        tmem_st32(q_addr + 32, q1);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.q_full);
      }
      float m = -INFINITY;   // running max in log2 units (possibly stale by < 2^8)
      float l = 0.f;         // running sum of exp2(x - m)
      int blk = __ldg(list);
      for (int j = 0; j < p.topk; ++j) {
        const uint32_t gg = g + j;
        const uint32_t buf = gg & 1;
        const int blk_next = (j + 1 < p.topk) ? __ldg(list + j + 1) : 0;
        ok = mbar_wait(&sm.s_full[buf], (gg >> 1) & 1, abort_flag, kSiteSFull);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128_wait(tmem + lane_off + kColS + buf * 128, sr);
        if (blk == p.nb - 1 && tail_valid < kBlock) {
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e >= tail_valid) sr[e] = __float_as_uint(-INFINITY);
        }
        // row max: 16 independent chains, then a small tree
        float pm[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) pm[c] = fmaxf(__uint_as_float(sr[c]), __uint_as_float(sr[c + 16]));
#pragma unroll
        for (int e = 32; e < 128; e += 32)
#pragma unroll
          for (int c = 0; c < 16; ++c)
            pm[c] = fmax3(pm[c], __uint_as_float(sr[e + c]), __uint_as_float(sr[e + 16 + c]));
#pragma unroll
        for (int c = 0; c < 5; ++c) pm[c] = fmax3(pm[c], pm[c + 5], pm[c + 10]);
        const float mx = fmaxf(fmax3(pm[0], pm[1], pm[2]), fmax3(pm[3], pm[4], pm[15])) * p.scale_log2;
        const bool rescale = mx > m + kRescaleLog2;
        const float m_use = rescale ? mx : m;
        const uint64_t neg_m2 = f2_pack(-m_use, -m_use);
        const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
        // P = exp2(s * scale - m) as bf16 pairs (kept in registers); 8 partial sums
        uint32_t pk0[32], pk1[32];
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int e = 0; e < 128; e += 2) {
          float a0, a1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), scale2, neg_m2), a0, a1);
          float p0, p1;
          if (((e >> 1) & 7) >= 8 - kPolyPairsPer8) {
            exp2_poly_pair(a0, a1, p0, p1);        // FMA pipe
          } else {
            p0 = ex2_approx(a0);                   // MUFU
            p1 = ex2_approx(a1);
          }
          acc[(e >> 1) & 3] = f2_add(acc[(e >> 1) & 3], f2_pack(p0, p1));
          if (e < 64) pk0[e >> 1] = pack_bf16x2(p0, p1);
          else pk1[(e - 64) >> 1] = pack_bf16x2(p0, p1);
        }
        float rs0, rs1, rs2, rs3;
        f2_unpack(f2_add(acc[0], acc[1]), rs0, rs1);
        f2_unpack(f2_add(acc[2], acc[3]), rs2, rs3);
        const float rowsum = (rs0 + rs1) + (rs2 + rs3);
        if (j > 0) {
          // PV of the previous step must be done before P is overwritten and O
          // rescaled; waited every step so this thread tracks every phase.
          ok = mbar_wait(&sm.pv_done, (gg - 1) & 1, abort_flag, kSitePvDone);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            const float alpha = rescale ? ex2_approx(m - m_use) : 1.f;
            const uint64_t alpha2 = f2_pack(alpha, alpha);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t orr[32];
              tmem_ld32_wait(o_addr + c * 32, orr);
#pragma unroll
              for (int e = 0; e < 32; e += 2) {
                float o0, o1;
                f2_unpack(f2_mul(f2_pack(__uint_as_float(orr[e]), __uint_as_float(orr[e + 1])), alpha2), o0, o1);
                orr[e] = __float_as_uint(o0);
                orr[e + 1] = __float_as_uint(o1);
              }
              tmem_st32(o_addr + c * 32, orr);
            }
            l *= alpha;
          }
        }
        tmem_st32(p_addr, pk0);          // 128 keys -> 64 columns of bf16 pairs
        tmem_st32(p_addr + 32, pk1);
        m = m_use;
        l += rowsum;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
        blk = blk_next;
      }
      if (!ok) break;
      // epilogue: O / l and LSE
      ok = mbar_wait(&sm.pv_done, (g + p.topk - 1) & 1, abort_flag, kSitePvDone);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t orr[128];
      tmem_ld128_wait(o_addr, orr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free);
      if (n < p.N) {
        const float inv = 1.f / l;
        const uint64_t inv2 = f2_pack(inv, inv);
        uint4* dst = reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kHeadDim);
#pragma unroll
        for (int e = 0; e < 128; e += 8) {
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float o0, o1;
            f2_unpack(f2_mul(f2_pack(__uint_as_float(orr[e + 2 * u]), __uint_as_float(orr[e + 2 * u + 1])), inv2),
                      o0, o1);
            w[u] = pack_bf16x2(o0, o1);
          }
          dst[e / 8] = make_uint4(w[0], w[1], w[2], w[3]);
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
