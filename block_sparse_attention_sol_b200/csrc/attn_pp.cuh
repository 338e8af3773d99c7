// Block-sparse attention forward on sm_100a tensor cores, two query tiles per CTA
// in ping-pong (bf16 in, fp32 accumulate).
//
// Same operation as attn_sm100.cuh (ai-feiten.nl, "Videomodel MiniMax-H3
// rendert sneller dan afspelen", section "Waar de snelheidswinst vandaan
// komt"): for every (b, h, query block i), exact softmax attention over the
// keys m < N of the blocks idx[b,h,i,0..k-1], O and the natural-log LSE.
//
// Why two tiles: with one tile, each step's softmax (MUFU) waits for its S
// MMA and the next PV MMA waits for that softmax, so the tensor pipe and MUFU
// take turns.  Here a CTA owns two query tiles (slots 0 and 1, each with its
// own key list) and a softmax warpgroup per slot; while one slot's softmax
// runs, the tensor pipe works on the other slot.  MMA order per step j:
//     S0(j), PV1(j-1), S1(j), PV0(j)
//
// Roles (12 warps, setmaxnreg gives the softmax warpgroups the registers):
//   warp 0        TMA producer: Q tiles, then one ring of kRing 32 KB slots carrying
//                 K and V tiles of both slots in the order the MMAs consume them.
//   warp 1        TMEM owner + single-thread MMA issuer.
//   warps 4..7    softmax + epilogue of slot 0; warps 8..11 of slot 1: one thread
//                 per query row (its TMEM lane), the whole 128-key row in registers.
// TMEM: S0 [0,128) S1 [128,256) O0 [256,384) O1 [384,512).  P(j) of a slot is
// written as bf16 over the first 64 columns of its own S; S(j+1) of the slot is
// issued only after PV(j) has completed.  Q0, Q1 live in shared memory (the S MMAs
// read both operands from shared memory).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"

namespace sol {
namespace attnpp {

constexpr int kBlock = 128;
constexpr int kHeadDim = 128;
constexpr int kTileBytes = kBlock * kHeadDim * 2;   // 32 KB bf16 tile
constexpr int kHalfBytes = kTileBytes / 2;          // one 64-column swizzled box
constexpr int kRing = 5;                            // K/V ring slots
constexpr int kThreads = 384;
constexpr uint32_t kRegsControl = 88;               // warpgroup 0 after setmaxnreg.dec
constexpr uint32_t kRegsSoftmax = 208;              // warpgroups 1, 2 after setmaxnreg.inc
// 128 * 88 + 256 * 208 = 64,512 = 384 threads * 168 registers at launch: the
// build checks that the kernel launches with 168 registers per thread.
static_assert(128 * kRegsControl + 256 * kRegsSoftmax == kThreads * 168, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;                // lazy-rescale threshold (log2 units)

struct __align__(1024) Smem {
  uint8_t q[2][kTileBytes];
  uint8_t ring[kRing][kTileBytes];
  uint64_t q_full[2], q_empty[2];
  uint64_t ring_full[kRing], ring_free[kRing];
  uint64_t s_full[2], p_full[2], pv_done[2], o_free[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  const int32_t* idx;     // [B, H, nb, topk]
  __nv_bfloat16* o;       // [B, N, H, D]
  float* lse;             // [B, H, N]
  int B, N, H, nb, topk;
  int num_tiles, num_pairs;
  float scale_log2;       // softmax scale * log2(e)
};

enum : unsigned { kSiteQEmpty = 1, kSiteRingFree, kSiteQFull, kSiteRingFull, kSitePFull, kSiteOFree, kSiteSFull,
                  kSitePvDone, kSiteDrain, kSiteTail };

__device__ __forceinline__ constexpr uint32_t kstep_off(int kk) {
  return static_cast<uint32_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
}

__device__ __forceinline__ void decode_tile(const Params& p, int t, int& b, int& h, int& qb) {
  qb = t % p.nb;
  const int bh = t / p.nb;
  h = bh % p.H;
  b = bh / p.H;
}

// Tiles of pair pr: 2 pr and 2 pr + 1; an odd last pair repeats its tile in
// slot 1, whose results are then not stored.
__device__ __forceinline__ int pair_tile(const Params& p, int pr, int slot, bool& store) {
  const int t = 2 * pr + slot;
  store = t < p.num_tiles;
  return store ? t : 2 * pr;
}

// The ring carries, per step j of a pair, in the MMA order: K0(j), V1(j-1),
// K1(j), V0(j) (each present when its step lies in [0, topk)): 4 topk loads.

__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.q_full[x], 1);
      mbar_init(&sm.q_empty[x], 1);
      mbar_init(&sm.s_full[x], 1);
      mbar_init(&sm.p_full[x], 4);    // one arrival per softmax warp of the slot
      mbar_init(&sm.pv_done[x], 1);
      mbar_init(&sm.o_free[x], 4);
    }
    for (int s = 0; s < kRing; ++s) { mbar_init(&sm.ring_full[s], 1); mbar_init(&sm.ring_free[s], 1); }
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

  if (threadIdx.x < 128) {
    warpgroup_regs_dec<kRegsControl>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- TMA producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t rq = 0;   // ring loads issued
      int pi = 0;        // pairs begun by this CTA
      bool ok = true;
      for (int pr = blockIdx.x; pr < p.num_pairs && ok; pr += gridDim.x, ++pi) {
        int b[2], h[2], qb[2];
        const int32_t* list[2];
        for (int x = 0; x < 2; ++x) {
          bool store;
          decode_tile(p, pair_tile(p, pr, x, store), b[x], h[x], qb[x]);
          list[x] = p.idx + (static_cast<size_t>(b[x] * p.H + h[x]) * p.nb + qb[x]) * p.topk;
          if (pi > 0 && !(ok = mbar_wait(&sm.q_empty[x], (pi - 1) & 1, abort_flag, kSiteQEmpty))) break;
          mbar_arrive_expect_tx(&sm.q_full[x], kTileBytes);
          tma_load_4d(sm.q[x], &tm_q, &sm.q_full[x], 0, h[x], qb[x] * kBlock, b[x]);
          tma_load_4d(sm.q[x] + kHalfBytes, &tm_q, &sm.q_full[x], 64, h[x], qb[x] * kBlock, b[x]);
        }
        // one ring slot per load, in the order the MMA issuer consumes them
        auto load = [&](const CUtensorMap* map, const int32_t* lst, int hh, int bb, int step) -> bool {
          const uint32_t st = rq % kRing, use = rq / kRing;
          if (use > 0 && !mbar_wait(&sm.ring_free[st], (use - 1) & 1, abort_flag, kSiteRingFree)) return false;
          const int blk = __ldg(lst + step);
          mbar_arrive_expect_tx(&sm.ring_full[st], kTileBytes);
          tma_load_4d(sm.ring[st], map, &sm.ring_full[st], 0, hh, blk * kBlock, bb);
          tma_load_4d(sm.ring[st] + kHalfBytes, map, &sm.ring_full[st], 64, hh, blk * kBlock, bb);
          ++rq;
          return true;
        };
        for (int j = 0; j <= p.topk && ok; ++j) {
          if (j < p.topk && !(ok = load(&tm_k, list[0], h[0], b[0], j))) break;        // K0(j)
          if (j >= 1 && !(ok = load(&tm_v, list[1], h[1], b[1], j - 1))) break;       // V1(j-1)
          if (j < p.topk && !(ok = load(&tm_k, list[1], h[1], b[1], j))) break;        // K1(j)
          if (j < p.topk && !(ok = load(&tm_v, list[0], h[0], b[0], j))) break;        // V0(j)
        }
      }
      // Before the CTA exits, every load issued must have landed.
      for (uint32_t st = 0; st < kRing; ++st)
        if (st < rq) {
          const uint32_t uses = (rq - st + kRing - 1) / kRing;
          mbar_wait(&sm.ring_full[st], (uses - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
        }
      if (pi > 0)
        for (int x = 0; x < 2; ++x) mbar_wait(&sm.q_full[x], (pi - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
    } else if (warp == 1 && lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, true);
      uint32_t rq = 0;
      int pi = 0;
      bool ok = true;
      for (int pr = blockIdx.x; pr < p.num_pairs && ok; pr += gridDim.x, ++pi) {
        const uint32_t g = static_cast<uint32_t>(pi) * p.topk;   // steps of each slot before this pair
        // S_x(step) = Q_x K^T over S_x, which still holds P_x(step-1): PV_x(step-1) must be done.
        auto issue_s = [&](int x, int step) -> bool {
          const uint32_t st = rq % kRing, ph = (rq / kRing) & 1;
          const uint32_t gg = g + step;
          if (step == 0 && !mbar_wait(&sm.q_full[x], pi & 1, abort_flag, kSiteQFull)) return false;
          if (gg > 0 && !mbar_wait(&sm.pv_done[x], (gg - 1) & 1, abort_flag, kSitePvDone)) return false;
          if (!mbar_wait(&sm.ring_full[st], ph, abort_flag, kSiteRingFull)) return false;
          tc_fence_after();
          const uint64_t qd = smem_desc_sw128(smem_addr(sm.q[x]), 16, 1024);
          const uint64_t kd = smem_desc_sw128(smem_addr(sm.ring[st]), 16, 1024);
          const uint32_t d = tmem + x * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) mma_ss(d, qd + kstep_off(kk), kd + kstep_off(kk), kIdescS, kk > 0 ? 1u : 0u);
          tc_commit(&sm.ring_free[st]);
          tc_commit(&sm.s_full[x]);
          if (step == p.topk - 1) tc_commit(&sm.q_empty[x]);
          ++rq;
          return true;
        };
        // O_x += P_x(step) V(step), P from the first 64 columns of S_x.
        auto issue_pv = [&](int x, int step) -> bool {
          const uint32_t st = rq % kRing, ph = (rq / kRing) & 1;
          const uint32_t gs = g + step;
          if (!mbar_wait(&sm.p_full[x], gs & 1, abort_flag, kSitePFull)) return false;
          if (step == 0 && pi > 0 && !mbar_wait(&sm.o_free[x], (pi - 1) & 1, abort_flag, kSiteOFree)) return false;
          if (!mbar_wait(&sm.ring_full[st], ph, abort_flag, kSiteRingFull)) return false;
          tc_fence_after();
          const uint64_t vd = smem_desc_sw128(smem_addr(sm.ring[st]), kHalfBytes, 1024);
          const uint32_t p_tm = tmem + x * 128;
          const uint32_t o_tm = tmem + 256 + x * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(o_tm, p_tm + kk * 8, vd + static_cast<uint32_t>(kk * 128), kIdescPV, (step > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&sm.ring_free[st]);
          tc_commit(&sm.pv_done[x]);
          ++rq;
          return true;
        };
        for (int j = 0; j <= p.topk && ok; ++j) {
          if (j < p.topk && !(ok = issue_s(0, j))) break;
          if (j >= 1 && !(ok = issue_pv(1, j - 1))) break;
          if (j < p.topk && !(ok = issue_s(1, j))) break;
          if (j < p.topk && !(ok = issue_pv(0, j))) break;
        }
      }
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, abort_flag, kSiteDrain, 200000000ull, false);
    }
  } else {
    warpgroup_regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax + epilogue of one slot
    const int x = (threadIdx.x >> 7) - 1;      // slot: warpgroup 1 -> 0, warpgroup 2 -> 1
    const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;          // query row inside the tile
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_addr = tmem + lane_off + x * 128;         // S_x, and P_x over its first 64 columns
    const uint32_t o_addr = tmem + lane_off + 256 + x * 128;   // O_x
    const int tail_valid = p.N - (p.nb - 1) * kBlock;          // valid keys in the last block
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    uint32_t g = 0;
    bool ok = true;
    for (int pr = blockIdx.x; pr < p.num_pairs && ok; pr += gridDim.x) {
      bool store;
      int b, h, qb;
      decode_tile(p, pair_tile(p, pr, x, store), b, h, qb);
      const int32_t* list = p.idx + (static_cast<size_t>(b * p.H + h) * p.nb + qb) * p.topk;
      float m = -INFINITY;   // running max in log2 units (possibly stale by < 2^8)
      float l = 0.f;         // running sum of exp2(x - m)
      int blk = __ldg(list);
      for (int j = 0; j < p.topk; ++j) {
        const uint32_t gg = g + j;
        const int blk_next = (j + 1 < p.topk) ? __ldg(list + j + 1) : 0;
        ok = mbar_wait(&sm.s_full[x], gg & 1, abort_flag, kSiteSFull);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld128_wait(s_addr, sr);
        if (blk == p.nb - 1 && tail_valid < kBlock) {
#pragma unroll
          for (int e = 0; e < 128; ++e)
            if (e >= tail_valid) sr[e] = __float_as_uint(-INFINITY);
        }
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
        uint32_t pk0[32], pk1[32];
        uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int e = 0; e < 128; e += 2) {
          float a0, a1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), scale2, neg_m2), a0, a1);
          const float p0 = ex2_approx(a0), p1 = ex2_approx(a1);
          acc[(e >> 1) & 3] = f2_add(acc[(e >> 1) & 3], f2_pack(p0, p1));
          if (e < 64) pk0[e >> 1] = pack_bf16x2(p0, p1);
          else pk1[(e - 64) >> 1] = pack_bf16x2(p0, p1);
        }
        float rs0, rs1, rs2, rs3;
        f2_unpack(f2_add(acc[0], acc[1]), rs0, rs1);
        f2_unpack(f2_add(acc[2], acc[3]), rs2, rs3);
        // P over the first 64 columns of S (their S values are in registers already)
        tmem_st32(s_addr, pk0);
        tmem_st32(s_addr + 32, pk1);
        if (j > 0 && __any_sync(0xffffffffu, rescale)) {
          // O holds the sum through PV(j-1); it must be complete before the rescale.
          ok = mbar_wait(&sm.pv_done[x], (gg - 1) & 1, abort_flag, kSitePvDone);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; tmem_wait_st(); break; }
          tc_fence_after();
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
        m = m_use;
        l += (rs0 + rs1) + (rs2 + rs3);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[x]);
        blk = blk_next;
      }
      if (!ok) break;
      // epilogue: O / l and LSE
      {
        const uint32_t last = g + p.topk - 1;
        ok = mbar_wait(&sm.pv_done[x], last & 1, abort_flag, kSitePvDone);
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t orr[128];
      tmem_ld128_wait(o_addr, orr);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free[x]);
      const int n = qb * kBlock + row;
      if (store && n < p.N) {
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

}  // namespace attnpp
}  // namespace sol
