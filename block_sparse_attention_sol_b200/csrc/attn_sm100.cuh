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
//   warps 2..9  softmax + epilogue, two warps per SM sub-partition: each warp
//               owns 16 TMEM lanes (query rows) and each thread two rows, a
//               quarter of the columns of each (the .16x256b layout), so one
//               warp's max/exp work overlaps the other's latency.  Each tile
//               starts by loading the Q rows from global memory into TMEM.
//               Online softmax in the exp2 domain with a lazy rescale (O is
//               rescaled only when the running max grows by more than 2^8); P
//               is written to TMEM as bf16 once PV of the previous step has
//               completed (single P buffer); epilogue O / l -> bf16 with
//               16-byte stores, and LSE.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P [384,448) Q [448,512).
// Shared memory: K 3 x 32 KB, V 3 x 32 KB.
//
// Descriptor note: the MMA descriptors are built once per call and each K-step
// adds a compile-time offset; building them per instruction measurably slows
// tcgen05.mma issue.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include "blocks.cuh"
#include "sm100_ptx.cuh"

namespace sol {
namespace attn100 {

constexpr int kBlock = 128;            // tokens per query / key block
constexpr int kHeadDim = 128;
constexpr int kSlots = 3;               // K/V ring: slot s holds K_s and V_{s-2} of a tile
constexpr int kTileBytes = kBlock * kHeadDim * 2;   // 32 KB bf16 tile
constexpr int kHalfBytes = kTileBytes / 2;          // one 64-column swizzled box
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 64 + 32 * kSoftmaxWarps;   // producer, MMA, 8 softmax warps
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384, kColQ = 448;
constexpr float kRescaleLog2 = 8.0f;   // lazy-rescale threshold (log2 units)
// Of every 8 exponentials, this many run as a polynomial on the FMA pipe
// instead of on MUFU (16 results per clock per SM).
constexpr int kPolyPer8 = 0;

struct __align__(1024) Smem {
  uint8_t k[kSlots][kTileBytes];
  uint8_t v[kSlots][kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t kv_full[kSlots];     // the slot's K and/or V tile has landed
  uint64_t slot_done[kSlots];   // every MMA reading the slot is complete (for a K slot: S_s readable)
  uint64_t pv_done;             // PV of the step complete: P writable, O updated
  uint64_t p_full, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  const __nv_bfloat16* q; // [B, N, H, D]
  const int32_t* idx;     // [B, H, nb, topk]
  const int32_t* counts;  // [B, H, nb] blocks used per row (clamped to [1, topk]), or null: topk
  __nv_bfloat16* o;       // [B, N, H, D]
  float* lse;             // [B, H, N]
  int B, N, H, nb, topk;
  int num_tiles;
  float scale_log2;       // softmax scale * log2(e)
  BlockMap bm;            // token blocks (block == kBlock); tiled: K/V maps are 5-D (c, h, x, y, b * T + t)
  int T;                  // frames of the grid
};

// Wait-site ids reported in the error info word.
enum : unsigned { kSiteQEmpty = 1, kSiteSlotFree, kSiteQFull, kSiteSlotFull, kSitePFull, kSiteOFree, kSiteSDone,
                  kSitePvDone, kSiteDrain, kSiteTail };

// K-step offsets (16-byte units) inside a 128-byte-swizzled K-major tile: 16
// channels = 32 bytes per step, the second 64-channel box 16 KB further.
__device__ __forceinline__ constexpr uint32_t kstep_off(int kk) {
  return static_cast<uint32_t>(((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4);
}

// Key blocks of tile t (row t of idx in [B, H, nb] order); every role reads the same value.
__device__ __forceinline__ int tile_steps(const Params& p, int t) {
  return p.counts == nullptr ? p.topk : min(max(__ldg(p.counts + t), 1), p.topk);
}

// Both 64-channel halves of key block `blk` of (b, h) into a slot: one 4-D box of
// 128 consecutive tokens, or one 5-D box of a tt x th x tw tile (rows in the
// same tile-raster order as block_token).
__device__ __forceinline__ void load_block(uint8_t* dst, const CUtensorMap* tm, uint64_t* bar, const Params& p, int blk,
                                           int h, int b) {
  if (p.bm.tw == 0) {
    tma_load_4d(dst, tm, bar, 0, h, blk * kBlock, b);
    tma_load_4d(dst + kHalfBytes, tm, bar, 64, h, blk * kBlock, b);
  } else {
    int t0, y0, x0;
    tile_origin(p.bm, blk, t0, y0, x0);
    tma_load_5d(dst, tm, bar, 0, h, x0, y0, b * p.T + t0);
    tma_load_5d(dst + kHalfBytes, tm, bar, 64, h, x0, y0, b * p.T + t0);
  }
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
    mbar_init(&sm.q_full, kSoftmaxWarps);   // one arrival per softmax warp
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kSlots; ++s) { mbar_init(&sm.kv_full[s], 1); mbar_init(&sm.slot_done[s], 1); }
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.p_full, kSoftmaxWarps);
    mbar_init(&sm.o_free, kSoftmaxWarps);
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
      uint32_t sq = 0;   // slots filled so far
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int b, h, qb;
        decode_tile(p, t, b, h, qb);
        const int32_t* list = p.idx + (static_cast<size_t>(b * p.H + h) * p.nb + qb) * p.topk;
        const int kt = tile_steps(p, t);
        // slot s of the tile: K_s (s < kt) and V_{s-2} (s >= 2), in the order the MMA issuer uses them
        for (int s = 0; s < kt + 2; ++s, ++sq) {
          const uint32_t st = sq % kSlots, use = sq / kSlots;
          if (use > 0 && !(ok = mbar_wait(&sm.slot_done[st], (use - 1) & 1, abort_flag, kSiteSlotFree))) break;
          const bool has_k = s < kt, has_v = s >= 2;
          mbar_arrive_expect_tx(&sm.kv_full[st], (has_k ? kTileBytes : 0) + (has_v ? kTileBytes : 0));
          if (has_k) {
            const int id = __ldg(list + s);
            if (static_cast<unsigned>(id) >= static_cast<unsigned>(p.nb)) raise_bad_arg();
            load_block(sm.k[st], &tm_k, &sm.kv_full[st], p, usable_block(id, p.nb), h, b);
          }
          if (has_v) load_block(sm.v[st], &tm_v, &sm.kv_full[st], p, usable_block(__ldg(list + s - 2), p.nb), h, b);
        }
      }
      // Before the CTA exits, every load issued must have landed (slot s was
      // filled for the fills s, s + 3, ...; wait for the phase of its last one).
      for (uint32_t st = 0; st < kSlots; ++st)
        if (st < sq) {
          const uint32_t uses = (sq - st + kSlots - 1) / kSlots;
          mbar_wait(&sm.kv_full[st], (uses - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // tcgen05.mma issue runs only a couple of instructions ahead of execution,
    // so the tensor pipe idles whenever this thread waits or does bookkeeping.
    // Each step therefore has one wait point: P_j ready and slot j + 2 (V_j and
    // K_{j+2}) landed; then PV_j and S_{j+2} go out back to back.  S runs two
    // steps ahead of PV, so the softmax of step j + 1 finds S_{j+1} complete.
    if (lane == 0) {
      constexpr uint32_t kIdescS = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, true);
      const uint32_t q_tm = tmem + kColQ;
      const uint32_t p_tm = tmem + kColP;
      const uint32_t o_tm = tmem + kColO;
      uint32_t g = 0;    // steps (S / PV pairs) before this tile
      uint32_t sq = 0;   // slots before this tile
      int it = 0;
      bool ok = true;
      // S(gg) = Q K^T into S[gg % 2] from slot stage st.  The buffer was last
      // read by the softmax of step gg - 2, which arrived on p_full before
      // PV(gg - 2), and with it S(gg), was issued.
      auto mma_s = [&](uint32_t gg, uint32_t st) {
        const uint64_t kd = smem_desc_sw128(smem_addr(sm.k[st]), 16, 1024);
        const uint32_t d = tmem + kColS + (gg & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) mma_ts(d, q_tm + kk * 8, kd + kstep_off(kk), kIdescS, kk > 0 ? 1u : 0u);
      };
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
        if (!(ok = mbar_wait(&sm.q_full, it & 1, abort_flag, kSiteQFull))) break;
        const int kt = tile_steps(p, t);
        // slots 0 and 1 of the tile: K_0 and K_1 (slot 1 is empty when kt = 1)
        for (int s = 0; s < 2 && ok; ++s) {
          const uint32_t sl = sq + s, st = sl % kSlots;
          if (!(ok = mbar_wait(&sm.kv_full[st], (sl / kSlots) & 1, abort_flag, kSiteSlotFull))) break;
          tc_fence_after();
          if (s < kt) mma_s(g + s, st);
          tc_commit(&sm.slot_done[st]);
        }
        if (!ok) break;
        if (kt <= 2) tc_commit(&sm.q_empty);   // every S MMA of this tile has been issued
        for (int j = 0; j < kt; ++j) {
          const uint32_t gg = g + j, sl = sq + j + 2, st = sl % kSlots;
          if (!(ok = mbar_wait(&sm.p_full, gg & 1, abort_flag, kSitePFull))) break;
          if (j == 0 && it > 0 && !(ok = mbar_wait(&sm.o_free, (it - 1) & 1, abort_flag, kSiteOFree))) break;
          if (!(ok = mbar_wait(&sm.kv_full[st], (sl / kSlots) & 1, abort_flag, kSiteSlotFull))) break;
          tc_fence_after();
          const uint64_t vd = smem_desc_sw128(smem_addr(sm.v[st]), kHalfBytes, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: P columns kk*8.., V rows kk*16.. (2 KB)
            mma_ts(o_tm, p_tm + kk * 8, vd + static_cast<uint32_t>(kk * 128), kIdescPV,
                   (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&sm.pv_done);
          if (j + 2 < kt) mma_s(gg + 2, st);
          tc_commit(&sm.slot_done[st]);
          if (j + 3 == kt) tc_commit(&sm.q_empty);
        }
        g += kt;
        sq += kt + 2;
      }
      // Drain: every MMA issued must complete before TMEM is released.
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, abort_flag, kSiteDrain, 200000000ull, false);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Warp w owns the 16 TMEM lanes quad*32 + half*16 .. +15 of its lane
    // quadrant (quad = w % 4, the quadrant it may access).  Thread 4r + c holds
    // rows r and r + 8 of them, columns 8i + 2c and 8i + 2c + 1 of each (the
    // .16x256b layout), so four threads share a row and a row max costs two
    // shuffles.  P goes back with the .16x128b layout: column 4i + c of a row
    // is the bf16 pair of keys 8i + 2c, 8i + 2c + 1, which this thread holds.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = lane >> 2, c4 = lane & 3;
    const int row0 = quad * 32 + half * 16 + r;    // this thread's rows: row0 and row0 + 8
    const uint32_t lanes16 = static_cast<uint32_t>(quad * 32 + half * 16) << 16;
    const uint32_t lanes32 = static_cast<uint32_t>(quad * 32) << 16;
    const int tail_valid = p.N - (p.nb - 1) * kBlock;   // valid keys in the last block
    const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
    // This thread's 64 Q channels (one row of its quadrant) of tile tt, as bf16 pairs.
    auto load_q_rows = [&](int tt, uint32_t (&qv)[32]) {
      int tb, th, tq;
      decode_tile(p, tt, tb, th, tq);
      const int nq = block_token(p.bm, tq, quad * 32 + lane);
      if (nq < p.N) {
        const uint4* src = reinterpret_cast<const uint4*>(
            p.q + ((static_cast<size_t>(tb) * p.N + nq) * p.H + th) * kHeadDim + 64 * half);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint4 w = __ldg(src + c);
          qv[4 * c] = w.x; qv[4 * c + 1] = w.y; qv[4 * c + 2] = w.z; qv[4 * c + 3] = w.w;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) qv[c] = 0u;
      }
    };
    auto store_q = [&](const uint32_t (&qv)[32]) {
      tmem_st32(tmem + lanes32 + kColQ + 32 * half, qv);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_full);
    };
    uint32_t g = 0;    // steps before this tile
    uint32_t sq = 0;   // K/V slots before this tile (topk + 2 per tile)
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
      int b, h, qb;
      decode_tile(p, t, b, h, qb);
      const int32_t* list = p.idx + (static_cast<size_t>(b * p.H + h) * p.nb + qb) * p.topk;
      const int kt = tile_steps(p, t);
      // ---- Q into TMEM (A operand of the S MMAs: lane = row, 2 bf16 per column).
      // The two warps of a quadrant write channels [64 half, 64 half + 64) of its 32
      // rows.  The first tile's Q is stored here; each later tile's Q is loaded during
      // the previous tile's epilogue, so that its first S products overlap that epilogue.
      if (it == 0) {
        uint32_t qv[32];
        load_q_rows(t, qv);
        store_q(qv);
      }
      float m0 = -INFINITY, m1 = -INFINITY;   // running max per row, log2 units (stale by < 2^8)
      float l0 = 0.f, l1 = 0.f;               // this thread's part of the running sums
      int blk = usable_block(__ldg(list), p.nb);
      for (int j = 0; j < kt; ++j) {
        const uint32_t gg = g + j;
        const uint32_t buf = gg & 1;
        const int blk_next = (j + 1 < kt) ? usable_block(__ldg(list + j + 1), p.nb) : 0;
        const uint32_t sl = sq + j;   // slot of K_j: its slot_done also means S_j is complete
        ok = mbar_wait(&sm.slot_done[sl % kSlots], (sl / kSlots) & 1, abort_flag, kSiteSDone);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];   // row0: sr[4i], sr[4i+1]; row0 + 8: sr[4i+2], sr[4i+3]; keys 8i + 2c4 + {0,1}
        tmem_ld16x256b_x16_wait(tmem + lanes16 + kColS + buf * 128, sr);
        if (blk == p.nb - 1 && tail_valid < kBlock) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (8 * i + 2 * c4 + (e & 1) >= tail_valid) sr[4 * i + e] = __float_as_uint(-INFINITY);
        }
        // row max: two chains per row, then across the four threads of the row
        float pm[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pm[e] = fmaxf(__uint_as_float(sr[e]), __uint_as_float(sr[4 + e]));
#pragma unroll
          for (int i = 2; i < 16; i += 2)
            pm[e] = fmax3(pm[e], __uint_as_float(sr[4 * i + e]), __uint_as_float(sr[4 * i + 4 + e]));
        }
        float mx0 = fmaxf(pm[0], pm[1]), mx1 = fmaxf(pm[2], pm[3]);
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2)) * p.scale_log2;
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2)) * p.scale_log2;
        const bool rs0 = mx0 > m0 + kRescaleLog2, rs1 = mx1 > m1 + kRescaleLog2;
        const float mu0 = rs0 ? mx0 : m0, mu1 = rs1 ? mx1 : m1;
        const uint64_t nm0 = f2_pack(-mu0, -mu0), nm1 = f2_pack(-mu1, -mu1);
        // P = exp2(s * scale - m) as bf16 pairs; two partial sums per row
        uint32_t pk[32];
        uint64_t acc0[2] = {0ull, 0ull}, acc1[2] = {0ull, 0ull};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[4 * i]), __uint_as_float(sr[4 * i + 1])), scale2, nm0), x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[4 * i + 2]), __uint_as_float(sr[4 * i + 3])), scale2, nm1), x2,
                    x3);
          float p0, p1, p2, p3;
          if ((i & 7) >= 8 - kPolyPer8) {
            exp2_poly_pair(x0, x1, p0, p1);   // FMA pipe
            exp2_poly_pair(x2, x3, p2, p3);
          } else {
            p0 = ex2_approx(x0);              // MUFU
            p1 = ex2_approx(x1);
            p2 = ex2_approx(x2);
            p3 = ex2_approx(x3);
          }
          acc0[i & 1] = f2_add(acc0[i & 1], f2_pack(p0, p1));
          acc1[i & 1] = f2_add(acc1[i & 1], f2_pack(p2, p3));
          pk[2 * i] = pack_bf16x2(p0, p1);
          pk[2 * i + 1] = pack_bf16x2(p2, p3);
        }
        float s0a, s0b, s1a, s1b;
        f2_unpack(f2_add(acc0[0], acc0[1]), s0a, s0b);
        f2_unpack(f2_add(acc1[0], acc1[1]), s1a, s1b);
        if (j > 0) {
          // PV of the previous step must be done before P is overwritten and O rescaled.
          ok = mbar_wait(&sm.pv_done, (gg - 1) & 1, abort_flag, kSitePvDone);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
        }
        tmem_st16x128b_x16(tmem + lanes16 + kColP, pk);   // 128 keys -> 64 columns of bf16 pairs
        // O is rescaled after P is stored (P's registers are free by then) and
        // before p_full, which is what lets the next PV accumulate into O.
        if (j > 0) {
          if (__any_sync(0xffffffffu, rs0 || rs1)) {
            const float al0 = rs0 ? ex2_approx(m0 - mu0) : 1.f;
            const float al1 = rs1 ? ex2_approx(m1 - mu1) : 1.f;
            const uint64_t a0 = f2_pack(al0, al0), a1 = f2_pack(al1, al1);
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {   // O columns [64 hc, 64 hc + 64)
              uint32_t orr[32];
              tmem_ld16x256b_x8_wait(tmem + lanes16 + kColO + 64 * hc, orr);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                float o0, o1, o2, o3;
                f2_unpack(f2_mul(f2_pack(__uint_as_float(orr[4 * i]), __uint_as_float(orr[4 * i + 1])), a0), o0, o1);
                f2_unpack(f2_mul(f2_pack(__uint_as_float(orr[4 * i + 2]), __uint_as_float(orr[4 * i + 3])), a1), o2,
                          o3);
                orr[4 * i] = __float_as_uint(o0);
                orr[4 * i + 1] = __float_as_uint(o1);
                orr[4 * i + 2] = __float_as_uint(o2);
                orr[4 * i + 3] = __float_as_uint(o3);
              }
              tmem_st16x256b_x8(tmem + lanes16 + kColO + 64 * hc, orr);
            }
            l0 *= al0;
            l1 *= al1;
          }
        }
        m0 = mu0;
        m1 = mu1;
        l0 += s0a + s0b;
        l1 += s1a + s1b;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
        blk = blk_next;
      }
      if (!ok) break;
      // The next tile's Q: global loads issued now, stored into TMEM once this
      // tile's O has been read below (its S products are complete by then: every
      // S of this tile has been consumed).
      const int t_next = t + gridDim.x;
      uint32_t qn[32];
      if (t_next < p.num_tiles) load_q_rows(t_next, qn);
      // epilogue: O / l and LSE
      {
        ok = mbar_wait(&sm.pv_done, (g + kt - 1) & 1, abort_flag, kSitePvDone);
      }
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      const float inv0 = 1.f / l0, inv1 = 1.f / l1;
      const uint64_t i0 = f2_pack(inv0, inv0), i1 = f2_pack(inv1, inv1);
      uint32_t ob[2][16];   // bf16 pairs of O / l: row u, channels 8i + 2c4, 8i + 2c4 + 1
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        uint32_t orr[32];
        tmem_ld16x256b_x8_wait(tmem + lanes16 + kColO + 64 * hc, orr);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float o0, o1, o2, o3;
          f2_unpack(f2_mul(f2_pack(__uint_as_float(orr[4 * i]), __uint_as_float(orr[4 * i + 1])), i0), o0, o1);
          f2_unpack(f2_mul(f2_pack(__uint_as_float(orr[4 * i + 2]), __uint_as_float(orr[4 * i + 3])), i1), o2, o3);
          ob[0][8 * hc + i] = pack_bf16x2(o0, o1);
          ob[1][8 * hc + i] = pack_bf16x2(o2, o3);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free);
      if (t_next < p.num_tiles) {
        ok = mbar_wait(&sm.q_empty, it & 1, abort_flag, kSiteQEmpty);   // this tile's S MMAs done
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        store_q(qn);
      }
      // The four threads of a row hold its channel pairs 8i + 2c (thread c); a 4 x 4
      // exchange per group of four i gives thread c the 16 contiguous bytes of
      // channels 8 (4a + c) .. + 7, which it stores in one instruction.
      uint4 seg[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          uint32_t got[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {   // round k: send pair 4a + (c4 - k) & 3, receive from thread (c4 + k) & 3
            const int sidx = (c4 - k) & 3;
            const uint32_t send = sidx == 0 ? ob[u][4 * a] : sidx == 1 ? ob[u][4 * a + 1]
                                : sidx == 2 ? ob[u][4 * a + 2] : ob[u][4 * a + 3];
            got[k] = __shfl_sync(0xffffffffu, send, (lane & ~3) | ((c4 + k) & 3));
          }
          // got[k] is the pair of channels 8 (4a + c4) + 2 ((c4 + k) & 3): put it in place
          uint32_t w[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int k = (c - c4) & 3;
            w[c] = k == 0 ? got[0] : k == 1 ? got[1] : k == 2 ? got[2] : got[3];
          }
          seg[u][a] = make_uint4(w[0], w[1], w[2], w[3]);
        }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int n = block_token(p.bm, qb, row0 + 8 * u);
        if (n < p.N) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kHeadDim);
#pragma unroll
          for (int a = 0; a < 4; ++a) dst[4 * a + c4] = seg[u][a];
          if (c4 == 0)
            p.lse[(static_cast<size_t>(b) * p.H + h) * p.N + n] =
                ((u ? m1 : m0) + __log2f(u ? l1 : l0)) * 0.69314718055994531f;
        }
      }
      g += kt;
      sq += kt + 2;
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
