// Block-sparse attention forward with FP8 (e4m3) operands on sm_100a tensor cores.
//
// The Sol-H3 runtime uses FP8 on its hot paths (ai-feiten.nl, "Videomodel
// MiniMax-H3 rendert sneller dan afspelen", section "Waar de snelheidswinst
// vandaan komt"); this is the FP8 variant of the Sol-Attn kernel in
// attn_sm100.cuh: the same definition, computed on the dequantised inputs
//     q = qc * sq[row],  k = kc * sk[block],  v = vc * sv[head]
// (codes e4m3, scales fp32), with tcgen05.mma kind::f8f6f4 (K = 32 per
// instruction, twice the bf16 rate) for both products:
//   S_j = Qc Kc_j^T                          (Qc in TMEM, Kc_j in shared memory)
//   l   = scale * sq[i] * sk[j] * S_im        (one factor per row and step in the softmax)
//   O  += Pc_j Vc_j                           (P rounded to e4m3 in TMEM, Vc^T in shared memory)
//   O   = sv * O / sum(P)
// P is formed as 2^(l - m + 6) with a lazy rescale threshold of 2.5 (log2
// units), so it stays within e4m3's range (<= 2^8.5 < 448) while values down to
// 2^-12 of the running maximum keep full e4m3 precision (subnormal to 2^-15).
// (Offset 8 with threshold 0.5 kept more of the small weights but rescaled O in
// TMEM on most early steps of a row and ran 40% slower than the bf16 kernel.)  The sum uses the fp32
// P; the e4m3 rounding of P (relative 2^-4 at most) is the kernel's only
// approximation beyond fp32 accumulation order.
//
// Layouts: Qc, Kc [B, N, H, D] e4m3; sq [B, H, N], sk [B, H, nb] fp32; Vc^T [B, H, D, N]
// e4m3 with the keys of every aligned group of 16 stored in the order
// 0 1 8 9 2 3 10 11 4 5 12 13 6 7 14 15 (so that each softmax thread builds
// whole TMEM columns of P from the keys it holds, without shuffles); sv [B, H].
// N % 16 == 0 (TMA row strides), D == 128, blocks of 128 consecutive tokens.
//
// Roles as in attn_sm100.cuh: warp 0 TMA producer, warp 1 MMA issuer, warps
// 2..9 softmax (16 TMEM lanes each, two rows per thread).  The block's K scale is
// one global load per step, folded into the per-row factor.
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P [384,416) Q [416,448).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include "sm100_ptx.cuh"

namespace sol {
namespace attnfp8 {

constexpr int kBlock = 128;
constexpr int kHeadDim = 128;
constexpr int kSlots = 3;                         // slot s holds K_s and V_{s-2} of a tile
constexpr int kTileBytes = kBlock * kHeadDim;     // 16 KB e4m3 tile
constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 64 + 32 * kSoftmaxWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 384, kColQ = 416;
constexpr float kRescaleLog2 = 2.5f;              // lazy-rescale threshold (log2 units)
constexpr float kPOffsetLog2 = 6.0f;              // P = 2^(x - m + 6) <= 2^8.5 < 448
// Of every 8 exponentials, this many run as a polynomial on the FMA pipe instead
// of on MUFU (16 results per clock per SM, the bound once the FP8 MMAs take half
// the bf16 time).
constexpr int kPolyPer8 = 2;

struct __align__(1024) Smem {
  uint8_t k[kSlots][kTileBytes];
  uint8_t v[kSlots][kTileBytes];
  uint64_t q_full, q_empty;
  uint64_t kv_full[kSlots];
  uint64_t slot_done[kSlots];
  uint64_t pv_done;
  uint64_t p_full, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

struct Params {
  const uint8_t* q;        // [B, N, H, D] e4m3 codes
  const float* q_scale;    // [B, H, N]
  const float* k_scale;    // [B, H, nb]
  const float* v_scale;    // [B, H]
  const int32_t* idx;      // [B, H, nb, topk]
  const int32_t* counts;   // [B, H, nb] or null
  __nv_bfloat16* o;        // [B, N, H, D]
  float* lse;              // [B, H, N]
  int B, N, H, nb, topk;
  int num_tiles;
  float scale_log2;        // softmax scale * log2(e)
};

enum : unsigned { kSiteQEmpty = 1, kSiteSlotFree, kSiteQFull, kSiteSlotFull, kSitePFull, kSiteOFree, kSiteSDone,
                  kSitePvDone, kSiteDrain, kSiteTail };

// kind::f8f6f4, e4m3 A and B, fp32 accumulator, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (0u << 7)                                 // A format: e4m3
         | (0u << 10)                                // B format: e4m3
         | (static_cast<uint32_t>(N >> 3) << 17)
         | (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_addr(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_addr(bar))
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp writes lane (base + i).
__device__ __forceinline__ void tmem_st32x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// 16 lanes x 32 columns in the .16x128b shape: thread 4r + q writes lane r
// (registers 2i) and lane r + 8 (registers 2i + 1) of column 4i + q.
__device__ __forceinline__ void tmem_st16x128b_x8(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Two fp32 values as an e4m3 pair (lo in the low byte), round to nearest even, saturating.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ int tile_steps(const Params& p, int t) {
  return p.counts == nullptr ? p.topk : min(max(__ldg(p.counts + t), 1), p.topk);
}

__device__ __forceinline__ void decode_tile(const Params& p, int t, int& b, int& h, int& qb) {
  qb = t % p.nb;
  const int bh = t / p.nb;
  h = bh % p.H;
  b = bh / p.H;
}


__global__ void __launch_bounds__(kThreads, 1)
sparse_attn_fp8_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_vt,
                       const Params p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    sm.abort_flag = 0;
    mbar_init(&sm.q_full, kSoftmaxWarps);
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
      tma_prefetch_desc(&tm_vt);
      uint32_t sq = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x) {
        int b, h, qb;
        decode_tile(p, t, b, h, qb);
        const int32_t* list = p.idx + (static_cast<size_t>(b * p.H + h) * p.nb + qb) * p.topk;
        const int kt = tile_steps(p, t);
        for (int s = 0; s < kt + 2; ++s, ++sq) {
          const uint32_t st = sq % kSlots, use = sq / kSlots;
          if (use > 0 && !(ok = mbar_wait(&sm.slot_done[st], (use - 1) & 1, abort_flag, kSiteSlotFree))) break;
          const bool has_k = s < kt, has_v = s >= 2;
          mbar_arrive_expect_tx(&sm.kv_full[st], (has_k ? kTileBytes : 0) + (has_v ? kTileBytes : 0));
          if (has_k) {
            const int id = __ldg(list + s);
            if (static_cast<unsigned>(id) >= static_cast<unsigned>(p.nb)) raise_bad_arg();
            tma_load_4d(sm.k[st], &tm_k, &sm.kv_full[st], 0, h, usable_block(id, p.nb) * kBlock, b);
          }
          if (has_v)
            tma_load_3d(sm.v[st], &tm_vt, &sm.kv_full[st], usable_block(__ldg(list + s - 2), p.nb) * kBlock, 0,
                        b * p.H + h);
        }
      }
      for (uint32_t st = 0; st < kSlots; ++st)
        if (st < sq) {
          const uint32_t uses = (sq - st + kSlots - 1) / kSlots;
          mbar_wait(&sm.kv_full[st], (uses - 1) & 1, abort_flag, kSiteTail, 200000000ull, false);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // As in the bf16 kernel: one wait point per step (P_j ready and slot j + 2
    // landed), then PV_j and S_{j+2} back to back; 4 MMAs of K = 32 per product.
    if (lane == 0) {
      constexpr uint32_t kIdesc = idesc_e4m3_f32(128, 128);
      const uint32_t q_tm = tmem + kColQ;
      const uint32_t p_tm = tmem + kColP;
      const uint32_t o_tm = tmem + kColO;
      uint32_t g = 0, sq = 0;
      int it = 0;
      bool ok = true;
      auto mma_s = [&](uint32_t gg, uint32_t st) {
        const uint64_t kd = smem_desc_sw128(smem_addr(sm.k[st]), 16, 1024);
        const uint32_t d = tmem + kColS + (gg & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) mma_ts_f8(d, q_tm + kk * 8, kd + 2 * kk, kIdesc, kk > 0 ? 1u : 0u);
      };
      for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
        if (!(ok = mbar_wait(&sm.q_full, it & 1, abort_flag, kSiteQFull))) break;
        const int kt = tile_steps(p, t);
        for (int s = 0; s < 2 && ok; ++s) {
          const uint32_t sl = sq + s, st = sl % kSlots;
          if (!(ok = mbar_wait(&sm.kv_full[st], (sl / kSlots) & 1, abort_flag, kSiteSlotFull))) break;
          tc_fence_after();
          if (s < kt) mma_s(g + s, st);
          tc_commit(&sm.slot_done[st]);
        }
        if (!ok) break;
        if (kt <= 2) tc_commit(&sm.q_empty);
        for (int j = 0; j < kt; ++j) {
          const uint32_t gg = g + j, sl = sq + j + 2, st = sl % kSlots;
          if (!(ok = mbar_wait(&sm.p_full, gg & 1, abort_flag, kSitePFull))) break;
          if (j == 0 && it > 0 && !(ok = mbar_wait(&sm.o_free, (it - 1) & 1, abort_flag, kSiteOFree))) break;
          if (!(ok = mbar_wait(&sm.kv_full[st], (sl / kSlots) & 1, abort_flag, kSiteSlotFull))) break;
          tc_fence_after();
          const uint64_t vd = smem_desc_sw128(smem_addr(sm.v[st]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // 32 keys per MMA: P columns kk*8.., V^T bytes kk*32..
            mma_ts_f8(o_tm, p_tm + kk * 8, vd + 2 * kk, kIdesc, (j > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&sm.pv_done);
          if (j + 2 < kt) mma_s(gg + 2, st);
          tc_commit(&sm.slot_done[st]);
          if (j + 3 == kt) tc_commit(&sm.q_empty);
        }
        g += kt;
        sq += kt + 2;
      }
      tc_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, abort_flag, kSiteDrain, 200000000ull, false);
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Thread 4r + c4 of a warp holds rows row0, row0 + 8 and keys 8i + 2c4, +1
    // (i < 16) of S (.16x256b).  P goes back with .16x128b: column 4m + c4 of a
    // row holds keys 16m + 2c4, +1, 16m + 8 + 2c4, +1 (this thread's keys of
    // i = 2m and 2m + 1), the order V^T is stored in.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int r = lane >> 2, c4 = lane & 3;
    const int row0 = quad * 32 + half * 16 + r;
    const uint32_t lanes16 = static_cast<uint32_t>(quad * 32 + half * 16) << 16;
    const uint32_t lanes32 = static_cast<uint32_t>(quad * 32) << 16;
    const int tail_valid = p.N - (p.nb - 1) * kBlock;
    // This thread's 64 Q codes (one row of its quadrant) of tile tt.
    auto load_q_rows = [&](int tt, uint32_t (&qv)[16]) {
      int tb, th, tq;
      decode_tile(p, tt, tb, th, tq);
      const int nq = tq * kBlock + quad * 32 + lane;
      if (nq < p.N) {
        const uint4* src = reinterpret_cast<const uint4*>(
            p.q + ((static_cast<size_t>(tb) * p.N + nq) * p.H + th) * kHeadDim + 64 * half);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint4 w = __ldg(src + c);
          qv[4 * c] = w.x; qv[4 * c + 1] = w.y; qv[4 * c + 2] = w.z; qv[4 * c + 3] = w.w;
        }
      } else {
#pragma unroll
        for (int c = 0; c < 16; ++c) qv[c] = 0u;
      }
    };
    auto store_q = [&](const uint32_t (&qv)[16]) {
      tmem_st32x16(tmem + lanes32 + kColQ + 16 * half, qv);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_full);
    };
    uint32_t g = 0, sq = 0;
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.num_tiles && ok; t += gridDim.x, ++it) {
      int b, h, qb;
      decode_tile(p, t, b, h, qb);
      const int32_t* list = p.idx + (static_cast<size_t>(b * p.H + h) * p.nb + qb) * p.topk;
      const float* ksc = p.k_scale + static_cast<size_t>(b * p.H + h) * p.nb;
      const int kt = tile_steps(p, t);
      // Qc rows into TMEM: lane = row, 4 codes per column; the two warps of a quadrant
      // write channels [64 half, 64 half + 64) = 16 columns each.  The first tile's
      // Q is stored here; each later tile's Q is loaded during the previous tile's
      // epilogue, so that its first S products overlap that epilogue.
      if (it == 0) {
        uint32_t qv[16];
        load_q_rows(t, qv);
        store_q(qv);
      }
      // per-row factor scale * log2(e) * sq[row]
      float rf0 = 0.f, rf1 = 0.f;
      {
        const int n0 = qb * kBlock + row0, n1 = n0 + 8;
        const float* qsc = p.q_scale + static_cast<size_t>(b * p.H + h) * p.N;
        if (n0 < p.N) rf0 = p.scale_log2 * __ldg(qsc + n0);
        if (n1 < p.N) rf1 = p.scale_log2 * __ldg(qsc + n1);
      }
      float m0 = -INFINITY, m1 = -INFINITY;
      float l0 = 0.f, l1 = 0.f;
      for (int j = 0; j < kt; ++j) {
        const uint32_t gg = g + j;
        const uint32_t buf = gg & 1;
        const int blk = usable_block(__ldg(list + j), p.nb);
        const float ksb = __ldg(ksc + blk);   // the block's K scale
        const uint32_t sl = sq + j;
        ok = mbar_wait(&sm.slot_done[sl % kSlots], (sl / kSlots) & 1, abort_flag, kSiteSDone);
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld16x256b_x16_wait(tmem + lanes16 + kColS + buf * 128, sr);
        // keys beyond N masked
        if (blk == p.nb - 1 && tail_valid < kBlock) {
#pragma unroll
          for (int i = 0; i < 16; ++i)
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (8 * i + 2 * c4 + (e & 1) >= tail_valid) sr[4 * i + e] = __float_as_uint(-INFINITY);
        }
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
        const float rs0f = rf0 * ksb, rs1f = rf1 * ksb;   // this step's row factors
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2)) * rs0f;
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2)) * rs1f;
        const bool rs0 = mx0 > m0 + kRescaleLog2, rs1 = mx1 > m1 + kRescaleLog2;
        const float mu0 = rs0 ? mx0 : m0, mu1 = rs1 ? mx1 : m1;
        const uint64_t nm0 = f2_pack(kPOffsetLog2 - mu0, kPOffsetLog2 - mu0);
        const uint64_t nm1 = f2_pack(kPOffsetLog2 - mu1, kPOffsetLog2 - mu1);
        const uint64_t f0 = f2_pack(rs0f, rs0f), f1 = f2_pack(rs1f, rs1f);
        // P = 2^(s * rf - m + 6): fp32 sums, e4m3 words for TMEM
        uint32_t pw[16];
        uint64_t acc0[2] = {0ull, 0ull}, acc1[2] = {0ull, 0ull};
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1, x2, x3;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[4 * i]), __uint_as_float(sr[4 * i + 1])), f0, nm0), x0, x1);
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[4 * i + 2]), __uint_as_float(sr[4 * i + 3])), f1, nm1), x2, x3);
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
          // i = 2m: low half of column 4m + c4; i = 2m + 1: high half
          const uint32_t sh = (i & 1) ? 16u : 0u;
          if ((i & 1) == 0) { pw[i] = 0u; pw[i + 1] = 0u; }
          pw[(i & ~1)] |= pack_e4m3x2(p0, p1) << sh;
          pw[(i & ~1) + 1] |= pack_e4m3x2(p2, p3) << sh;
        }
        float s0a, s0b, s1a, s1b;
        f2_unpack(f2_add(acc0[0], acc0[1]), s0a, s0b);
        f2_unpack(f2_add(acc1[0], acc1[1]), s1a, s1b);
        if (j > 0) {
          ok = mbar_wait(&sm.pv_done, (gg - 1) & 1, abort_flag, kSitePvDone);
          if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
          tc_fence_after();
        }
        tmem_st16x128b_x8(tmem + lanes16 + kColP, pw);   // 128 keys -> 32 columns of e4m3 quads
        if (j > 0) {
          if (__any_sync(0xffffffffu, rs0 || rs1)) {
            const float al0 = rs0 ? ex2_approx(m0 - mu0) : 1.f;
            const float al1 = rs1 ? ex2_approx(m1 - mu1) : 1.f;
            const uint64_t a0 = f2_pack(al0, al0), a1 = f2_pack(al1, al1);
#pragma unroll
            for (int hc = 0; hc < 2; ++hc) {
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
      }
      if (!ok) break;
      // The next tile's Q: loads issued now, stored once this tile's O has been read.
      const int t_next = t + gridDim.x;
      uint32_t qn[16];
      if (t_next < p.num_tiles) load_q_rows(t_next, qn);
      ok = mbar_wait(&sm.pv_done, (g + kt - 1) & 1, abort_flag, kSitePvDone);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      const float sv = __ldg(p.v_scale + b * p.H + h);
      const float inv0 = sv / l0, inv1 = sv / l1;
      const uint64_t i0 = f2_pack(inv0, inv0), i1 = f2_pack(inv1, inv1);
      uint32_t ob[2][16];
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
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int n = qb * kBlock + row0 + 8 * u;
        if (n < p.N) {
          uint32_t* dst = reinterpret_cast<uint32_t*>(p.o + ((static_cast<size_t>(b) * p.N + n) * p.H + h) * kHeadDim);
#pragma unroll
          for (int i = 0; i < 16; ++i) dst[4 * i + c4] = ob[u][i];
          if (c4 == 0)
            p.lse[(static_cast<size_t>(b) * p.H + h) * p.N + n] =
                ((u ? m1 : m0) + __log2f(u ? l1 : l0) - kPOffsetLog2) * 0.69314718055994531f;
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

}  // namespace attnfp8
}  // namespace sol
