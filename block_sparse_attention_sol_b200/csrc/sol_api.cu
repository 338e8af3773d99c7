// libsol: the C ABI declared in include/sol.h.
//
// Host side of every call: validate arguments (before any CUDA call, so that a
// bad argument never launches anything), build TMA tensor maps where a kernel
// needs them, size grids from the device's SM count, and launch on the
// caller's stream.  Nothing here allocates device memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>
#include <utility>

#include "../../include/sol.h"
#include "sm100_ptx.cuh"
#include "attn_f32.cuh"
#include "blocks.cuh"
#include "attn_sm100.cuh"
#include "prologue.cuh"
#include "select.cuh"
#include "quant.cuh"
#include "attn_fp8.cuh"
#include "attn_bwd.cuh"


namespace {

constexpr int kMaxDevices = 64;
constexpr size_t kMaxSmemPerBlock = 227 * 1024;   // opt-in dynamic shared memory per CTA on sm_100

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool shape_ok(const sol_shape& s) {
  if (s.B <= 0 || s.N <= 0 || s.H <= 0 || s.D <= 0) return false;
  if (s.grid_t <= 0 || s.grid_h <= 0 || s.grid_w <= 0) return false;
  const long long n = static_cast<long long>(s.grid_t) * s.grid_h * s.grid_w;
  if (n != s.N) return false;
  // every tensor is indexed with 64-bit offsets; keep each dimension product sane
  const long long elems = static_cast<long long>(s.B) * s.N * s.H * s.D;
  return elems > 0 && elems < (1ll << 40);
}

int num_blocks(int N, int block) { return (N + block - 1) / block; }

// Unique id of the calling thread's current CUDA context (0: none yet).  A
// context created after cudaDeviceReset (or any other teardown of the primary
// context) gets a new id, so per-device caches keyed by it never outlive the
// context they were filled in.
sol_status current_context_id(unsigned long long* id) {
  static const auto fns = [] {
    void* cur = nullptr;
    void* get_id = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &cur, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess)
      cur = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &get_id, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      get_id = nullptr;
    return std::make_pair(reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(cur),
                          reinterpret_cast<PFN_cuCtxGetId_v12000>(get_id));
  }();
  if (fns.first == nullptr || fns.second == nullptr) return SOL_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (fns.first(&ctx) != CUDA_SUCCESS) return SOL_ERR_CUDA;
  *id = 0;
  if (ctx != nullptr && fns.second(ctx, id) != CUDA_SUCCESS) return SOL_ERR_CUDA;
  return SOL_OK;
}

struct DeviceInfo {
  int sm_count = 0;
  unsigned long long ctx_id = 0;   // context the attribute flags below were set in
  bool attn_attr = false, attn_fp8_attr = false;
  bool prologue_staged_attr[2] = {};   // qk_prologue_pool_staged_kernel without / with block means
  bool select_attr[32] = {};   // score_topk / score_topp_kernel instantiations with the shared-memory opt-in set
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

sol_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SOL_ERR_CUDA;
  unsigned long long ctx = 0;
  if (sol_status st = current_context_id(&ctx)) return st;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (ctx == 0 || ctx != d.ctx_id) {   // kernel attributes belong to a context: set them again in this one
    d.attn_attr = d.attn_fp8_attr = false;
    d.prologue_staged_attr[0] = d.prologue_staged_attr[1] = false;
    for (bool& f : d.select_attr) f = false;
    d.ctx_id = ctx;
  }
  if (d.sm_count == 0) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
      return SOL_ERR_CUDA;
    d.sm_count = sms;
  }
  *out = &d;
  return SOL_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// [B, N, H, D=128] bf16 viewed as a 4-D tensor (D, H, N, B); box = 64 channels x
// 1 head x 128 tokens x 1 batch, 128-byte swizzle; tokens past N read as zero.
sol_status make_bshd_map(CUtensorMap* map, const void* base, const sol_shape& s) {
  auto enc = tensor_map_encoder();
  if (!enc) return SOL_ERR_CUDA;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(s.D), static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(s.N),
                        static_cast<cuuint64_t>(s.B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s.D) * 2, static_cast<cuuint64_t>(s.H) * s.D * 2,
                           static_cast<cuuint64_t>(s.N) * s.H * s.D * 2};
  cuuint32_t box[4] = {64, 1, 128, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOL_OK : SOL_ERR_CUDA;
}

// 5-D view (channel, head, x, y, b * T + t) of a [B, N, H, D] bf16 tensor whose
// tokens are the grid in raster order; a box is 64 channels of one head over a
// tw x th x tt tile of tokens, rows in tile-raster order (x fastest).
sol_status make_tile_map(CUtensorMap* map, const void* base, const sol_shape& s, const sol::BlockMap& bm) {
  auto enc = tensor_map_encoder();
  if (!enc) return SOL_ERR_CUDA;
  const cuuint64_t row = static_cast<cuuint64_t>(s.H) * s.D * 2;   // bytes per token
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(s.D), static_cast<cuuint64_t>(s.H),
                        static_cast<cuuint64_t>(s.grid_w), static_cast<cuuint64_t>(s.grid_h),
                        static_cast<cuuint64_t>(s.grid_t) * s.B};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(s.D) * 2, row, row * s.grid_w, row * s.grid_w * s.grid_h};
  cuuint32_t box[5] = {64, 1, static_cast<cuuint32_t>(bm.tw), static_cast<cuuint32_t>(bm.th),
                       static_cast<cuuint32_t>(bm.tt)};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOL_OK : SOL_ERR_CUDA;
}

// Block map of 3-D tiles that cover the grid exactly, or SOL_ERR_INVALID_ARG.
sol_status tile_blocks(const sol_shape& s, sol_tile tile, sol::BlockMap* out) {
  if (tile.t < 1 || tile.h < 1 || tile.w < 1) return SOL_ERR_INVALID_ARG;
  if (s.grid_t % tile.t || s.grid_h % tile.h || s.grid_w % tile.w) return SOL_ERR_INVALID_ARG;
  if (static_cast<long long>(tile.t) * tile.h * tile.w > 4096) return SOL_ERR_UNSUPPORTED;
  *out = sol::tiled_blocks(tile.t, tile.h, tile.w, s.grid_h, s.grid_w);
  return SOL_OK;
}

int blocks_of(const sol_shape& s, const sol::BlockMap& bm) {
  return bm.tw == 0 ? num_blocks(s.N, bm.block) : s.N / bm.block;
}

// e4m3 code maps of the FP8 attention: K codes [B, N, H, D] as 4-D (c, h, n, b)
// with one 128-channel box per block of 128 tokens; V^T codes [B, H, D, N] as
// 3-D (n, d, b * H + h) with one 128-key x 128-channel box.  Both 128-byte swizzled.
sol_status make_fp8_maps(CUtensorMap* tk, CUtensorMap* tvt, const void* k8, const void* vt8, const sol_shape& s) {
  auto enc = tensor_map_encoder();
  if (!enc) return SOL_ERR_CUDA;
  cuuint64_t kd[4] = {static_cast<cuuint64_t>(s.D), static_cast<cuuint64_t>(s.H), static_cast<cuuint64_t>(s.N),
                      static_cast<cuuint64_t>(s.B)};
  cuuint64_t ks[3] = {static_cast<cuuint64_t>(s.D), static_cast<cuuint64_t>(s.H) * s.D,
                      static_cast<cuuint64_t>(s.N) * s.H * s.D};
  cuuint32_t kb[4] = {128, 1, 128, 1};
  cuuint32_t e4[4] = {1, 1, 1, 1};
  CUresult r = enc(tk, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(k8), kd, ks, kb, e4,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return SOL_ERR_CUDA;
  cuuint64_t vd[3] = {static_cast<cuuint64_t>(s.N), static_cast<cuuint64_t>(s.D),
                      static_cast<cuuint64_t>(s.B) * s.H};
  cuuint64_t vs[2] = {static_cast<cuuint64_t>(s.N), static_cast<cuuint64_t>(s.D) * s.N};
  cuuint32_t vb[3] = {128, 128, 1};
  cuuint32_t e3[3] = {1, 1, 1};
  r = enc(tvt, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(vt8), vd, vs, vb, e3, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? SOL_OK : SOL_ERR_CUDA;
}

sol_status launch_status() { return cudaGetLastError() == cudaSuccess ? SOL_OK : SOL_ERR_CUDA; }

__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    sol::mbar_init(&bar, 1);
    sol::fence_mbar_init();
    // nothing ever arrives on `bar`: the bounded wait must give up and report
    sol::mbar_wait(&bar, 0, &abort_flag, 0xFFu, limit_ns);
  }
}

}  // namespace

namespace {

// Launch shape of the score / top-k kernel: 32 rows per CTA when their scores
// fit in shared memory, else 16; keys per lane for the top-k.
struct ScorePlan {
  int rpw = 4, kpl = 8;
  size_t smem = 0;
  dim3 grid;
};

sol_status plan_scores(const sol_shape& s, int nb, ScorePlan* plan) {
  if (s.D != 64 && s.D != 128) return SOL_ERR_UNSUPPORTED;
  if (nb > sol::select::kMaxNb) return SOL_ERR_UNSUPPORTED;
  if (static_cast<long long>(s.B) * s.H > 65535) return SOL_ERR_UNSUPPORTED;
  plan->rpw = sol::select::score_topk_smem_bytes(s.D, 32, nb) <= kMaxSmemPerBlock ? 4 : 2;
  plan->smem = sol::select::score_topk_smem_bytes(s.D, 8 * plan->rpw, nb);
  if (plan->smem > kMaxSmemPerBlock) return SOL_ERR_UNSUPPORTED;
  plan->kpl = nb <= 256 ? 8 : nb <= 512 ? 16 : nb <= 1024 ? 32 : 64;
  plan->grid = dim3((nb + 8 * plan->rpw - 1) / (8 * plan->rpw), s.B * s.H);
  return SOL_OK;
}

// Launches score_topk_kernel<D, RPW, KPL> (or score_topp_kernel with kTopP) for the
// runtime choices (shared-memory opt-in set once per device and instantiation).
template <int D, int RPW, int KPL>
sol_status launch_score_topk_t(DeviceInfo* di, dim3 grid, size_t smem, cudaStream_t stream, const float* qbar,
                               const float* kbar, const sol::select::SelectArgs& a) {
  const bool topp = (a.flags & sol::select::kTopP) != 0u;
  auto kernel = topp ? sol::select::score_topp_kernel<D, RPW, KPL> : sol::select::score_topk_kernel<D, RPW, KPL>;
  const int slot = (topp ? 16 : 0) + (D == 128 ? 8 : 0) + (RPW == 4 ? 4 : 0) +
                   (KPL == 8 ? 0 : KPL == 16 ? 1 : KPL == 32 ? 2 : 3);
  if (!di->select_attr[slot]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kMaxSmemPerBlock)) != cudaSuccess)
      return SOL_ERR_CUDA;
    di->select_attr[slot] = true;
  }
  kernel<<<grid, sol::select::kThreads, smem, stream>>>(qbar, kbar, a);
  return launch_status();
}

template <int D, int RPW>
sol_status launch_score_topk_k(DeviceInfo* di, int kpl, dim3 grid, size_t smem, cudaStream_t stream,
                               const float* qbar, const float* kbar, const sol::select::SelectArgs& a) {
  switch (kpl) {
    case 8: return launch_score_topk_t<D, RPW, 8>(di, grid, smem, stream, qbar, kbar, a);
    case 16: return launch_score_topk_t<D, RPW, 16>(di, grid, smem, stream, qbar, kbar, a);
    case 32: return launch_score_topk_t<D, RPW, 32>(di, grid, smem, stream, qbar, kbar, a);
    default: return launch_score_topk_t<D, RPW, 64>(di, grid, smem, stream, qbar, kbar, a);
  }
}

sol_status launch_score_topk(DeviceInfo* di, int D, const ScorePlan& plan, cudaStream_t stream, const float* qbar,
                             const float* kbar, const sol::select::SelectArgs& a) {
  if (D == 128)
    return plan.rpw == 4 ? launch_score_topk_k<128, 4>(di, plan.kpl, plan.grid, plan.smem, stream, qbar, kbar, a)
                         : launch_score_topk_k<128, 2>(di, plan.kpl, plan.grid, plan.smem, stream, qbar, kbar, a);
  return plan.rpw == 4 ? launch_score_topk_k<64, 4>(di, plan.kpl, plan.grid, plan.smem, stream, qbar, kbar, a)
                       : launch_score_topk_k<64, 2>(di, plan.kpl, plan.grid, plan.smem, stream, qbar, kbar, a);
}

// Plain top-k arguments: no forced blocks, one k for every head, no counts.
sol::select::SelectArgs plain_select(const sol_shape& s, int nb, int topk, int32_t* idx, float* scores) {
  sol::select::SelectArgs a{};
  a.idx = idx;
  a.scores = scores;
  a.nb = nb;
  a.topk = topk;
  a.H = s.H;
  return a;
}

}  // namespace

namespace {

// Argument checks and kernel parameters shared by both prologue entry points.
sol_status prologue_params(const void* q_raw, const void* k_raw, void* q_out, void* k_out, const float* gamma_q,
                           const float* gamma_k, sol_shape s, int rope_dt, int rope_dh, int rope_dw, float rope_theta,
                           float eps, sol_dtype dt, sol::prologue::Params* out, size_t* smem_out) {
  if (!q_raw || !k_raw || !q_out || !k_out || !gamma_q || !gamma_k) return SOL_ERR_INVALID_ARG;
  if (!aligned16(q_raw) || !aligned16(k_raw) || !aligned16(q_out) || !aligned16(k_out)) return SOL_ERR_INVALID_ARG;
  if (!shape_ok(s)) return SOL_ERR_INVALID_ARG;
  if (dt != SOL_F32 && dt != SOL_BF16) return SOL_ERR_INVALID_ARG;
  if (rope_dt < 0 || rope_dh < 0 || rope_dw < 0 || (rope_dt | rope_dh | rope_dw) & 1) return SOL_ERR_INVALID_ARG;
  if (rope_dt + rope_dh + rope_dw != s.D) return SOL_ERR_INVALID_ARG;
  if (!(rope_theta > 0.f) || !(eps >= 0.f) || !std::isfinite(rope_theta) || !std::isfinite(eps))
    return SOL_ERR_INVALID_ARG;
  if (s.D != 64 && s.D != 128) return SOL_ERR_UNSUPPORTED;
  if (static_cast<long long>(s.B) * s.N >= (1ll << 31)) return SOL_ERR_UNSUPPORTED;
  sol::prologue::Params& p = *out;
  p.q_in = q_raw; p.k_in = k_raw; p.q_out = q_out; p.k_out = k_out;
  p.gamma_q = gamma_q; p.gamma_k = gamma_k;
  p.tokens = s.B * s.N;
  p.N = s.N; p.H = s.H;
  p.gt = s.grid_t; p.gh = s.grid_h; p.gw = s.grid_w;
  p.dt = rope_dt; p.dh = rope_dh; p.dw = rope_dw;
  p.log2_theta = std::log2(static_cast<double>(rope_theta));
  p.eps = eps;
  p.tab_t = s.grid_t * (rope_dt / 2);
  p.tab_h = p.tab_t + s.grid_h * (rope_dh / 2);
  p.tab_total = p.tab_h + s.grid_w * (rope_dw / 2);
  *smem_out = static_cast<size_t>(p.tab_total) * sizeof(float2);
  if (*smem_out > 48 * 1024) return SOL_ERR_UNSUPPORTED;
  return SOL_OK;
}

// The staged prologue (bf16, D = 128, H <= 32, the ring fits in shared memory):
// with block means when qbar_out is given, else plain over runs of 128 tokens.
// *launched stays false where the shape needs the register-streaming kernels.
sol_status launch_prologue_staged(const sol::prologue::Params& p, const sol_shape& s, sol_dtype dt,
                                  const sol::BlockMap& bm, int nb, float* qbar_out, float* kbar_out,
                                  cudaStream_t stream, bool* launched) {
  namespace ps = sol::prologue::staged;
  *launched = false;
  if (dt != SOL_BF16 || s.D != 128 || s.H > ps::kGroups) return SOL_OK;
  constexpr int kMaxSmem = 227 * 1024;
  const int off = ps::stage_offset(p.tab_total);
  const int stage_bytes = 2 * s.H * 128 * 2;
  const int stages = std::min(8, (kMaxSmem - off) / stage_bytes);
  if (stages < 2) return SOL_OK;
  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  const bool pool = qbar_out != nullptr;
  auto kern = pool ? sol::prologue::qk_prologue_pool_staged_kernel<1, true>
                   : sol::prologue::qk_prologue_pool_staged_kernel<1, false>;
  bool& attr = di->prologue_staged_attr[pool ? 1 : 0];
  if (!attr) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem) != cudaSuccess)
      return SOL_ERR_CUDA;
    attr = true;
  }
  const size_t total = static_cast<size_t>(off) + static_cast<size_t>(stages) * stage_bytes;
  const int units = s.B * nb;
  kern<<<std::min(units, di->sm_count), ps::kThreads, total, stream>>>(p, bm, nb, stages, qbar_out, kbar_out);
  *launched = true;
  return SOL_OK;
}

// The fused prologue + block means for any block map.
sol_status prologue_pool_impl(const void* q_raw, const void* k_raw, void* q_out, void* k_out, const float* gamma_q,
                              const float* gamma_k, sol_shape s, int rope_dt, int rope_dh, int rope_dw,
                              float rope_theta, float eps, sol_dtype dt, const sol::BlockMap& bm, float* qbar_out,
                              float* kbar_out, cudaStream_t stream) {
  sol::prologue::Params p;
  size_t smem = 0;
  if (sol_status st = prologue_params(q_raw, k_raw, q_out, k_out, gamma_q, gamma_k, s, rope_dt, rope_dh, rope_dw,
                                      rope_theta, eps, dt, &p, &smem))
    return st;
  if (!qbar_out || !kbar_out || !aligned16(qbar_out) || !aligned16(kbar_out) || bm.block <= 0)
    return SOL_ERR_INVALID_ARG;
  const int nb = blocks_of(s, bm);
  if (nb > 65535 || s.B > 65535) return SOL_ERR_UNSUPPORTED;
  const dim3 grid(nb, s.B);
  bool launched = false;
  if (sol_status st = launch_prologue_staged(p, s, dt, bm, nb, qbar_out, kbar_out, stream, &launched)) return st;
  if (launched) return launch_status();
  if (dt == SOL_BF16) {
    if (s.D == 128)
      sol::prologue::qk_prologue_pool_kernel<__nv_bfloat16, 128><<<grid, 256, smem, stream>>>(p, bm, nb, qbar_out,
                                                                                              kbar_out);
    else
      sol::prologue::qk_prologue_pool_kernel<__nv_bfloat16, 64><<<grid, 256, smem, stream>>>(p, bm, nb, qbar_out,
                                                                                             kbar_out);
  } else {
    if (s.D == 128)
      sol::prologue::qk_prologue_pool_kernel<float, 128><<<grid, 256, smem, stream>>>(p, bm, nb, qbar_out, kbar_out);
    else
      sol::prologue::qk_prologue_pool_kernel<float, 64><<<grid, 256, smem, stream>>>(p, bm, nb, qbar_out, kbar_out);
  }
  return launch_status();
}

}  // namespace

namespace {
// Attention with optional per-row block counts (both attention entry points).
sol_status sparse_attn_impl(const void* q, const void* k, const void* v, const int32_t* idx, const int32_t* counts,
                            sol_shape s, const sol::BlockMap& bm, int topk, float softmax_scale, sol_dtype dt, void* o,
                            float* lse, cudaStream_t stream);
}  // namespace

extern "C" {

const char* sol_status_string(sol_status st) {
  switch (st) {
    case SOL_OK: return "SOL_OK";
    case SOL_ERR_INVALID_ARG: return "SOL_ERR_INVALID_ARG";
    case SOL_ERR_UNSUPPORTED: return "SOL_ERR_UNSUPPORTED";
    case SOL_ERR_CUDA: return "SOL_ERR_CUDA";
    case SOL_ERR_TIMEOUT: return "SOL_ERR_TIMEOUT";
  }
  return "SOL_ERR_UNKNOWN";
}

sol_status sol_qk_prologue(const void* q_raw, const void* k_raw, void* q_out, void* k_out, const float* gamma_q,
                           const float* gamma_k, sol_shape s, int rope_dt, int rope_dh, int rope_dw, float rope_theta,
                           float eps, sol_dtype dt, cudaStream_t stream) {
  sol::prologue::Params p;
  size_t smem = 0;
  if (sol_status st = prologue_params(q_raw, k_raw, q_out, k_out, gamma_q, gamma_k, s, rope_dt, rope_dh, rope_dw,
                                      rope_theta, eps, dt, &p, &smem))
    return st;
  {
    const sol::BlockMap runs = sol::raster_blocks(128, s.grid_h, s.grid_w);
    bool launched = false;
    if (sol_status st = launch_prologue_staged(p, s, dt, runs, (s.N + 127) / 128, nullptr, nullptr, stream, &launched))
      return st;
    if (launched) return launch_status();
  }
  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  // Every row group keeps one head: the number of groups must be a multiple of H.
  const int threads = 256;
  const int lanes_per_row = (dt == SOL_BF16) ? s.D / 8 : s.D / 4;
  const int groups_per_cta = threads / lanes_per_row;
  int a = s.H, b = groups_per_cta;
  while (b) { const int r = a % b; a = b; b = r; }
  const long long unit = s.H / a;                       // CTAs per whole set of heads
  const long long needed = (static_cast<long long>(p.tokens) * s.H + groups_per_cta - 1) / groups_per_cta;
  const long long target = static_cast<long long>(dt == SOL_BF16 ? 2 : 4) * di->sm_count;   // one resident wave (the kernel's launch bound)
  long long grid_ll = std::min(needed, target);
  grid_ll = (grid_ll + unit - 1) / unit * unit;
  if (grid_ll > 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(grid_ll);
  if (dt == SOL_BF16) {
    if (s.D == 128) sol::prologue::qk_prologue_kernel<__nv_bfloat16, 128><<<grid, threads, smem, stream>>>(p);
    else sol::prologue::qk_prologue_kernel<__nv_bfloat16, 64><<<grid, threads, smem, stream>>>(p);
  } else {
    if (s.D == 128) sol::prologue::qk_prologue_kernel<float, 128><<<grid, threads, smem, stream>>>(p);
    else sol::prologue::qk_prologue_kernel<float, 64><<<grid, threads, smem, stream>>>(p);
  }
  return launch_status();
}

sol_status sol_qk_prologue_pool(const void* q_raw, const void* k_raw, void* q_out, void* k_out, const float* gamma_q,
                                const float* gamma_k, sol_shape s, int rope_dt, int rope_dh, int rope_dw,
                                float rope_theta, float eps, sol_dtype dt, int block, float* qbar_out,
                                float* kbar_out, cudaStream_t stream) {
  if (block <= 0) return SOL_ERR_INVALID_ARG;
  return prologue_pool_impl(q_raw, k_raw, q_out, k_out, gamma_q, gamma_k, s, rope_dt, rope_dh, rope_dw, rope_theta,
                            eps, dt, sol::raster_blocks(block, s.grid_h, s.grid_w), qbar_out, kbar_out, stream);
}

sol_status sol_qk_prologue_pool_tiled(const void* q_raw, const void* k_raw, void* q_out, void* k_out,
                                      const float* gamma_q, const float* gamma_k, sol_shape s, int rope_dt,
                                      int rope_dh, int rope_dw, float rope_theta, float eps, sol_dtype dt,
                                      sol_tile tile, float* qbar_out, float* kbar_out, cudaStream_t stream) {
  if (!shape_ok(s)) return SOL_ERR_INVALID_ARG;
  sol::BlockMap bm;
  if (sol_status st = tile_blocks(s, tile, &bm)) return st;
  return prologue_pool_impl(q_raw, k_raw, q_out, k_out, gamma_q, gamma_k, s, rope_dt, rope_dh, rope_dw, rope_theta,
                            eps, dt, bm, qbar_out, kbar_out, stream);
}

size_t sol_block_select_workspace_bytes(sol_shape s, int block) {
  if (!shape_ok(s) || block <= 0) return 0;
  return 2ull * s.B * s.H * static_cast<size_t>(num_blocks(s.N, block)) * s.D * sizeof(float);
}

sol_status sol_block_select(const void* q, const void* k, sol_shape s, int block, int topk, sol_dtype dt,
                            int32_t* idx_out, float* scores_out, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
  if (!q || !k || !idx_out || !workspace) return SOL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(workspace) || !aligned16(idx_out)) return SOL_ERR_INVALID_ARG;
  if (scores_out && !aligned16(scores_out)) return SOL_ERR_INVALID_ARG;
  if (!shape_ok(s) || block <= 0) return SOL_ERR_INVALID_ARG;
  if (dt != SOL_F32 && dt != SOL_BF16) return SOL_ERR_INVALID_ARG;
  const int nb = num_blocks(s.N, block);
  if (topk < 1 || topk > nb) return SOL_ERR_INVALID_ARG;
  if (workspace_bytes < sol_block_select_workspace_bytes(s, block)) return SOL_ERR_INVALID_ARG;
  ScorePlan plan;
  if (sol_status st = plan_scores(s, nb, &plan)) return st;

  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  float* qbar = static_cast<float*>(workspace);
  float* kbar = qbar + static_cast<size_t>(s.B) * s.H * nb * s.D;
  dim3 pg(nb, s.B, 2);
  if (dt == SOL_BF16)
    sol::select::block_pool_kernel<__nv_bfloat16><<<pg, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), qbar, kbar, s.N, s.H, s.D, block,
        nb);
  else
    sol::select::block_pool_kernel<float><<<pg, 256, 0, stream>>>(static_cast<const float*>(q),
                                                                  static_cast<const float*>(k), qbar, kbar, s.N, s.H,
                                                                  s.D, block, nb);
  if (sol_status st = launch_status()) return st;
  return launch_score_topk(di, s.D, plan, stream, qbar, kbar, plain_select(s, nb, topk, idx_out, scores_out));
}

sol_status sol_block_select_pooled(const float* qbar, const float* kbar, sol_shape s, int block, int topk,
                                   int32_t* idx_out, float* scores_out, cudaStream_t stream) {
  if (!qbar || !kbar || !idx_out) return SOL_ERR_INVALID_ARG;
  if (!aligned16(qbar) || !aligned16(kbar) || !aligned16(idx_out)) return SOL_ERR_INVALID_ARG;
  if (scores_out && !aligned16(scores_out)) return SOL_ERR_INVALID_ARG;
  if (!shape_ok(s) || block <= 0) return SOL_ERR_INVALID_ARG;
  const int nb = num_blocks(s.N, block);
  if (topk < 1 || topk > nb) return SOL_ERR_INVALID_ARG;
  ScorePlan plan;
  if (sol_status st = plan_scores(s, nb, &plan)) return st;
  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  return launch_score_topk(di, s.D, plan, stream, qbar, kbar, plain_select(s, nb, topk, idx_out, scores_out));
}

sol_status sol_block_select_pooled_ex(const float* qbar, const float* kbar, sol_shape s, int block, int topk,
                                      const sol_select_opts* opts, int32_t* idx_out, int32_t* counts_out,
                                      float* scores_out, cudaStream_t stream) {
  if (!qbar || !kbar || !idx_out || !counts_out || !opts) return SOL_ERR_INVALID_ARG;
  if (!aligned16(qbar) || !aligned16(kbar) || !aligned16(idx_out) || !aligned16(counts_out))
    return SOL_ERR_INVALID_ARG;
  if (scores_out && !aligned16(scores_out)) return SOL_ERR_INVALID_ARG;
  if (!shape_ok(s) || block <= 0) return SOL_ERR_INVALID_ARG;
  const unsigned known = SOL_SELECT_FORCE_DIAGONAL | SOL_SELECT_FORCE_FIRST_FRAME | SOL_SELECT_TOP_P;
  if (opts->flags & ~known) return SOL_ERR_INVALID_ARG;
  const bool topp = (opts->flags & SOL_SELECT_TOP_P) != 0u;
  if (topp && !(opts->top_p > 0.f && opts->top_p <= 1.f)) return SOL_ERR_INVALID_ARG;
  if (topp && !std::isfinite(opts->softmax_scale)) return SOL_ERR_INVALID_ARG;
  const int nb = num_blocks(s.N, block);
  if (topk < 1 || topk > nb) return SOL_ERR_INVALID_ARG;
  // blocks holding a token of frame t = 0: tokens 0 .. grid_h * grid_w - 1 of runs of `block`
  // tokens, or the tiles of the first tile layer
  int n_first = num_blocks(s.grid_h * s.grid_w, block);
  const sol_tile tile = opts->tile;
  if (tile.t != 0 || tile.h != 0 || tile.w != 0) {
    sol::BlockMap bm;
    if (sol_status st = tile_blocks(s, tile, &bm)) return st;
    if (bm.block != block) return SOL_ERR_INVALID_ARG;
    n_first = bm.nty * bm.ntx;
  }
  ScorePlan plan;
  if (sol_status st = plan_scores(s, nb, &plan)) return st;
  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  sol::select::SelectArgs a = plain_select(s, nb, topk, idx_out, scores_out);
  a.counts = counts_out;
  a.head_k = opts->head_k;
  a.flags = (opts->flags & SOL_SELECT_FORCE_DIAGONAL ? sol::select::kForceDiagonal : 0u) |
            (opts->flags & SOL_SELECT_FORCE_FIRST_FRAME ? sol::select::kForceFirstFrame : 0u) |
            (topp ? sol::select::kTopP : 0u);
  a.n_first = n_first;
  a.top_p = opts->top_p;
  const float scale = opts->softmax_scale > 0.f ? opts->softmax_scale : 1.0f / std::sqrt(static_cast<float>(s.D));
  a.scale_log2 = scale * 1.4426950408889634f;   // log2(e)
  return launch_score_topk(di, s.D, plan, stream, qbar, kbar, a);
}

}  // extern "C"

namespace {
// Threads per CTA of the exchange kernels: D / 16 lanes per row, at most 512
// (each thread takes two rows per pass, so half the rows' lanes suffice)
int quant_block(int rows, int D) { return std::min(((rows + 1) / 2) * (D / 16), 512); }
// CTAs of the exchange kernels: two resident waves (2048 threads per SM), the CTAs loop over tokens.
long long quant_grid(const DeviceInfo* di, int threads) {
  return 2ll * di->sm_count * std::max(1, 2048 / threads);
}
}  // namespace

extern "C" {

sol_status sol_quant_pack(const void* x, int B, int N, int H, int D, int G, sol_split split, sol_code code,
                          void* codes_out, float* scales_out, long long g_stride_rows, cudaStream_t stream) {
  if (!x || !codes_out || !scales_out) return SOL_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes_out) || reinterpret_cast<uintptr_t>(scales_out) % 4) return SOL_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || H < 1 || G < 1) return SOL_ERR_INVALID_ARG;
  if (split != SOL_SPLIT_HEADS && split != SOL_SPLIT_TOKENS) return SOL_ERR_INVALID_ARG;
  if (code != SOL_CODE_INT8 && code != SOL_CODE_E4M3) return SOL_ERR_INVALID_ARG;
  if ((split == SOL_SPLIT_HEADS ? H : N) % G != 0) return SOL_ERR_INVALID_ARG;
  const long long per_g = static_cast<long long>(B) * N * H / G;
  if (g_stride_rows == 0) g_stride_rows = per_g;
  if (g_stride_rows < per_g) return SOL_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SOL_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * N * H >= 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* cb = static_cast<uint8_t*>(codes_out);
  const int threads = quant_block(H, D);
  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  const dim3 g(static_cast<unsigned>(std::min<long long>(static_cast<long long>(B) * N, quant_grid(di, threads))));
  if (D == 128) {
    if (code == SOL_CODE_INT8)
      sol::quant::quant_pack_kernel<128, sol::quant::kInt8><<<g, threads, 0, stream>>>(xb, cb, scales_out, B, N, H, G, split,
                                                                                   g_stride_rows);
    else
      sol::quant::quant_pack_kernel<128, sol::quant::kE4M3><<<g, threads, 0, stream>>>(xb, cb, scales_out, B, N, H, G, split,
                                                                                   g_stride_rows);
  } else {
    if (code == SOL_CODE_INT8)
      sol::quant::quant_pack_kernel<64, sol::quant::kInt8><<<g, threads, 0, stream>>>(xb, cb, scales_out, B, N, H, G, split,
                                                                                  g_stride_rows);
    else
      sol::quant::quant_pack_kernel<64, sol::quant::kE4M3><<<g, threads, 0, stream>>>(xb, cb, scales_out, B, N, H, G, split,
                                                                                  g_stride_rows);
  }
  return launch_status();
}

sol_status sol_dequant_unpack(const void* codes, const float* scales, int B, int Nc, int Hc, int D, int G,
                              sol_split split, sol_code code, void* out, long long g_stride_rows, cudaStream_t stream) {
  if (!codes || !scales || !out) return SOL_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(out) || reinterpret_cast<uintptr_t>(scales) % 4) return SOL_ERR_INVALID_ARG;
  if (B < 1 || Nc < 1 || Hc < 1 || G < 1) return SOL_ERR_INVALID_ARG;
  if (split != SOL_SPLIT_HEADS && split != SOL_SPLIT_TOKENS) return SOL_ERR_INVALID_ARG;
  if (code != SOL_CODE_INT8 && code != SOL_CODE_E4M3) return SOL_ERR_INVALID_ARG;
  const long long per_g = static_cast<long long>(B) * Nc * Hc;
  if (g_stride_rows == 0) g_stride_rows = per_g;
  if (g_stride_rows < per_g) return SOL_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return SOL_ERR_UNSUPPORTED;
  if (G * per_g >= 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  const auto* cb = static_cast<const uint8_t*>(codes);
  auto* ob = static_cast<__nv_bfloat16*>(out);
  const int threads = std::min(((Hc + sol::quant::kUnpackRows - 1) / sol::quant::kUnpackRows) * (D / 16), 512);
  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  const dim3 g(static_cast<unsigned>(std::min<long long>(static_cast<long long>(G) * B * Nc, quant_grid(di, threads))));
  if (D == 128) {
    if (code == SOL_CODE_INT8)
      sol::quant::dequant_unpack_kernel<128, sol::quant::kInt8><<<g, threads, 0, stream>>>(cb, scales, ob, B, Nc, Hc, G,
                                                                                       split, g_stride_rows);
    else
      sol::quant::dequant_unpack_kernel<128, sol::quant::kE4M3><<<g, threads, 0, stream>>>(cb, scales, ob, B, Nc, Hc, G,
                                                                                       split, g_stride_rows);
  } else {
    if (code == SOL_CODE_INT8)
      sol::quant::dequant_unpack_kernel<64, sol::quant::kInt8><<<g, threads, 0, stream>>>(cb, scales, ob, B, Nc, Hc, G,
                                                                                      split, g_stride_rows);
    else
      sol::quant::dequant_unpack_kernel<64, sol::quant::kE4M3><<<g, threads, 0, stream>>>(cb, scales, ob, B, Nc, Hc, G,
                                                                                      split, g_stride_rows);
  }
  return launch_status();
}

size_t sol_quant_attn_fp8_workspace_bytes(sol_shape s) {
  if (!shape_ok(s)) return 0;
  return (static_cast<size_t>(s.B) * s.H * sizeof(unsigned) + 15) / 16 * 16;
}

sol_status sol_quant_attn_fp8(const void* q, const void* k, const void* v, sol_shape s, void* q8, float* q_scale,
                              void* k8, float* k_scale, void* vt8, float* v_scale, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !k || !v || !q8 || !q_scale || !k8 || !k_scale || !vt8 || !v_scale || !workspace)
    return SOL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(q8) || !aligned16(k8) || !aligned16(vt8) ||
      !aligned16(workspace))
    return SOL_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q_scale) % 8 || reinterpret_cast<uintptr_t>(k_scale) % 8 ||
      reinterpret_cast<uintptr_t>(v_scale) % 4)
    return SOL_ERR_INVALID_ARG;
  if (!shape_ok(s)) return SOL_ERR_INVALID_ARG;
  if (workspace_bytes < sol_quant_attn_fp8_workspace_bytes(s)) return SOL_ERR_INVALID_ARG;
  if (s.D != 128 || s.N % 16 != 0) return SOL_ERR_UNSUPPORTED;
  if (static_cast<long long>(s.B) * s.N * s.H >= 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  const int threads = std::min(s.H * (s.D / 16), 512);
  const unsigned grid = static_cast<unsigned>(std::min<long long>(static_cast<long long>(s.B) * s.N,
                                                                  quant_grid(di, threads)));
  sol::quant::quant_rows_e4m3_kernel<128><<<grid, threads, 0, stream>>>(qb, static_cast<uint8_t*>(q8), q_scale, s.B,
                                                                        s.N, s.H);
  const int nbk = num_blocks(s.N, 128);
  if (static_cast<long long>(s.B) * s.H * nbk > 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  sol::quant::quant_kblock_e4m3_kernel<<<static_cast<unsigned>(s.B * s.H * nbk), 256, 0, stream>>>(
      kb, static_cast<uint8_t*>(k8), k_scale, s.B, s.N, s.H, nbk);
  auto* amax = static_cast<unsigned*>(workspace);
  if (cudaMemsetAsync(amax, 0, static_cast<size_t>(s.B) * s.H * sizeof(unsigned), stream) != cudaSuccess)
    return SOL_ERR_CUDA;
  const int athreads = std::min(s.H * (s.D / 16), 256);
  const unsigned agrid = static_cast<unsigned>(std::min<long long>(static_cast<long long>(s.B) * s.N,
                                                                   quant_grid(di, athreads)));
  sol::quant::head_amax_kernel<128><<<agrid, athreads, 0, stream>>>(vb, amax, s.B, s.N, s.H);
  const int nb = num_blocks(s.N, 128);
  const long long vgrid = static_cast<long long>(s.B) * s.H * nb;
  if (vgrid > 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  sol::quant::quant_vt_e4m3_kernel<<<static_cast<unsigned>(vgrid), 256, 0, stream>>>(
      vb, amax, static_cast<uint8_t*>(vt8), v_scale, s.B, s.N, s.H, nb);
  return launch_status();
}

sol_status sol_sparse_attn_fwd_fp8(const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                                   const void* vt8, const float* v_scale, const int32_t* idx, const int32_t* counts,
                                   sol_shape s, int block, int topk, float softmax_scale, void* o, float* lse,
                                   cudaStream_t stream) {
  if (!q8 || !q_scale || !k8 || !k_scale || !vt8 || !v_scale || !idx || !o || !lse) return SOL_ERR_INVALID_ARG;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(vt8) || !aligned16(idx) || !aligned16(o) || !aligned16(lse))
    return SOL_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q_scale) % 8 || reinterpret_cast<uintptr_t>(k_scale) % 8) return SOL_ERR_INVALID_ARG;
  if (!shape_ok(s) || block <= 0) return SOL_ERR_INVALID_ARG;
  const int nb = num_blocks(s.N, block);
  if (topk < 1 || topk > nb) return SOL_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return SOL_ERR_INVALID_ARG;
  if (s.D != sol::attnfp8::kHeadDim || block != sol::attnfp8::kBlock || s.N % 16 != 0) return SOL_ERR_UNSUPPORTED;
  const long long tiles = static_cast<long long>(s.B) * s.H * nb;
  if (tiles > 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(s.D));
  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;
  CUtensorMap tk, tvt;
  if (sol_status st = make_fp8_maps(&tk, &tvt, k8, vt8, s)) return st;
  const size_t smem = sizeof(sol::attnfp8::Smem) + 1024;
  if (!di->attn_fp8_attr) {
    if (cudaFuncSetAttribute(sol::attnfp8::sparse_attn_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return SOL_ERR_CUDA;
    di->attn_fp8_attr = true;
  }
  sol::attnfp8::Params p;
  p.q = static_cast<const uint8_t*>(q8);
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.idx = idx;
  p.counts = counts;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = s.B; p.N = s.N; p.H = s.H; p.nb = nb; p.topk = topk;
  p.num_tiles = static_cast<int>(tiles);
  p.scale_log2 = scale * 1.4426950408889634f;
  const int grid = static_cast<int>(std::min<long long>(tiles, di->sm_count));
  sol::attnfp8::sparse_attn_fp8_kernel<<<grid, sol::attnfp8::kThreads, smem, stream>>>(tk, tvt, p);
  return launch_status();
}

size_t sol_sparse_attn_bwd_workspace_bytes(sol_shape s, int block) {
  if (!shape_ok(s) || block <= 0) return 0;
  const size_t bh = static_cast<size_t>(s.B) * s.H, nb = static_cast<size_t>(num_blocks(s.N, block));
  auto r16 = [](size_t x) { return (x + 15) / 16 * 16; };
  return r16(bh * s.N * sizeof(float)) + r16(bh * nb * nb * sizeof(int32_t)) + r16(bh * nb * sizeof(int32_t));
}

sol_status sol_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dout, const int32_t* idx, const int32_t* counts, sol_shape s, int block,
                               int topk, float softmax_scale, sol_dtype dt, float* dq, float* dk, float* dv,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!q || !k || !v || !o || !lse || !dout || !idx || !dq || !dk || !dv || !workspace) return SOL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
    return SOL_ERR_INVALID_ARG;
  if (!shape_ok(s) || block <= 0) return SOL_ERR_INVALID_ARG;
  if (dt != SOL_F32 && dt != SOL_BF16) return SOL_ERR_INVALID_ARG;
  const int nb = num_blocks(s.N, block);
  if (topk < 1 || topk > nb) return SOL_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return SOL_ERR_INVALID_ARG;
  if (workspace_bytes < sol_sparse_attn_bwd_workspace_bytes(s, block)) return SOL_ERR_INVALID_ARG;
  if (s.D != 64 && s.D != 128) return SOL_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(s.B) * s.H * s.N;
  const long long grid = (rows + sol::attnbwd::kWarps - 1) / sol::attnbwd::kWarps;
  const long long tiles = static_cast<long long>(s.B) * s.H * nb;
  if (grid > 0x7fffffffll || (tiles + 255) / 256 > 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(s.D));
  auto r16 = [](size_t x) { return (x + 15) / 16 * 16; };
  const size_t bh = static_cast<size_t>(s.B) * s.H;
  auto* base = static_cast<uint8_t*>(workspace);
  auto* delta = reinterpret_cast<float*>(base);
  auto* inv = reinterpret_cast<int32_t*>(base + r16(bh * s.N * sizeof(float)));
  auto* inv_cnt = reinterpret_cast<int32_t*>(base + r16(bh * s.N * sizeof(float)) +
                                             r16(bh * nb * static_cast<size_t>(nb) * sizeof(int32_t)));
  const sol::attnbwd::Shape sh{s.B, s.N, s.H, block, nb, topk};
  const dim3 g(static_cast<unsigned>(grid)), t(sol::attnbwd::kWarps * 32);
  sol::attnbwd::bwd_invert_kernel<<<static_cast<unsigned>((tiles + 255) / 256), 256, 0, stream>>>(idx, counts, inv,
                                                                                                    inv_cnt, sh);
  auto run = [&](auto tag, auto dtag) {
    using T = decltype(tag);
    constexpr int D = decltype(dtag)::value;
    const T* qq = static_cast<const T*>(q);
    const T* kk = static_cast<const T*>(k);
    const T* vv = static_cast<const T*>(v);
    const T* oo = static_cast<const T*>(o);
    const T* dd = static_cast<const T*>(dout);
    sol::attnbwd::bwd_delta_kernel<T, D><<<g, t, 0, stream>>>(oo, dd, delta, sh);
    sol::attnbwd::bwd_dq_kernel<T, D><<<g, t, 0, stream>>>(qq, kk, vv, dd, lse, delta, idx, counts, dq, sh, scale);
    sol::attnbwd::bwd_dkdv_kernel<T, D><<<g, t, 0, stream>>>(qq, kk, vv, dd, lse, delta, inv, inv_cnt, dk, dv, sh,
                                                             scale);
  };
  if (dt == SOL_BF16) {
    if (s.D == 128) run(__nv_bfloat16{}, std::integral_constant<int, 128>{});
    else run(__nv_bfloat16{}, std::integral_constant<int, 64>{});
  } else {
    if (s.D == 128) run(float{}, std::integral_constant<int, 128>{});
    else run(float{}, std::integral_constant<int, 64>{});
  }
  return launch_status();
}

sol_status sol_sparse_attn_fwd(const void* q, const void* k, const void* v, const int32_t* idx, sol_shape s,
                               int block, int topk, float softmax_scale, sol_dtype dt, void* o, float* lse,
                               cudaStream_t stream) {
  if (block <= 0) return SOL_ERR_INVALID_ARG;
  return sparse_attn_impl(q, k, v, idx, nullptr, s, sol::raster_blocks(block, s.grid_h, s.grid_w), topk,
                          softmax_scale, dt, o, lse, stream);
}

sol_status sol_sparse_attn_fwd_counts(const void* q, const void* k, const void* v, const int32_t* idx,
                                      const int32_t* counts, sol_shape s, int block, int topk, float softmax_scale,
                                      sol_dtype dt, void* o, float* lse, cudaStream_t stream) {
  if (!counts || block <= 0) return SOL_ERR_INVALID_ARG;
  return sparse_attn_impl(q, k, v, idx, counts, s, sol::raster_blocks(block, s.grid_h, s.grid_w), topk,
                          softmax_scale, dt, o, lse, stream);
}

sol_status sol_sparse_attn_fwd_tiled(const void* q, const void* k, const void* v, const int32_t* idx,
                                     const int32_t* counts, sol_shape s, sol_tile tile, int topk, float softmax_scale,
                                     sol_dtype dt, void* o, float* lse, cudaStream_t stream) {
  if (!shape_ok(s)) return SOL_ERR_INVALID_ARG;
  sol::BlockMap bm;
  if (sol_status st = tile_blocks(s, tile, &bm)) return st;
  return sparse_attn_impl(q, k, v, idx, counts, s, bm, topk, softmax_scale, dt, o, lse, stream);
}

}  // extern "C"

namespace {

sol_status sparse_attn_impl(const void* q, const void* k, const void* v, const int32_t* idx, const int32_t* counts,
                            sol_shape s, const sol::BlockMap& bm, int topk, float softmax_scale, sol_dtype dt, void* o,
                            float* lse, cudaStream_t stream) {
  if (!q || !k || !v || !idx || !o || !lse) return SOL_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(idx) || !aligned16(lse))
    return SOL_ERR_INVALID_ARG;
  if (!shape_ok(s) || bm.block <= 0) return SOL_ERR_INVALID_ARG;
  if (dt != SOL_F32 && dt != SOL_BF16) return SOL_ERR_INVALID_ARG;
  const int nb = blocks_of(s, bm);
  if (topk < 1 || topk > nb) return SOL_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return SOL_ERR_INVALID_ARG;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt(static_cast<float>(s.D));

  DeviceInfo* di = nullptr;
  if (sol_status st = device_info(&di)) return st;

  if (dt == SOL_F32) {
    if (s.D != 64 && s.D != 128) return SOL_ERR_UNSUPPORTED;
    const long long rows = static_cast<long long>(s.B) * s.H * s.N;
    const long long grid = (rows + sol::attnf32::kWarps - 1) / sol::attnf32::kWarps;
    if (grid > 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
    if (s.D == 128)
      sol::attnf32::sparse_attn_fwd_f32_kernel<128><<<static_cast<int>(grid), sol::attnf32::kWarps * 32, 0, stream>>>(
          static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), idx, counts,
          static_cast<float*>(o), lse, s.B, s.N, s.H, bm, nb, topk, scale);
    else
      sol::attnf32::sparse_attn_fwd_f32_kernel<64><<<static_cast<int>(grid), sol::attnf32::kWarps * 32, 0, stream>>>(
          static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), idx, counts,
          static_cast<float*>(o), lse, s.B, s.N, s.H, bm, nb, topk, scale);
    return launch_status();
  }

  // bf16: tcgen05 tensor-core path
  if (s.D != sol::attn100::kHeadDim || bm.block != sol::attn100::kBlock) return SOL_ERR_UNSUPPORTED;
  const long long tiles = static_cast<long long>(s.B) * s.H * nb;
  if (tiles > 0x7fffffffll) return SOL_ERR_UNSUPPORTED;
  CUtensorMap tk, tv;
  if (bm.tw == 0) {
    if (sol_status st = make_bshd_map(&tk, k, s)) return st;
    if (sol_status st = make_bshd_map(&tv, v, s)) return st;
  } else {
    if (sol_status st = make_tile_map(&tk, k, s, bm)) return st;
    if (sol_status st = make_tile_map(&tv, v, s, bm)) return st;
  }
  const size_t smem = sizeof(sol::attn100::Smem) + 1024;
  if (!di->attn_attr) {
    if (cudaFuncSetAttribute(sol::attn100::sparse_attn_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return SOL_ERR_CUDA;
    di->attn_attr = true;
  }
  sol::attn100::Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.counts = counts;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = s.B; p.N = s.N; p.H = s.H; p.nb = nb; p.topk = topk;
  p.num_tiles = static_cast<int>(tiles);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.bm = bm;
  p.T = s.grid_t;
  const int grid = static_cast<int>(std::min<long long>(tiles, di->sm_count));
  sol::attn100::sparse_attn_fwd_kernel<<<grid, sol::attn100::kThreads, smem, stream>>>(tk, tv, p);
  return launch_status();
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------- no-alloc select
// Scratch for sol_block_select_noalloc: one array per device, shared by every
// call on that device (see include/sol.h for the size limit and the race rule).
static __device__ __align__(256) unsigned char g_noalloc_scratch[SOL_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};
std::mutex g_noalloc_mu;

// Host code may not pass g_noalloc_scratch itself to a kernel (on the host it
// names a stand-in, not device memory): look up its device address once per
// device and context, with that device current.  The address is cached with
// the id of the context it was looked up in; a new context on the device (after
// cudaDeviceReset, for instance) looks it up again.
sol_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SOL_ERR_CUDA;
  unsigned long long ctx = 0;
  if (sol_status st = current_context_id(&ctx)) return st;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SOL_ERR_CUDA;
    if (sol_status st = current_context_id(&ctx)) return st;   // the lookup made the context current if it was not
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return SOL_OK;
}
}  // namespace

sol_status sol_block_select_noalloc(const void* q, const void* k, sol_shape s, int block, int topk, sol_dtype dt,
                                    int32_t* idx_out, float* scores_out, cudaStream_t stream) {
  const size_t need = sol_block_select_workspace_bytes(s, block);
  if (need == 0) return SOL_ERR_INVALID_ARG;
  if (need > SOL_NOALLOC_SCRATCH_BYTES) return SOL_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (sol_status st = noalloc_scratch(&scratch)) return st;
  return sol_block_select(q, k, s, block, topk, dt, idx_out, scores_out, scratch, SOL_NOALLOC_SCRATCH_BYTES,
                          stream);
}

sol_status sol_check_device_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return SOL_ERR_CUDA;
  unsigned int word = 0;
  if (cudaMemcpyFromSymbol(&word, sol::g_error_word, sizeof(word)) != cudaSuccess) return SOL_ERR_CUDA;
  if (word != 0u) {
    const unsigned int zero = 0u;
    if (cudaMemcpyToSymbol(sol::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return SOL_ERR_CUDA;
    return (word & sol::kErrTimeout) ? SOL_ERR_TIMEOUT : SOL_ERR_INVALID_ARG;
  }
  return SOL_OK;
}

sol_status sol_selftest_wait_timeout(unsigned limit_us, cudaStream_t stream) {
  if (limit_us < 1u || limit_us > 1000000u) return SOL_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<unsigned long long>(limit_us) * 1000ull);
  return launch_status();
}

}  // extern "C"
