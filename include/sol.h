/*
 * sol.h -- C ABI of libsol, the B200 (sm_100a) implementation of the Sol-Attn
 * hot path: fused QK-RMSNorm + 3D RoPE, block selection, and block-sparse
 * attention returning O and LSE.
 *
 * Source of the method.  The Sol-H3 runtime for MiniMax-H3 video diffusion
 * credits Sol-Attn -- a training-free sparse attention that decides per query
 * which parts of the attention computation matter -- with the largest share of
 * its speed-up, and merges normalisation and RoPE into single kernels
 * (ai-feiten.nl, "Videomodel MiniMax-H3 rendert sneller dan afspelen", section
 * "Waar de snelheidswinst vandaan komt").  The pages give no formulas; the
 * concrete definition implemented here is stated at each call.
 *
 * Conventions shared by every call
 *  - Layouts: activations are [B, N, H, D] contiguous ("BSHD": token-major,
 *    then head, then channel).  Tokens are the latent video grid
 *    (grid_t, grid_h, grid_w) flattened in raster order, n = (t*grid_h + y)*grid_w + x.
 *    Blocks are runs of `block` consecutive tokens; the last may be short (the
 *    *_tiled calls use 3-D tiles instead, see sol_tile).
 *  - Memory: every pointer is a DEVICE pointer on the current CUDA device,
 *    16-byte aligned, owned by the caller.  The library never allocates,
 *    frees or synchronises, except sol_check_device_status(), which
 *    synchronises its stream.
 *  - Asynchrony: work is enqueued on `stream` and returns immediately.
 *    Argument errors are reported synchronously (SOL_ERR_INVALID_ARG /
 *    SOL_ERR_UNSUPPORTED) before anything is launched; launch failures return
 *    SOL_ERR_CUDA.  Device-side waits are bounded (2 s); a wait that runs out
 *    sets a device error word that sol_check_device_status() reports as
 *    SOL_ERR_TIMEOUT.
 *  - Thread safety: stateless apart from that error word and per-device
 *    caches of kernel attributes; calls may come from several host threads.
 */
#ifndef SOL_H_
#define SOL_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SOL_OK = 0,
  SOL_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, inconsistent shape, k out of range */
  SOL_ERR_UNSUPPORTED = 2,   /* valid request outside the implemented shapes / dtypes          */
  SOL_ERR_CUDA = 3,          /* a CUDA runtime or driver call failed                            */
  SOL_ERR_TIMEOUT = 4        /* a device-side bounded wait ran out (see sol_check_device_status) */
} sol_status;

typedef enum { SOL_F32 = 0, SOL_BF16 = 1 } sol_dtype;

/* B batch, N tokens (== grid_t*grid_h*grid_w), H heads, D head dim. */
typedef struct {
  int B, N, H, D;
  int grid_t, grid_h, grid_w;
} sol_shape;

/* 3-D token tiles (the *_tiled calls): block i is the tile (it, iy, ix) of
 * t x h x w tokens, i = (it * (grid_h/h) + iy) * (grid_w/w) + ix, its tokens
 * taken in raster order (frame, row, column) inside the tile; block = t*h*w.
 * The tiles must cover the grid exactly (grid_t % t == grid_h % h ==
 * grid_w % w == 0), else SOL_ERR_INVALID_ARG.  The pages leave the shape of
 * the attention's "parts" open; runs of consecutive tokens are the default. */
typedef struct {
  int t, h, w;
} sol_tile;

/*
 * sol_qk_prologue -- fused QK-RMSNorm + 3D RoPE (normalisation and RoPE merged
 * into one kernel: ai-feiten.nl, "Videomodel MiniMax-H3 rendert sneller dan
 * afspelen", "Waar de snelheidswinst vandaan komt").
 *
 * For Q and K, per (b, n, h):
 *   y_d = x_d / sqrt(mean_d x_d^2 + eps) * gamma[h*D + d]
 *   then channel pairs (2p, 2p+1) rotate by angle pos * theta^(-2i/d_axis):
 *   the first rope_dt/2 pairs use the frame index t, the next rope_dh/2 the row
 *   y, the last rope_dw/2 the column x; i counts pairs within the axis.
 *   (y0, y1) -> (y0 cos - y1 sin, y0 sin + y1 cos).
 * q_raw, k_raw : [B,N,H,D] inputs (dtype dt);  q_out, k_out : [B,N,H,D] outputs
 *                (may alias the inputs exactly, not partially).
 * gamma_q, gamma_k : fp32 [H*D].
 * rope_dt + rope_dh + rope_dw == D, each even.  D in {64, 128}.
 * Arithmetic in fp32; bf16 outputs are rounded to nearest even.
 */
sol_status sol_qk_prologue(const void* q_raw, const void* k_raw, void* q_out, void* k_out,
                           const float* gamma_q, const float* gamma_k, sol_shape s,
                           int rope_dt, int rope_dh, int rope_dw, float rope_theta, float eps,
                           sol_dtype dt, cudaStream_t stream);

/* Bytes of scratch sol_block_select needs: the fp32 pooled means of Q and K,
 * 2 * B * H * ceil(N/block) * D * 4.  Returns 0 for an invalid shape. */
size_t sol_block_select_workspace_bytes(sol_shape s, int block);

/*
 * sol_block_select -- the "preparation" of the sparse attention
 * (ai-feiten.nl, same section: it became 76.4% faster in Sol-H3).
 *
 * qbar[b,h,i] = mean of q over the valid tokens of block i (likewise kbar);
 * s[b,h,i,j]  = qbar[b,h,i] . kbar[b,h,j]  (fp32);
 * idx[b,h,i,:] = the topk largest s[b,h,i,:], exact ties to the lower j,
 *                listed in ascending j.
 * q, k        : [B,N,H,D] (dtype dt), normally sol_qk_prologue's outputs.
 * idx_out     : int32 [B, H, nb, topk], nb = ceil(N/block).
 * scores_out  : optional fp32 [B, H, nb, nb] copy of s (NULL to skip).
 * workspace   : device scratch of at least sol_block_select_workspace_bytes().
 * 1 <= topk <= nb, D in {64, 128}, nb <= 2048.
 */
sol_status sol_block_select(const void* q, const void* k, sol_shape s, int block, int topk,
                            sol_dtype dt, int32_t* idx_out, float* scores_out,
                            void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * sol_qk_prologue_pool -- sol_qk_prologue that also emits the block means the
 * selection pools, from the same pass over Q and K (the runtime on the pages
 * made this "preparation" 76.4% faster: ai-feiten.nl, same section).
 *
 * q_out, k_out : exactly sol_qk_prologue's outputs (same arithmetic, bit for bit).
 * qbar_out[b,h,i,:] = mean over the valid tokens n of block i of the STORED
 *                     (rounded) q_out[b,n,h,:], fp32 [B, H, nb, D], nb =
 *                     ceil(N/block); kbar_out likewise from k_out.  Summed in
 *                     ascending token order in fp32, so they equal the means
 *                     sol_block_select computes from q_out and k_out.
 * Other arguments, aliasing and limits as for sol_qk_prologue; block >= 1;
 * qbar_out, kbar_out 16-byte aligned, caller-owned.
 */
sol_status sol_qk_prologue_pool(const void* q_raw, const void* k_raw, void* q_out, void* k_out,
                                const float* gamma_q, const float* gamma_k, sol_shape s,
                                int rope_dt, int rope_dh, int rope_dw, float rope_theta, float eps,
                                sol_dtype dt, int block, float* qbar_out, float* kbar_out,
                                cudaStream_t stream);

/*
 * sol_block_select_pooled -- the scoring and top-k of sol_block_select from
 * block means already computed (by sol_qk_prologue_pool): no pooling pass and
 * no workspace.
 *
 * qbar, kbar : fp32 [B, H, nb, D], 16-byte aligned.  idx_out, scores_out and
 * the limits as for sol_block_select.  Given equal means, the result equals
 * sol_block_select's.
 */
sol_status sol_block_select_pooled(const float* qbar, const float* kbar, sol_shape s, int block, int topk,
                                   int32_t* idx_out, float* scores_out, cudaStream_t stream);

/*
 * Selection variants -- the per-query choices the pages leave open (Sol-Attn
 * "decides per query" which parts of the attention matter: ai-feiten.nl,
 * "Videomodel MiniMax-H3 rendert sneller dan afspelen", section "Waar de
 * snelheidswinst vandaan komt"; the rules below are this library's readings).
 *
 * flags:
 *  SOL_SELECT_FORCE_DIAGONAL    every query block keeps its own key block i.
 *  SOL_SELECT_FORCE_FIRST_FRAME every query block keeps the key blocks that hold
 *                               tokens of frame t = 0: ids 0 .. ceil(grid_h *
 *                               grid_w / block) - 1 (runs), or the first
 *                               (grid_h/h)*(grid_w/w) ids (tiles).
 *  SOL_SELECT_TOP_P             the row keeps a mass-based count instead of a
 *                               fixed one (below).
 * A row's order is: forced blocks (ascending id), then the other blocks by
 * descending score, exact ties to the lower id.  A row keeps a prefix of that
 * order of length c, written in ascending id:
 *  - without TOP_P, c = k_h;
 *  - with TOP_P, c = min(k_h, max(forced blocks in the row, 1, the shortest
 *    prefix length whose mass reaches top_p)), where the mass of block j is
 *    softmax_j(scale * s[b,h,i,j]) over all nb key blocks and scale =
 *    softmax_scale (<= 0: 1/sqrt(D)).
 * k_h = topk, or head_k[h] clamped to [1, topk] when head_k (device int32 [H])
 * is not NULL.  Forced blocks beyond k_h: the lowest ids are kept.
 */
#define SOL_SELECT_FORCE_DIAGONAL 1u
#define SOL_SELECT_FORCE_FIRST_FRAME 2u
#define SOL_SELECT_TOP_P 4u
typedef struct {
  unsigned flags;          /* OR of SOL_SELECT_* (0: plain top-k)           */
  float top_p;             /* in (0, 1], read with SOL_SELECT_TOP_P         */
  float softmax_scale;     /* top-p softmax scale, <= 0: 1/sqrt(D)          */
  const int32_t* head_k;   /* NULL, or device int32 [H] per-head k          */
  sol_tile tile;           /* {0,0,0}: blocks are runs of `block` tokens;
                              else the means are of these tiles (t*h*w ==
                              block) and the first-frame blocks are the
                              (grid_h/h)*(grid_w/w) tiles of the first layer */
} sol_select_opts;

/*
 * sol_block_select_pooled_ex -- sol_block_select_pooled with the variants above.
 *
 * idx_out    : int32 [B, H, nb, topk]; row (b,h,i) holds its c ids in ascending
 *              order, then topk - c entries of -1.
 * counts_out : int32 [B, H, nb], c per row (required: sol_sparse_attn_fwd_counts
 *              reads it).
 * opts       : host pointer, read during the call.  Unknown flags, top_p outside
 *              (0, 1] with TOP_P, or a non-finite softmax_scale: SOL_ERR_INVALID_ARG.
 * With opts->flags == 0 and head_k NULL, idx_out equals sol_block_select_pooled's
 * and every count is topk.  Other arguments and limits as sol_block_select_pooled.
 */
sol_status sol_block_select_pooled_ex(const float* qbar, const float* kbar, sol_shape s, int block, int topk,
                                      const sol_select_opts* opts, int32_t* idx_out, int32_t* counts_out,
                                      float* scores_out, cudaStream_t stream);

/*
 * sol_sparse_attn_fwd -- Sol-Attn block-sparse attention forward
 * (ai-feiten.nl, same section: attention restricted, per query, to the parts
 * that matter).
 *
 * For each query n of block i of (b, h), over the keys m < N of the blocks
 * idx[b,h,i,0..topk-1]:
 *   l_m = scale * q_n . k_m;  o_n = sum_m softmax(l)_m v_m;  lse_n = ln sum_m exp(l_m).
 * q, k, v : [B,N,H,D] (dtype dt).  idx : int32 [B,H,nb,topk], distinct ids in
 *           [0, nb) per row (any order).  An id outside [0, nb) is never used
 *           to address memory: the fp32 kernel skips it, the tensor-core
 *           kernels read block 0 in its place, and either way the device error
 *           word is set, which sol_check_device_status() reports as
 *           SOL_ERR_INVALID_ARG (the outputs of that call are then undefined).
 *           Repeated ids are not detected here: the block is attended once per
 *           occurrence.
 * o       : [B,N,H,D] (dtype dt).  lse : fp32 [B,H,N], natural log, scale included.
 * softmax_scale <= 0 selects 1/sqrt(D).
 * bf16: D == 128 and block == 128 (tcgen05 tensor-core kernel, fp32 accumulate,
 *       P rounded to bf16 for the PV product).
 * f32 : D in {64, 128}, any block (CUDA-core kernel, fp32 throughout).
 */
sol_status sol_sparse_attn_fwd(const void* q, const void* k, const void* v, const int32_t* idx,
                               sol_shape s, int block, int topk, float softmax_scale,
                               sol_dtype dt, void* o, float* lse, cudaStream_t stream);

/*
 * sol_sparse_attn_fwd_counts -- sol_sparse_attn_fwd where row (b,h,i) attends
 * to the key blocks idx[b,h,i,0 .. c-1] only, c = counts[b,h,i] clamped to
 * [1, topk] (the variable-length rows of sol_block_select_pooled_ex).
 *
 * counts : device int32 [B, H, nb], required (NULL: SOL_ERR_INVALID_ARG).
 * idx keeps its row stride topk; entries at and beyond c are not read.
 * Everything else as sol_sparse_attn_fwd; counts all equal to topk give its result.
 */
sol_status sol_sparse_attn_fwd_counts(const void* q, const void* k, const void* v, const int32_t* idx,
                                      const int32_t* counts, sol_shape s, int block, int topk,
                                      float softmax_scale, sol_dtype dt, void* o, float* lse,
                                      cudaStream_t stream);

/*
 * sol_qk_prologue_pool_tiled -- sol_qk_prologue_pool with 3-D tile blocks:
 * q_out, k_out are identical (tokens stay in place); qbar_out[b,h,i,:] is the
 * fp32 mean of the stored q_out over the tokens of tile i, summed in the
 * tile's raster order.  nb = N / (t*h*w).  Other arguments as
 * sol_qk_prologue_pool.
 */
sol_status sol_qk_prologue_pool_tiled(const void* q_raw, const void* k_raw, void* q_out, void* k_out,
                                      const float* gamma_q, const float* gamma_k, sol_shape s,
                                      int rope_dt, int rope_dh, int rope_dw, float rope_theta, float eps,
                                      sol_dtype dt, sol_tile tile, float* qbar_out, float* kbar_out,
                                      cudaStream_t stream);

/*
 * sol_sparse_attn_fwd_tiled -- sol_sparse_attn_fwd (counts == NULL) or
 * sol_sparse_attn_fwd_counts with 3-D tile blocks: the queries of tile i attend
 * to the keys of the tiles idx[b,h,i,0..c-1].  Tokens stay in place in q, k,
 * v and o (the kernel gathers each tile with one 5-D tensor-map copy); lse is
 * [B,H,N] by token.  bf16: t*h*w == 128.  Other arguments as
 * sol_sparse_attn_fwd_counts.
 */
sol_status sol_sparse_attn_fwd_tiled(const void* q, const void* k, const void* v, const int32_t* idx,
                                     const int32_t* counts, sol_shape s, sol_tile tile, int topk,
                                     float softmax_scale, sol_dtype dt, void* o, float* lse,
                                     cudaStream_t stream);

/*
 * Quantised exchange buffers for sequence-parallel runs (multi-GPU runs of the
 * Sol-H3 runtime move Q, K, V as INT8 and the attention output as FP8, about
 * half the inter-GPU bytes: ai-feiten.nl, "Videomodel MiniMax-H3 rendert
 * sneller dan afspelen", "Waar de snelheidswinst vandaan komt").
 *
 * A row is the D bf16 channels of one (b, n, h).  Its fp32 scale is
 * s = max|x| / L (L = 127 INT8, 448 e4m3); its codes are x * r with
 * r = L / max|x| (one fp32 division per row, one fp32 product per value)
 * rounded to nearest even, INT8 clamped to [-127, 127], e4m3 saturating at
 * +-448; an all-zero row has s = 0 and zero codes.  Dequantised
 * values are bf16_rn(code * s) (one fp32 product).
 *
 * sol_quant_pack: x bf16 [B, N, H, D] -> codes (1 byte each) [G][B][Nc][Hc][D]
 *   and scales fp32 [G][B][Nc][Hc], slice g holding what rank g receives:
 *   SOL_SPLIT_HEADS  (token shard -> head shards): Hc = H/G, Nc = N, heads
 *                    g*Hc .. g*Hc+Hc-1 (H % G == 0);
 *   SOL_SPLIT_TOKENS (head shard -> token shards): Nc = N/G, Hc = H, tokens
 *                    g*Nc .. g*Nc+Nc-1 (N % G == 0).
 *   Slice g starts at row g * g_stride_rows of both buffers (0: B*Nc*Hc,
 *   dense), so several tensors can share one exchange buffer.
 * sol_dequant_unpack: codes / scales [G][B][Nc][Hc] (slice g from rank g, same
 *   g_stride_rows rule) -> out bf16: SOL_SPLIT_HEADS concatenates the slices
 *   along tokens, out [B, G*Nc, Hc, D] (token g*Nc + n); SOL_SPLIT_TOKENS
 *   along heads, out [B, Nc, G*Hc, D] (head g*Hc + h).
 * D in {64, 128}; x, out and codes 16-byte aligned, scales 4-byte aligned (device memory).
 */
typedef enum { SOL_CODE_INT8 = 0, SOL_CODE_E4M3 = 1 } sol_code;
typedef enum { SOL_SPLIT_HEADS = 0, SOL_SPLIT_TOKENS = 1 } sol_split;
sol_status sol_quant_pack(const void* x, int B, int N, int H, int D, int G, sol_split split, sol_code code,
                          void* codes_out, float* scales_out, long long g_stride_rows, cudaStream_t stream);
sol_status sol_dequant_unpack(const void* codes, const float* scales, int B, int Nc, int Hc, int D, int G,
                              sol_split split, sol_code code, void* out, long long g_stride_rows,
                              cudaStream_t stream);

/*
 * FP8 (e4m3) attention -- the Sol-Attn forward on e4m3 operands (the pages'
 * runtime uses FP8 on its hot paths: ai-feiten.nl, "Videomodel MiniMax-H3
 * rendert sneller dan afspelen", "Waar de snelheidswinst vandaan komt"; the
 * formats are this library's).
 *
 * sol_quant_attn_fp8: bf16 q, k, v [B,N,H,D] (D == 128, N % 16 == 0) ->
 *   q8, k8      e4m3 codes [B,N,H,D]; q_scale fp32 [B,H,N], one per (token,
 *               head) row; k_scale fp32 [B,H,nb], one per (b, h, block of 128
 *               tokens): s = max|x| over the row or block / 448, codes
 *               x * (448 / max|x|) rounded to nearest even (all zero: s = 0,
 *               zero codes);
 *   vt8         e4m3 codes of V transposed, [B,H,D,N], the keys of every
 *               aligned group of 16 stored in the order
 *               0 1 8 9 2 3 10 11 4 5 12 13 6 7 14 15;
 *   v_scale     fp32 [B,H], one per (b, h): s = max|v| / 448 over all tokens
 *               and channels, codes v * (448 / max|v|);
 *   workspace   device scratch of sol_quant_attn_fp8_workspace_bytes(s).
 *   q_scale, k_scale 8-byte aligned; the others 16-byte aligned.
 * sol_sparse_attn_fwd_fp8: the attention of sol_sparse_attn_fwd(_counts) on
 *   the dequantised q = q8 * q_scale, k = k8 * k_scale, v = vt8^T * v_scale,
 *   with e4m3 tensor-core products (fp32 accumulation) and the softmax weights
 *   rounded to e4m3 for the P V product (relative error 2^-4 per weight; the
 *   normaliser uses the unrounded weights).  counts may be NULL (every row uses
 *   topk blocks).  block == 128; o bf16 [B,N,H,D], lse fp32 [B,H,N].
 */
size_t sol_quant_attn_fp8_workspace_bytes(sol_shape s);
sol_status sol_quant_attn_fp8(const void* q, const void* k, const void* v, sol_shape s, void* q8, float* q_scale,
                              void* k8, float* k_scale, void* vt8, float* v_scale, void* workspace,
                              size_t workspace_bytes, cudaStream_t stream);
sol_status sol_sparse_attn_fwd_fp8(const void* q8, const float* q_scale, const void* k8, const float* k_scale,
                                   const void* vt8, const float* v_scale, const int32_t* idx, const int32_t* counts,
                                   sol_shape s, int block, int topk, float softmax_scale, void* o, float* lse,
                                   cudaStream_t stream);

/*
 * sol_sparse_attn_bwd -- gradients of sol_sparse_attn_fwd(_counts) (the method is
 * used for inference; provided for completeness).  With P the softmax of
 * scale * q k^T over the kept keys, recomputed from the forward's lse:
 *   delta_n = do_n . o_n;  dS = P (do . v^T - delta);
 *   dq = scale dS k;  dk = scale dS^T q;  dv = P^T do
 * summed over every query block that kept a key block.
 * q, k, v, o, dout : [B,N,H,D] (dtype dt); lse fp32 [B,H,N] from the forward;
 * idx, counts (nullable) as for the forward; dq, dk, dv fp32 [B,N,H,D].
 * A row that repeats an id, or holds an id outside [0, nb), sets the device
 * error word (sol_check_device_status() then returns SOL_ERR_INVALID_ARG) and
 * the gradients of that call are undefined: the inverted index behind dk and
 * dv records each (query block, key block) pair once.
 * workspace: sol_sparse_attn_bwd_workspace_bytes() (delta and the inverted
 * selection index).  D in {64, 128}, any block; CUDA-core kernels, fp32 math;
 * deterministic (no atomics).
 */
size_t sol_sparse_attn_bwd_workspace_bytes(sol_shape s, int block);
sol_status sol_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dout, const int32_t* idx, const int32_t* counts, sol_shape s, int block,
                               int topk, float softmax_scale, sol_dtype dt, float* dq, float* dk, float* dv,
                               void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * sol_block_select_noalloc -- sol_block_select for callers that cannot
 * allocate device memory.  No counterpart on the pages: this is a convenience
 * of this library.
 *
 * Some callers cannot call cudaMalloc: code running inside a host framework's
 * launch callback or plugin hook that owns all device memory and forbids
 * allocation there, and latency-critical loops where an allocation (which may
 * synchronise the device) is not acceptable.  This entry point takes the same
 * inputs and outputs as sol_block_select but needs no workspace: its scratch
 * (the pooled means of Q and K) lives in one file-scope device array of
 * SOL_NOALLOC_SCRATCH_BYTES inside libsol, which every GPU that loads the
 * library holds until the process exits.
 *  - Size limit: shapes whose sol_block_select_workspace_bytes() exceeds
 *    SOL_NOALLOC_SCRATCH_BYTES are rejected with SOL_ERR_UNSUPPORTED before
 *    anything is launched (the five video workloads need at most 33.4 MB).
 *  - First call per device: it looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current and caches it together
 *    with the id of the current CUDA context; make that first call before any
 *    stream capture.  If the context changes (cudaDeviceReset, or another
 *    teardown of the device's primary context, followed by new work), the next
 *    call sees a new context id and looks the address up again: that call,
 *    too, must come before any stream capture.  A failed lookup returns
 *    SOL_ERR_CUDA.
 *  - Sharing: every call on a device uses the same array and it keeps the
 *    last call's contents.  Nothing in it needs to start at zero (the pooling
 *    kernel overwrites every byte it later reads), but calls that overlap on
 *    the GPU (different streams, or different host threads) race on it:
 *    serialise them.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 */
#define SOL_NOALLOC_SCRATCH_BYTES (40u * 1024u * 1024u)
sol_status sol_block_select_noalloc(const void* q, const void* k, sol_shape s, int block, int topk,
                                    sol_dtype dt, int32_t* idx_out, float* scores_out,
                                    cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns SOL_ERR_TIMEOUT if a bounded device wait ran out since the last
 * check, SOL_ERR_CUDA if the stream reports a CUDA error, else SOL_OK. */
sol_status sol_check_device_status(cudaStream_t stream);

/* Launches one thread that waits on a barrier nothing will complete, bounded
 * by limit_us (1..1000000) microseconds, so that the timeout path can be
 * exercised without a hang.  The following sol_check_device_status() on the
 * same stream returns SOL_ERR_TIMEOUT.  No counterpart on the pages: this is a
 * self-test of the library's failure detection. */
sol_status sol_selftest_wait_timeout(unsigned limit_us, cudaStream_t stream);

/* Static, human-readable name of a status code. */
const char* sol_status_string(sol_status status);

#ifdef __cplusplus
}
#endif
#endif /* SOL_H_ */
