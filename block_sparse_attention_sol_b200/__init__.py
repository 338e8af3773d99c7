"""Python binding of libsol, the sm_100a Sol-Attn hot path (see include/sol.h).

Argument marshalling only: every step runs in the CUDA kernels of libsol.so.
PyTorch provides device memory and the current stream.  There is no fallback:
if the library is missing this import fails, and every call checks that its
tensors live on a CUDA device.

Functions (same names as the C ABI):
    sol_qk_prologue(q_raw, k_raw, gamma_q, gamma_k, grid, ...)  -> (q, k)
    sol_block_select(q, k, grid, block, topk, ...)              -> idx [, scores]
    sol_sparse_attn_fwd(q, k, v, idx, grid, block, ...)         -> (o, lse)
    sol_qk_prologue_pool(q_raw, k_raw, gamma_q, gamma_k, grid, block, ...) -> (q, k, qbar, kbar)
    sol_block_select_pooled(qbar, kbar, grid, block, topk, ...) -> idx [, scores]
    sol_block_select_pooled_ex(qbar, kbar, grid, block, topk, flags=..., ...) -> (idx, counts) [, scores]
    sol_sparse_attn_fwd_counts(q, k, v, idx, counts, grid, block, ...) -> (o, lse)
    sol_qk_prologue_pool_tiled(q_raw, k_raw, gamma_q, gamma_k, grid, tile, ...) -> (q, k, qbar, kbar)
    sol_sparse_attn_fwd_tiled(q, k, v, idx, grid, tile, counts=None, ...) -> (o, lse)
    sol_quant_pack(x, G, split, code, codes_out, scales_out, ...)  (exchange buffers)
    sol_dequant_unpack(codes, scales, B, Nc, Hc, D, G, split, code, out, ...)
    sol_quant_attn_fp8(q, k, v, grid) -> dict of e4m3 codes and scales
    sol_sparse_attn_fwd_fp8(fp8_inputs, idx, grid, block, counts=None, ...) -> (o, lse)
    sol_sparse_attn_bwd(q, k, v, o, lse, dout, idx, grid, block, counts=None, ...) -> (dq, dk, dv) fp32
    sol_check_device_status(stream=None)
    sol_selftest_wait_timeout(limit_us, stream=None)
    sol_block_select_workspace_bytes(shape, block)
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "SolError", "SolShape", "LIB_PATH", "lib",
    "sol_qk_prologue", "sol_block_select", "sol_block_select_workspace_bytes", "sol_sparse_attn_fwd",
    "sol_qk_prologue_pool", "sol_block_select_pooled", "sol_block_select_pooled_ex", "sol_sparse_attn_fwd_counts",
    "SolSelectOpts", "SolTile", "sol_quant_pack", "sol_dequant_unpack", "sol_quant_attn_fp8", "sol_sparse_attn_fwd_fp8", "sol_sparse_attn_bwd",
    "SOL_CODE_INT8", "SOL_CODE_E4M3", "SOL_SPLIT_HEADS", "SOL_SPLIT_TOKENS", "sol_qk_prologue_pool_tiled", "sol_sparse_attn_fwd_tiled", "SOL_SELECT_FORCE_DIAGONAL", "SOL_SELECT_FORCE_FIRST_FRAME", "SOL_SELECT_TOP_P",
    "sol_check_device_status", "sol_selftest_wait_timeout", "sol_status_string", "sol_attention_chain",
    "sol_attention_chain_fused",
    "SOL_OK", "SOL_ERR_INVALID_ARG", "SOL_ERR_UNSUPPORTED", "SOL_ERR_CUDA", "SOL_ERR_TIMEOUT",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsol.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python block_sparse_attention_sol_b200/build.py` "
        "(there is no non-CUDA fallback)")
lib = ctypes.CDLL(LIB_PATH)

SOL_OK, SOL_ERR_INVALID_ARG, SOL_ERR_UNSUPPORTED, SOL_ERR_CUDA, SOL_ERR_TIMEOUT = range(5)
SOL_F32, SOL_BF16 = 0, 1
SOL_SELECT_FORCE_DIAGONAL, SOL_SELECT_FORCE_FIRST_FRAME, SOL_SELECT_TOP_P = 1, 2, 4
SOL_CODE_INT8, SOL_CODE_E4M3 = 0, 1
SOL_SPLIT_HEADS, SOL_SPLIT_TOKENS = 0, 1


class SolShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "N", "H", "D", "grid_t", "grid_h", "grid_w")]


class SolTile(ctypes.Structure):
    _fields_ = [("t", ctypes.c_int), ("h", ctypes.c_int), ("w", ctypes.c_int)]


class SolSelectOpts(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint), ("top_p", ctypes.c_float), ("softmax_scale", ctypes.c_float),
                ("head_k", ctypes.c_void_p), ("tile", SolTile)]


class SolError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {sol_status_string(status)}")


_P, _I, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
lib.sol_status_string.restype = ctypes.c_char_p
lib.sol_status_string.argtypes = [_I]
lib.sol_qk_prologue.restype = _I
lib.sol_qk_prologue.argtypes = [_P, _P, _P, _P, _P, _P, SolShape, _I, _I, _I, _F, _F, _I, _P]
lib.sol_block_select_workspace_bytes.restype = _SZ
lib.sol_block_select_workspace_bytes.argtypes = [SolShape, _I]
lib.sol_block_select.restype = _I
lib.sol_block_select.argtypes = [_P, _P, SolShape, _I, _I, _I, _P, _P, _P, _SZ, _P]
lib.sol_qk_prologue_pool.restype = _I
lib.sol_qk_prologue_pool.argtypes = [_P, _P, _P, _P, _P, _P, SolShape, _I, _I, _I, _F, _F, _I, _I, _P, _P, _P]
lib.sol_block_select_pooled.restype = _I
lib.sol_block_select_pooled.argtypes = [_P, _P, SolShape, _I, _I, _P, _P, _P]
lib.sol_block_select_pooled_ex.restype = _I
lib.sol_block_select_pooled_ex.argtypes = [_P, _P, SolShape, _I, _I, ctypes.POINTER(SolSelectOpts), _P, _P, _P, _P]
lib.sol_sparse_attn_fwd_counts.restype = _I
lib.sol_sparse_attn_fwd_counts.argtypes = [_P, _P, _P, _P, _P, SolShape, _I, _I, _F, _I, _P, _P, _P]
lib.sol_qk_prologue_pool_tiled.restype = _I
lib.sol_qk_prologue_pool_tiled.argtypes = [_P, _P, _P, _P, _P, _P, SolShape, _I, _I, _I, _F, _F, _I, SolTile, _P, _P,
                                           _P]
lib.sol_sparse_attn_fwd_tiled.restype = _I
lib.sol_sparse_attn_fwd_tiled.argtypes = [_P, _P, _P, _P, _P, SolShape, SolTile, _I, _F, _I, _P, _P, _P]
lib.sol_quant_pack.restype = _I
lib.sol_quant_pack.argtypes = [_P, _I, _I, _I, _I, _I, _I, _I, _P, _P, ctypes.c_longlong, _P]
lib.sol_dequant_unpack.restype = _I
lib.sol_dequant_unpack.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, ctypes.c_longlong, _P]
lib.sol_quant_attn_fp8_workspace_bytes.restype = _SZ
lib.sol_quant_attn_fp8_workspace_bytes.argtypes = [SolShape]
lib.sol_quant_attn_fp8.restype = _I
lib.sol_quant_attn_fp8.argtypes = [_P, _P, _P, SolShape, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
lib.sol_sparse_attn_fwd_fp8.restype = _I
lib.sol_sparse_attn_fwd_fp8.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, SolShape, _I, _I, _F, _P, _P, _P]
lib.sol_sparse_attn_bwd_workspace_bytes.restype = _SZ
lib.sol_sparse_attn_bwd_workspace_bytes.argtypes = [SolShape, _I]
lib.sol_sparse_attn_bwd.restype = _I
lib.sol_sparse_attn_bwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, SolShape, _I, _I, _F, _I, _P, _P, _P, _P, _SZ, _P]
lib.sol_sparse_attn_fwd.restype = _I
lib.sol_sparse_attn_fwd.argtypes = [_P, _P, _P, _P, SolShape, _I, _I, _F, _I, _P, _P, _P]
lib.sol_check_device_status.restype = _I
lib.sol_check_device_status.argtypes = [_P]
lib.sol_selftest_wait_timeout.restype = _I
lib.sol_selftest_wait_timeout.argtypes = [ctypes.c_uint, _P]


def sol_status_string(status: int) -> str:
    return lib.sol_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != SOL_OK:
        raise SolError(status, what)


def _stream_handle(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SOL_BF16
    if t.dtype == torch.float32:
        return SOL_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _cuda(t: torch.Tensor, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _shape(x: torch.Tensor, grid) -> SolShape:
    if x.dim() != 4:
        raise ValueError("activations are [B, N, H, D]")
    B, N, H, D = x.shape
    return SolShape(B, N, H, D, int(grid[0]), int(grid[1]), int(grid[2]))


def sol_qk_prologue(q_raw, k_raw, gamma_q, gamma_k, grid, rope_split=None, rope_theta=10000.0, eps=1e-6,
                    q_out=None, k_out=None, stream=None):
    """Fused QK-RMSNorm + 3D RoPE.  Returns (q, k) with q_raw's shape and dtype."""
    _cuda(q_raw, "q_raw"), _cuda(k_raw, "k_raw"), _cuda(gamma_q, "gamma_q"), _cuda(gamma_k, "gamma_k")
    s = _shape(q_raw, grid)
    if rope_split is None:
        dh = 2 * (s.D // 6)
        rope_split = (s.D - 2 * dh, dh, dh)
    q_out = torch.empty_like(q_raw) if q_out is None else _cuda(q_out, "q_out")
    k_out = torch.empty_like(k_raw) if k_out is None else _cuda(k_out, "k_out")
    st = lib.sol_qk_prologue(q_raw.data_ptr(), k_raw.data_ptr(), q_out.data_ptr(), k_out.data_ptr(),
                             gamma_q.data_ptr(), gamma_k.data_ptr(), s, int(rope_split[0]), int(rope_split[1]),
                             int(rope_split[2]), float(rope_theta), float(eps), _dtype_code(q_raw),
                             _stream_handle(stream))
    _check(st, "sol_qk_prologue")
    return q_out, k_out


def sol_qk_prologue_pool(q_raw, k_raw, gamma_q, gamma_k, grid, block, rope_split=None, rope_theta=10000.0,
                         eps=1e-6, q_out=None, k_out=None, qbar_out=None, kbar_out=None, stream=None):
    """sol_qk_prologue plus the fp32 block means of its stored outputs.
    Returns (q, k, qbar, kbar); qbar, kbar are [B, H, nb, D]."""
    _cuda(q_raw, "q_raw"), _cuda(k_raw, "k_raw"), _cuda(gamma_q, "gamma_q"), _cuda(gamma_k, "gamma_k")
    s = _shape(q_raw, grid)
    if rope_split is None:
        dh = 2 * (s.D // 6)
        rope_split = (s.D - 2 * dh, dh, dh)
    nb = -(-s.N // block)
    q_out = torch.empty_like(q_raw) if q_out is None else _cuda(q_out, "q_out")
    k_out = torch.empty_like(k_raw) if k_out is None else _cuda(k_out, "k_out")
    pooled = (s.B, s.H, nb, s.D)
    qbar_out = (torch.empty(pooled, dtype=torch.float32, device=q_raw.device) if qbar_out is None
                else _cuda(qbar_out, "qbar_out"))
    kbar_out = (torch.empty(pooled, dtype=torch.float32, device=q_raw.device) if kbar_out is None
                else _cuda(kbar_out, "kbar_out"))
    st = lib.sol_qk_prologue_pool(q_raw.data_ptr(), k_raw.data_ptr(), q_out.data_ptr(), k_out.data_ptr(),
                                  gamma_q.data_ptr(), gamma_k.data_ptr(), s, int(rope_split[0]), int(rope_split[1]),
                                  int(rope_split[2]), float(rope_theta), float(eps), _dtype_code(q_raw), int(block),
                                  qbar_out.data_ptr(), kbar_out.data_ptr(), _stream_handle(stream))
    _check(st, "sol_qk_prologue_pool")
    return q_out, k_out, qbar_out, kbar_out


def sol_qk_prologue_pool_tiled(q_raw, k_raw, gamma_q, gamma_k, grid, tile, rope_split=None, rope_theta=10000.0,
                               eps=1e-6, q_out=None, k_out=None, qbar_out=None, kbar_out=None, stream=None):
    """sol_qk_prologue plus the fp32 means of its stored outputs over 3-D tiles
    tile = (t, h, w).  Returns (q, k, qbar, kbar); qbar, kbar are [B, H, N / (t h w), D]."""
    _cuda(q_raw, "q_raw"), _cuda(k_raw, "k_raw"), _cuda(gamma_q, "gamma_q"), _cuda(gamma_k, "gamma_k")
    s = _shape(q_raw, grid)
    if rope_split is None:
        dh = 2 * (s.D // 6)
        rope_split = (s.D - 2 * dh, dh, dh)
    block = int(tile[0]) * int(tile[1]) * int(tile[2])
    nb = max(s.N // block, 1)
    q_out = torch.empty_like(q_raw) if q_out is None else _cuda(q_out, "q_out")
    k_out = torch.empty_like(k_raw) if k_out is None else _cuda(k_out, "k_out")
    pooled = (s.B, s.H, nb, s.D)
    qbar_out = (torch.empty(pooled, dtype=torch.float32, device=q_raw.device) if qbar_out is None
                else _cuda(qbar_out, "qbar_out"))
    kbar_out = (torch.empty(pooled, dtype=torch.float32, device=q_raw.device) if kbar_out is None
                else _cuda(kbar_out, "kbar_out"))
    st = lib.sol_qk_prologue_pool_tiled(q_raw.data_ptr(), k_raw.data_ptr(), q_out.data_ptr(), k_out.data_ptr(),
                                        gamma_q.data_ptr(), gamma_k.data_ptr(), s, int(rope_split[0]),
                                        int(rope_split[1]), int(rope_split[2]), float(rope_theta), float(eps),
                                        _dtype_code(q_raw), SolTile(*(int(x) for x in tile)), qbar_out.data_ptr(),
                                        kbar_out.data_ptr(), _stream_handle(stream))
    _check(st, "sol_qk_prologue_pool_tiled")
    return q_out, k_out, qbar_out, kbar_out


def sol_block_select_pooled(qbar, kbar, grid, block, topk, idx_out=None, return_scores=False, stream=None):
    """Scores + top-k from block means [B, H, nb, D] (fp32).  Returns idx (and the scores)."""
    _cuda(qbar, "qbar"), _cuda(kbar, "kbar")
    if qbar.dtype != torch.float32 or kbar.dtype != torch.float32:
        raise TypeError("qbar and kbar must be float32")
    B, H, nb, D = qbar.shape
    N = int(grid[0]) * int(grid[1]) * int(grid[2])
    s = SolShape(B, N, H, D, int(grid[0]), int(grid[1]), int(grid[2]))
    if idx_out is None:
        idx_out = torch.empty((B, H, nb, topk), dtype=torch.int32, device=qbar.device)
    scores = torch.empty((B, H, nb, nb), dtype=torch.float32, device=qbar.device) if return_scores else None
    st = lib.sol_block_select_pooled(qbar.data_ptr(), kbar.data_ptr(), s, int(block), int(topk),
                                     _cuda(idx_out, "idx_out").data_ptr(),
                                     scores.data_ptr() if scores is not None else None, _stream_handle(stream))
    _check(st, "sol_block_select_pooled")
    return (idx_out, scores) if return_scores else idx_out


def sol_block_select_pooled_ex(qbar, kbar, grid, block, topk, flags=0, top_p=1.0, softmax_scale=0.0, head_k=None,
                               tile=None, idx_out=None, counts_out=None, return_scores=False, stream=None):
    """Selection variants (forced diagonal / first-frame blocks, top-p, per-head k)
    from block means.  Returns (idx, counts) (and the scores); rows of idx hold
    their count of ascending ids, then -1."""
    _cuda(qbar, "qbar"), _cuda(kbar, "kbar")
    if qbar.dtype != torch.float32 or kbar.dtype != torch.float32:
        raise TypeError("qbar and kbar must be float32")
    B, H, nb, D = qbar.shape
    N = int(grid[0]) * int(grid[1]) * int(grid[2])
    s = SolShape(B, N, H, D, int(grid[0]), int(grid[1]), int(grid[2]))
    if head_k is not None:
        _cuda(head_k, "head_k")
        if head_k.dtype != torch.int32 or head_k.numel() != H:
            raise ValueError("head_k must be int32 [H]")
    if idx_out is None:
        idx_out = torch.empty((B, H, nb, topk), dtype=torch.int32, device=qbar.device)
    if counts_out is None:
        counts_out = torch.empty((B, H, nb), dtype=torch.int32, device=qbar.device)
    scores = torch.empty((B, H, nb, nb), dtype=torch.float32, device=qbar.device) if return_scores else None
    opts = SolSelectOpts(int(flags), float(top_p), float(softmax_scale),
                         head_k.data_ptr() if head_k is not None else None,
                         SolTile(*(int(x) for x in tile)) if tile is not None else SolTile(0, 0, 0))
    st = lib.sol_block_select_pooled_ex(qbar.data_ptr(), kbar.data_ptr(), s, int(block), int(topk),
                                        ctypes.byref(opts), _cuda(idx_out, "idx_out").data_ptr(),
                                        _cuda(counts_out, "counts_out").data_ptr(),
                                        scores.data_ptr() if scores is not None else None, _stream_handle(stream))
    _check(st, "sol_block_select_pooled_ex")
    return (idx_out, counts_out, scores) if return_scores else (idx_out, counts_out)


def sol_block_select_workspace_bytes(shape: SolShape, block: int) -> int:
    return int(lib.sol_block_select_workspace_bytes(shape, int(block)))


def sol_block_select(q, k, grid, block, topk, workspace=None, idx_out=None, return_scores=False, stream=None):
    """Block mean-pool + pooled dot-product scores + top-k.  Returns idx int32
    [B, H, nb, topk] (and the fp32 score matrix when return_scores)."""
    _cuda(q, "q"), _cuda(k, "k")
    s = _shape(q, grid)
    nb = -(-s.N // block)
    need = sol_block_select_workspace_bytes(s, block)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _cuda(workspace, "workspace")
    if idx_out is None:
        idx_out = torch.empty((s.B, s.H, nb, topk), dtype=torch.int32, device=q.device)
    scores = torch.empty((s.B, s.H, nb, nb), dtype=torch.float32, device=q.device) if return_scores else None
    st = lib.sol_block_select(q.data_ptr(), k.data_ptr(), s, int(block), int(topk), _dtype_code(q),
                              _cuda(idx_out, "idx_out").data_ptr(), scores.data_ptr() if scores is not None else None,
                              workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                              _stream_handle(stream))
    _check(st, "sol_block_select")
    return (idx_out, scores) if return_scores else idx_out


def sol_sparse_attn_fwd(q, k, v, idx, grid, block, softmax_scale=0.0, o=None, lse=None, stream=None):
    """Exact softmax attention over the kept blocks.  Returns (o, lse)."""
    _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), _cuda(idx, "idx")
    if idx.dtype != torch.int32:
        raise TypeError("idx must be int32")
    s = _shape(q, grid)
    topk = idx.shape[-1]
    o = torch.empty_like(q) if o is None else _cuda(o, "o")
    lse = torch.empty((s.B, s.H, s.N), dtype=torch.float32, device=q.device) if lse is None else _cuda(lse, "lse")
    st = lib.sol_sparse_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), s, int(block), int(topk),
                                 float(softmax_scale), _dtype_code(q), o.data_ptr(), lse.data_ptr(),
                                 _stream_handle(stream))
    _check(st, "sol_sparse_attn_fwd")
    return o, lse


def sol_sparse_attn_fwd_counts(q, k, v, idx, counts, grid, block, softmax_scale=0.0, o=None, lse=None, stream=None):
    """sol_sparse_attn_fwd where row (b, h, i) uses only its first counts[b, h, i] ids."""
    _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), _cuda(idx, "idx"), _cuda(counts, "counts")
    if idx.dtype != torch.int32 or counts.dtype != torch.int32:
        raise TypeError("idx and counts must be int32")
    s = _shape(q, grid)
    topk = idx.shape[-1]
    o = torch.empty_like(q) if o is None else _cuda(o, "o")
    lse = torch.empty((s.B, s.H, s.N), dtype=torch.float32, device=q.device) if lse is None else _cuda(lse, "lse")
    st = lib.sol_sparse_attn_fwd_counts(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(), counts.data_ptr(),
                                        s, int(block), int(topk), float(softmax_scale), _dtype_code(q), o.data_ptr(),
                                        lse.data_ptr(), _stream_handle(stream))
    _check(st, "sol_sparse_attn_fwd_counts")
    return o, lse


def sol_sparse_attn_fwd_tiled(q, k, v, idx, grid, tile, counts=None, softmax_scale=0.0, o=None, lse=None,
                              stream=None):
    """Attention over 3-D tile blocks tile = (t, h, w) (optionally count-limited rows).  Returns (o, lse)."""
    _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v"), _cuda(idx, "idx")
    if idx.dtype != torch.int32 or (counts is not None and counts.dtype != torch.int32):
        raise TypeError("idx and counts must be int32")
    s = _shape(q, grid)
    topk = idx.shape[-1]
    o = torch.empty_like(q) if o is None else _cuda(o, "o")
    lse = torch.empty((s.B, s.H, s.N), dtype=torch.float32, device=q.device) if lse is None else _cuda(lse, "lse")
    st = lib.sol_sparse_attn_fwd_tiled(q.data_ptr(), k.data_ptr(), v.data_ptr(), idx.data_ptr(),
                                       _cuda(counts, "counts").data_ptr() if counts is not None else None, s,
                                       SolTile(*(int(x) for x in tile)), int(topk), float(softmax_scale),
                                       _dtype_code(q), o.data_ptr(), lse.data_ptr(), _stream_handle(stream))
    _check(st, "sol_sparse_attn_fwd_tiled")
    return o, lse


def sol_quant_pack(x, G, split, code, codes_out, scales_out, g_stride_rows=0, stream=None):
    """Quantise bf16 rows x [B, N, H, D] into per-destination slices (see include/sol.h).
    codes_out (uint8) and scales_out (float32) are caller buffers, slice g at row g * g_stride_rows."""
    _cuda(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 4:
        raise TypeError("x must be bf16 [B, N, H, D]")
    if codes_out.dtype != torch.uint8 or scales_out.dtype != torch.float32:
        raise TypeError("codes_out must be uint8 and scales_out float32")
    B, N, H, D = x.shape
    st = lib.sol_quant_pack(x.data_ptr(), B, N, H, D, int(G), int(split), int(code), _cuda(codes_out, "codes_out").data_ptr(),
                            _cuda(scales_out, "scales_out").data_ptr(), int(g_stride_rows), _stream_handle(stream))
    _check(st, "sol_quant_pack")


def sol_dequant_unpack(codes, scales, B, Nc, Hc, D, G, split, code, out, g_stride_rows=0, stream=None):
    """Dequantise G received slices into bf16 out (tokens or heads concatenated; see include/sol.h)."""
    _cuda(codes, "codes"), _cuda(scales, "scales"), _cuda(out, "out")
    if out.dtype != torch.bfloat16:
        raise TypeError("out must be bf16")
    st = lib.sol_dequant_unpack(codes.data_ptr(), scales.data_ptr(), int(B), int(Nc), int(Hc), int(D), int(G), int(split),
                                int(code), out.data_ptr(), int(g_stride_rows), _stream_handle(stream))
    _check(st, "sol_dequant_unpack")


def sol_quant_attn_fp8(q, k, v, grid, out=None, stream=None):
    """e4m3 codes and scales of bf16 q, k, v [B, N, H, D] for sol_sparse_attn_fwd_fp8 (layouts in include/sol.h).
    Returns a dict: q8, q_scale [B, H, N], k8, k_scale [B, H, nb], vt8 [B, H, D, N], v_scale [B, H]."""
    _cuda(q, "q"), _cuda(k, "k"), _cuda(v, "v")
    if q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16 or v.dtype != torch.bfloat16:
        raise TypeError("q, k, v must be bf16")
    s = _shape(q, grid)
    dev = q.device
    if out is None:
        out = {"q8": torch.empty(q.shape, dtype=torch.uint8, device=dev),
               "k8": torch.empty(k.shape, dtype=torch.uint8, device=dev),
               "vt8": torch.empty((s.B, s.H, s.D, s.N), dtype=torch.uint8, device=dev),
               "q_scale": torch.empty((s.B, s.H, s.N), dtype=torch.float32, device=dev),
               "k_scale": torch.empty((s.B, s.H, -(-s.N // 128)), dtype=torch.float32, device=dev),
               "v_scale": torch.empty((s.B, s.H), dtype=torch.float32, device=dev)}
        ws = max(int(lib.sol_quant_attn_fp8_workspace_bytes(s)), 16)
        out["workspace"] = torch.empty(ws, dtype=torch.uint8, device=dev)
    st = lib.sol_quant_attn_fp8(q.data_ptr(), k.data_ptr(), v.data_ptr(), s, out["q8"].data_ptr(),
                                out["q_scale"].data_ptr(), out["k8"].data_ptr(), out["k_scale"].data_ptr(),
                                out["vt8"].data_ptr(), out["v_scale"].data_ptr(), out["workspace"].data_ptr(),
                                out["workspace"].numel(), _stream_handle(stream))
    _check(st, "sol_quant_attn_fp8")
    return out


def sol_sparse_attn_fwd_fp8(fp8, idx, grid, block, counts=None, softmax_scale=0.0, o=None, lse=None, stream=None):
    """Attention on e4m3 operands (fp8: the dict of sol_quant_attn_fp8, or the same keys).  Returns (o bf16, lse)."""
    for n in ("q8", "k8", "vt8", "q_scale", "k_scale", "v_scale"):
        _cuda(fp8[n], n)
    _cuda(idx, "idx")
    if idx.dtype != torch.int32 or (counts is not None and counts.dtype != torch.int32):
        raise TypeError("idx and counts must be int32")
    q8 = fp8["q8"]
    B, N, H, D = q8.shape
    s = SolShape(B, N, H, D, int(grid[0]), int(grid[1]), int(grid[2]))
    o = torch.empty((B, N, H, D), dtype=torch.bfloat16, device=q8.device) if o is None else _cuda(o, "o")
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device) if lse is None else _cuda(lse, "lse")
    st = lib.sol_sparse_attn_fwd_fp8(q8.data_ptr(), fp8["q_scale"].data_ptr(), fp8["k8"].data_ptr(),
                                     fp8["k_scale"].data_ptr(), fp8["vt8"].data_ptr(), fp8["v_scale"].data_ptr(),
                                     idx.data_ptr(), _cuda(counts, "counts").data_ptr() if counts is not None else None,
                                     s, int(block), int(idx.shape[-1]), float(softmax_scale), o.data_ptr(),
                                     lse.data_ptr(), _stream_handle(stream))
    _check(st, "sol_sparse_attn_fwd_fp8")
    return o, lse


def sol_sparse_attn_bwd(q, k, v, o, lse, dout, idx, grid, block, counts=None, softmax_scale=0.0, workspace=None,
                        stream=None):
    """Gradients of the block-sparse attention.  Returns (dq, dk, dv) fp32 [B, N, H, D]."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (lse, "lse"), (dout, "dout"), (idx, "idx")):
        _cuda(t, n)
    if idx.dtype != torch.int32 or (counts is not None and counts.dtype != torch.int32):
        raise TypeError("idx and counts must be int32")
    s = _shape(q, grid)
    need = int(lib.sol_sparse_attn_bwd_workspace_bytes(s, int(block)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    dq, dk, dv = (torch.empty(q.shape, dtype=torch.float32, device=q.device) for _ in range(3))
    st = lib.sol_sparse_attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                 dout.data_ptr(), idx.data_ptr(),
                                 _cuda(counts, "counts").data_ptr() if counts is not None else None, s, int(block),
                                 int(idx.shape[-1]), float(softmax_scale), _dtype_code(q), dq.data_ptr(), dk.data_ptr(),
                                 dv.data_ptr(), _cuda(workspace, "workspace").data_ptr(), workspace.numel(),
                                 _stream_handle(stream))
    _check(st, "sol_sparse_attn_bwd")
    return dq, dk, dv


def sol_check_device_status(stream=None) -> int:
    """Synchronises the stream; returns the library status code (SOL_OK, SOL_ERR_TIMEOUT, ...)."""
    return int(lib.sol_check_device_status(_stream_handle(stream)))


def sol_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    _check(lib.sol_selftest_wait_timeout(int(limit_us), _stream_handle(stream)), "sol_selftest_wait_timeout")


def sol_attention_chain_fused(q_raw, k_raw, v, gamma_q, gamma_k, grid, block, topk, rope_split=None,
                              rope_theta=10000.0, eps=1e-6, softmax_scale=0.0, stream=None):
    """The whole hot path on device tensors, three launches: the prologue that also
    emits the block means -> scores and top-k from those means -> attention.
    Returns (o, lse, idx, q, k), q and k being the prologue outputs."""
    q, k, qbar, kbar = sol_qk_prologue_pool(q_raw, k_raw, gamma_q, gamma_k, grid, block, rope_split, rope_theta, eps,
                                            stream=stream)
    idx = sol_block_select_pooled(qbar, kbar, grid, block, topk, stream=stream)
    o, lse = sol_sparse_attn_fwd(q, k, v, idx, grid, block, softmax_scale, stream=stream)
    return o, lse, idx, q, k


def sol_attention_chain(q_raw, k_raw, v, gamma_q, gamma_k, grid, block, topk, rope_split=None, rope_theta=10000.0,
                        eps=1e-6, softmax_scale=0.0, workspace=None, stream=None):
    """The whole hot path on device tensors, four launches: prologue -> select
    (pooling q and k itself) -> attention.  Returns (o, lse, idx)."""
    q, k = sol_qk_prologue(q_raw, k_raw, gamma_q, gamma_k, grid, rope_split, rope_theta, eps, stream=stream)
    idx = sol_block_select(q, k, grid, block, topk, workspace=workspace, stream=stream)
    o, lse = sol_sparse_attn_fwd(q, k, v, idx, grid, block, softmax_scale, stream=stream)
    return o, lse, idx
