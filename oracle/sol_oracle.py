"""Plain fp64 CPU oracle of the Sol-Attn hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or links
this module; only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference arm use it.  It shares no code with the CUDA path.

Source of the method.  The Sol-H3 pages describe Sol-Attn as a training-free
sparse attention that decides, per query, which parts of the attention
computation matter, and credit it with the largest share of the runtime's
speed-up (ai-feiten.nl, "Videomodel MiniMax-H3 rendert sneller dan afspelen",
section "Waar de snelheidswinst vandaan komt"); the same section says
normalisation and RoPE were merged into single kernels and that the
preparation of the sparse attention became 76.4% faster.  The two-stage
pipeline uses Sol-Attn in its high-resolution refinement stage
(ainews.surl.tw, "NVIDIA Adds Two-Stage Generation for MiniMax H3").  The
pages give no formula, so this file writes out the concrete definition the
implementation follows, one plain loop nest or library primitive per step:

  a1  QK prologue: RMSNorm over the head dim, times a per-(head, channel)
      gain, then 3D rotary embedding on adjacent channel pairs, t/h/w axes in
      channel order.                                         (qk_prologue)
  a2  mean-pool Q and K over contiguous token blocks.         (block_pool)
  a3  score every (query block, key block) pair by the dot product of the
      pooled means.                                          (block_scores)
  a4  keep the k best key blocks per query block; exact ties go to the lower
      block id; the kept ids are listed in ascending order.  (topk_blocks)
  a5  exact softmax attention of every query over the keys of its kept
      blocks; returns O and the natural-log LSE of the scaled logits.
                                                             (sparse_attention)

Readings taken where the pages are silent are listed at each function.
Everything is float64; stored low-precision inputs are widened exactly.
Parity pins: see tests/test_oracle_pins.py (closed forms, brute force,
invariants and a library dense-attention routine).
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "bf16_round", "rope_angles", "qk_prologue", "block_pool", "block_scores",
    "topk_blocks", "near_tie_rows", "block_select", "sparse_attention",
    "sparse_attention_rows", "selected_flops", "first_frame_blocks", "select_variant", "tiled_blocks",
    "sparse_attention_backward",
]


def bf16_round(x) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (ties to even).

    bfloat16 keeps 8 significant bits (7 stored + the implicit one) and the
    float32 exponent range.  Returned as float64 (every bf16 value is exact).
    Subnormal bf16 results are handled by clamping the exponent at -126.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                 # below 2**-126 the spacing stays 2**-133
    scaled = np.ldexp(x, 8 - e)             # 8 significant bits left of the point
    r = np.ldexp(np.rint(scaled), e - 8)    # np.rint rounds half to even
    return np.where(np.isfinite(x), r, x)


def rope_angles(grid, split, theta: float) -> np.ndarray:
    """Rotation angle of every (token, channel pair), float64 [N, D/2].

    Reading: channels are taken in adjacent pairs (2p, 2p+1); the first
    split[0]/2 pairs rotate with the frame index t, the next split[1]/2 with the
    row y, the last split[2]/2 with the column x.  Pair i inside an axis of
    d_axis channels turns by pos * theta**(-2i/d_axis).  Positions are the
    integer grid coordinates of token n = (t*Hg + y)*Wg + x, starting at 0.
    """
    T, Hg, Wg = grid
    n = np.arange(T * Hg * Wg)
    pos = (n // (Hg * Wg), (n // Wg) % Hg, n % Wg)
    cols = []
    for axis in range(3):
        d_axis = split[axis]
        for i in range(d_axis // 2):
            freq = theta ** (-2.0 * i / d_axis)
            cols.append(pos[axis].astype(np.float64) * freq)
    return np.stack(cols, axis=1)


def qk_prologue(x, gamma, grid, split, theta: float, eps: float, tokens=None) -> np.ndarray:
    """Fused QK-RMSNorm + 3D RoPE of one tensor (Q or K), float64 result.

    x: [B, N, H, D] (any float dtype, widened exactly); gamma: [H*D].
    tokens: optional token indices; then only those rows are computed and the
    result is [B, len(tokens), H, D].
    y = x / sqrt(mean_d x^2 + eps) * gamma[h, d]; then each pair (y0, y1) of a
    token turns by its angle phi: (y0 cos phi - y1 sin phi, y0 sin phi + y1 cos phi).
    Reading: the norm runs over the head dimension of one (token, head); RMSNorm
    comes before RoPE; V is not touched.  The caller rounds to the stored dtype.
    """
    B, N, H, D = x.shape
    x = np.asarray(x if tokens is None else x[:, tokens], dtype=np.float64)
    g = np.asarray(gamma, dtype=np.float64).reshape(H, D)
    rms = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    y = x / rms * g[None, None, :, :]
    phi = rope_angles(grid, split, theta)                   # [N, D/2]
    if tokens is not None:
        phi = phi[tokens]
    c = np.cos(phi)[None, :, None, :]
    s = np.sin(phi)[None, :, None, :]
    y0 = y[..., 0::2]
    y1 = y[..., 1::2]
    out = np.empty_like(y)
    out[..., 0::2] = y0 * c - y1 * s
    out[..., 1::2] = y0 * s + y1 * c
    return out


def tiled_blocks(grid, tile) -> list:
    """Token ids of every 3-D tile block, a list of int arrays.

    The grid (T, Hg, Wg) is cut into tiles of tile = (t, h, w) tokens (exactly:
    each extent divides the grid's); tiles are numbered in raster order of
    their position (tile frame, tile row, tile column) and the tokens of a tile
    are listed in raster order (frame, row, column).  Token ids are raster
    order of the grid, n = (t * Hg + y) * Wg + x.
    """
    T, Hg, Wg = (int(g) for g in grid)
    tt, th, tw = (int(x) for x in tile)
    assert T % tt == 0 and Hg % th == 0 and Wg % tw == 0
    blocks = []
    for it in range(T // tt):
        for iy in range(Hg // th):
            for ix in range(Wg // tw):
                ids = [((it * tt + dt) * Hg + iy * th + dy) * Wg + ix * tw + dx
                       for dt in range(tt) for dy in range(th) for dx in range(tw)]
                blocks.append(np.asarray(ids, dtype=np.int64))
    return blocks


def _members(N: int, block) -> list:
    """Token ids of every block: `block` is a block size (runs of consecutive
    tokens, the last one possibly short) or a list of id arrays (tiled_blocks)."""
    if isinstance(block, (int, np.integer)):
        return [np.arange(i * block, min(N, (i + 1) * block)) for i in range(-(-N // block))]
    return list(block)


def block_pool(x, block) -> np.ndarray:
    """Mean of x over each block's tokens, float64 [B, H, nb, D].

    Reading: by default blocks are runs of `block` consecutive raster-order
    tokens; the last block may be short (N % block tokens) and is averaged over
    its valid tokens only.  `block` may instead list each block's token ids
    (3-D tiles: tiled_blocks).
    """
    B, N, H, D = x.shape
    members = _members(N, block)
    out = np.empty((B, H, len(members), D))
    for i, ids in enumerate(members):
        seg = np.asarray(x[:, ids], dtype=np.float64)   # [B, n_i, H, D]
        out[:, :, i, :] = seg.mean(axis=1)
    return out


def block_scores(qbar, kbar) -> np.ndarray:
    """s[b, h, i, j] = sum_d qbar[b, h, i, d] * kbar[b, h, j, d]  (float64)."""
    return np.matmul(np.asarray(qbar, np.float64), np.swapaxes(np.asarray(kbar, np.float64), -1, -2))


def topk_blocks(scores, k: int) -> np.ndarray:
    """Ids of the k largest scores per row, listed ascending; int32 [..., k].

    Order: by score descending, exact ties broken by the lower block id (a
    stable sort of -score keeps the original ascending id order among ties).
    Reading: "keeps its top-k key blocks" is taken literally, with no forced
    diagonal or sink block.
    """
    s = np.asarray(scores, np.float64)
    order = np.argsort(-s, axis=-1, kind="stable")[..., :k]
    return np.sort(order, axis=-1).astype(np.int32)


def near_tie_rows(scores, k: int, rel: float = 1e-4) -> np.ndarray:
    """Boolean [...] mask of rows whose k-th and (k+1)-th largest scores differ
    by less than rel * max(|s_k|, |s_k+1|).  Rows with k == number of blocks
    have no (k+1)-th score and are never near-tie rows."""
    s = -np.sort(-np.asarray(scores, np.float64), axis=-1)
    if k >= s.shape[-1]:
        return np.zeros(s.shape[:-1], dtype=bool)
    a, b = s[..., k - 1], s[..., k]
    return np.abs(a - b) < rel * np.maximum(np.abs(a), np.abs(b))


def block_select(q, k, block: int, topk: int):
    """Steps a2-a4: returns (idx int32 [B, H, nb, topk], scores float64 [B, H, nb, nb])."""
    s = block_scores(block_pool(q, block), block_pool(k, block))
    return topk_blocks(s, topk), s


def first_frame_blocks(grid, block: int, tile=None) -> int:
    """Number of blocks holding a token of frame t = 0 (they are blocks 0 .. count - 1).
    Runs: tokens 0 .. grid_h * grid_w - 1 come first in raster order, so
    ceil(grid_h * grid_w / block).  Tiles (t, h, w): the tiles of the first
    tile frame, (grid_h / h) * (grid_w / w)."""
    if tile is not None:
        return (int(grid[1]) // int(tile[1])) * (int(grid[2]) // int(tile[2]))
    return -(-(int(grid[1]) * int(grid[2])) // block)


def select_variant(scores, topk: int, *, diagonal: bool = False, first_blocks: int = 0, top_p=None,
                   scale: float = 1.0, head_k=None):
    """Selection variants over a score matrix [B, H, nb, nb]: forced blocks, top-p, per-head k.

    Sol-Attn decides per query which parts of the attention matter (ai-feiten.nl,
    "Videomodel MiniMax-H3 rendert sneller dan afspelen", section "Waar de
    snelheidswinst vandaan komt"); the pages fix no rule, so these are readings:
      - forced blocks: the query's own block i (diagonal) and blocks 0 ..
        first_blocks - 1 (the first latent frame) come first in the row's order,
        in ascending id; the other blocks follow by descending score, exact ties
        to the lower id;
      - k_h = topk, or head_k[h] clamped to [1, topk];
      - without top_p the row keeps the first k_h ids of its order; with top_p it
        keeps the first c = min(k_h, max(#forced, 1, c_p)), where c_p is the
        shortest prefix whose softmax mass, softmax_j(scale * s_ij) over all
        key blocks, reaches top_p.
    Returns (idx int32 [B, H, nb, topk]: the kept ids ascending, then -1;
    counts int32 [B, H, nb]).
    """
    s = np.asarray(scores, np.float64)
    B, H, nb, _ = s.shape
    idx = np.full((B, H, nb, topk), -1, dtype=np.int32)
    counts = np.zeros((B, H, nb), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            kh = topk if head_k is None else min(max(int(head_k[h]), 1), topk)
            for i in range(nb):
                row = s[b, h, i]
                forced = set(range(min(first_blocks, nb)))
                if diagonal:
                    forced.add(i)
                rest = [j for j in np.argsort(-row, kind="stable") if j not in forced]
                order = sorted(forced) + rest
                if top_p is None:
                    c = kh
                else:
                    e = np.exp(scale * (row - row.max()))
                    cum = np.cumsum(e[order])
                    c_p = int(np.argmax(cum >= top_p * cum[-1])) + 1   # cum[-1]: the row's total mass
                    c = min(kh, max(len(forced), 1, c_p))
                idx[b, h, i, :c] = np.sort(np.asarray(order[:c]))
                counts[b, h, i] = c
    return idx, counts


def sparse_attention_rows(q, k, v, idx, block, scale: float, b: int, h: int, i: int, count=None):
    """Attention of the queries of block i of (b, h) over its kept key blocks.

    Keys: every token m < N of the blocks idx[b, h, i, :count] (all of the row
    when count is None).  Logits
    l_m = scale * q_n . k_m; two-pass softmax: subtract the row max, exponentiate,
    normalise.  Returns (o [n_i, D], lse [n_i]) with lse = ln sum_m exp(l_m).
    """
    members = _members(q.shape[1], block)
    rows = members[i]
    kept = np.asarray(idx[b, h, i])[:count]
    cols = np.concatenate([members[j] for j in kept])
    qi = np.asarray(q[b, rows, h, :], np.float64)
    kj = np.asarray(k[b, cols, h, :], np.float64)
    vj = np.asarray(v[b, cols, h, :], np.float64)
    logits = scale * (qi @ kj.T)
    mx = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - mx)
    denom = p.sum(axis=1, keepdims=True)
    o = (p @ vj) / denom
    lse = mx[:, 0] + np.log(denom[:, 0])
    return o, lse


def sparse_attention(q, k, v, idx, block, scale: float | None = None, units=None, counts=None):
    """Step a5 over all (b, h, query block) units, or over the listed `units`.

    q, k, v: [B, N, H, D] stored tensors (widened exactly to float64).
    idx: [B, H, nb, k] kept key-block ids; with counts [B, H, nb], row (b, h, i)
    keeps only its first counts[b, h, i] ids.  scale defaults to 1/sqrt(D).
    block: block size (runs of consecutive tokens) or each block's token ids
    (3-D tiles: tiled_blocks).
    Returns (o [B, N, H, D], lse [B, H, N]) float64; rows of units not computed
    are NaN.
    """
    q = np.asarray(q)
    k = np.asarray(k)
    v = np.asarray(v)
    B, N, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    members = _members(N, block)
    o = np.full((B, N, H, D), np.nan)
    lse = np.full((B, H, N), np.nan)
    if units is None:
        units = [(b, h, i) for b in range(B) for h in range(H) for i in range(len(members))]
    for (b, h, i) in units:
        c = None if counts is None else int(counts[b, h, i])
        oi, li = sparse_attention_rows(q, k, v, idx, members, scale, b, h, i, c)
        o[b, members[i], h, :] = oi
        lse[b, h, members[i]] = li
    return o, lse


def sparse_attention_backward(q, k, v, idx, do, block, scale: float | None = None, counts=None):
    """Gradients of step a5 with respect to q, k and v, given the output gradient do.

    For the queries of block i of (b, h) and the keys m of its kept blocks,
    with P = softmax(scale * q k^T) over those keys and O = P v:
        dv_m += sum_n P_nm do_n
        dP_nm = do_n . v_m
        dS_nm = P_nm (dP_nm - sum_m' P_nm' dP_nm')      (softmax Jacobian; the
                 inner sum equals do_n . O_n)
        dq_n += scale * sum_m dS_nm k_m
        dk_m += scale * sum_n dS_nm q_n
    Keys kept by several query blocks accumulate contributions from all of them.
    The method is used for inference only; this is the definition a backward
    kernel would follow.  Returns (dq, dk, dv) float64 [B, N, H, D].
    """
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    B, N, H, D = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    members = _members(N, block)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            for i, rows in enumerate(members):
                kept = np.asarray(idx[b, h, i])[: None if counts is None else int(counts[b, h, i])]
                cols = np.concatenate([members[j] for j in kept])
                s_ = scale * (q[b, rows, h] @ k[b, cols, h].T)
                p_ = np.exp(s_ - s_.max(axis=1, keepdims=True))
                p_ /= p_.sum(axis=1, keepdims=True)
                o_ = p_ @ v[b, cols, h]
                dp = do[b, rows, h] @ v[b, cols, h].T
                ds = p_ * (dp - np.sum(do[b, rows, h] * o_, axis=1, keepdims=True))
                dq[b, rows, h] += scale * ds @ k[b, cols, h]
                np.add.at(dk[:, :, h], (b, cols), scale * ds.T @ q[b, rows, h])
                np.add.at(dv[:, :, h], (b, cols), p_.T @ do[b, rows, h])
    return dq, dk, dv


def selected_flops(idx, N: int, block: int, D: int) -> int:
    """4 * n_q * n_k * D summed over the selected (query block, key block) pairs,
    with n_q, n_k the valid token counts of each block."""
    idx = np.asarray(idx)
    nb = -(-N // block)
    sizes = np.minimum(block, N - np.arange(nb) * block)
    nk = sizes[idx].sum(axis=-1)                 # [B, H, nb] keys seen per query block
    return int(4 * D * (nk * sizes[None, None, :]).sum())
