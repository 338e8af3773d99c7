"""GPU parity of 3-D tile blocks (t x h x w tokens per block) against the oracle.

  * sol_qk_prologue_pool_tiled: Q / K identical to sol_qk_prologue; block means
    within the fp32 running-sum bound of the oracle's tile means of the stored
    outputs (the same bound as the run-based fused test).
  * sol_sparse_attn_fwd_tiled: O / LSE against the oracle's tiled attention
    (bf16 within 2e-2 / 1e-2; fp32 within 1e-5 relative), and bit for bit
    equal to the run-based kernel on the tokens permuted into tile order (the
    kernel stages the same rows in the same order, so nothing may differ).
  * the tiled chain: tiled means -> selection with forced first-frame tiles ->
    tiled count-limited attention.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.gpu_common import check_selection, cpu_inputs, np64, sample_units
from tests.test_gpu_variants import check_variant
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


def tile_permutation(grid, tile):
    T, Hg, Wg = grid
    t, h, w = tile
    ids = np.arange(T * Hg * Wg).reshape(T // t, t, Hg // h, h, Wg // w, w)
    return torch.from_numpy(ids.transpose(0, 2, 4, 1, 3, 5).reshape(-1).copy())


def tiled_mean_tolerance(x64, blocks, size):
    m = orc.block_pool(x64, blocks)
    mean_abs = orc.block_pool(np.abs(x64), blocks)
    k = size - 1
    gamma = k * U32 / (1 - k * U32)
    return m, gamma * mean_abs * (1 + 3 * U32) + 3 * U32 * np.abs(m)


CASES = [(0, (1, 8, 8)), (0, (2, 4, 8)), (1, (2, 8, 8)), (1, (4, 4, 8))]


@pytest.mark.parametrize("wl_id,tile", CASES, ids=[f"w{w}-{t}" for w, t in CASES])
def test_tiled_prologue_pool(sol, wl_id, tile):
    wl = WORKLOADS[wl_id]
    inp = cpu_inputs(wl_id)
    H = min(wl.H, 4)
    q_raw, k_raw = (inp[n][:, :, :H].contiguous().cuda() for n in ("q", "k"))
    gq, gk = (inp[n][:H * wl.D].contiguous().cuda() for n in ("gamma_q", "gamma_k"))
    q_ref, k_ref = sol.sol_qk_prologue(q_raw, k_raw, gq, gk, wl.grid, wl.rope_split, wl.rope_theta, wl.eps)
    q, k, qbar, kbar = sol.sol_qk_prologue_pool_tiled(q_raw, k_raw, gq, gk, wl.grid, tile, wl.rope_split,
                                                      wl.rope_theta, wl.eps)
    torch.cuda.synchronize()
    assert torch.equal(q, q_ref) and torch.equal(k, k_ref)
    blocks = orc.tiled_blocks(wl.grid, tile)
    size = tile[0] * tile[1] * tile[2]
    assert qbar.shape == (wl.B, H, len(blocks), wl.D)
    for out, bar in ((q, qbar), (k, kbar)):
        m, tol = tiled_mean_tolerance(np64(out), blocks, size)
        err = np.abs(np64(bar) - m)
        assert (err <= tol).all(), float((err - tol).max())
    # the selection over tile means follows the oracle's rule on the stored outputs
    topk = min(wl.topk) if wl_id else 4
    idx = sol.sol_block_select_pooled(qbar, kbar, wl.grid, size, topk)
    torch.cuda.synchronize()
    s_ref = orc.block_scores(orc.block_pool(np64(q), blocks), orc.block_pool(np64(k), blocks))
    check_selection(idx.cpu().numpy(), s_ref, topk)


@pytest.mark.parametrize("wl_id,tile", CASES, ids=[f"w{w}-{t}" for w, t in CASES])
def test_tiled_attention(sol, wl_id, tile):
    wl = WORKLOADS[wl_id]
    inp = cpu_inputs(wl_id)
    H = min(wl.H, 4)
    q, k, v = (inp[n][:, :, :H].contiguous().cuda() for n in ("q", "k", "v"))
    B, N, _, D = q.shape
    size = tile[0] * tile[1] * tile[2]
    nb = N // size
    topk = min(8, nb)
    rng = np.random.default_rng([wl_id, size, 5])
    idx = np.stack([rng.permutation(nb)[:topk] for _ in range(B * H * nb)]).reshape(B, H, nb, topk).astype(np.int32)
    counts = rng.integers(1, topk + 1, size=(B, H, nb)).astype(np.int32)
    idx_d, counts_d = torch.from_numpy(idx).cuda(), torch.from_numpy(counts).cuda()
    o, lse = sol.sol_sparse_attn_fwd_tiled(q, k, v, idx_d, wl.grid, tile)
    oc, lsec = sol.sol_sparse_attn_fwd_tiled(q, k, v, idx_d, wl.grid, tile, counts=counts_d)
    # the same attention on tokens permuted into tile order, with runs of `size` tokens
    perm = tile_permutation(wl.grid, tile).cuda()
    qp, kp, vp = (x[:, perm].contiguous() for x in (q, k, v))
    o_p, lse_p = sol.sol_sparse_attn_fwd(qp, kp, vp, idx_d, wl.grid, size)
    torch.cuda.synchronize()
    assert torch.equal(o[:, perm], o_p) and torch.equal(lse[:, :, perm], lse_p)
    blocks = orc.tiled_blocks(wl.grid, tile)
    units = sample_units(B, H, nb, per_head=min(nb, 12))
    q64, k64, v64 = (np64(x) for x in (q, k, v))
    for out_o, out_l, cnt in ((o, lse, None), (oc, lsec, counts)):
        o_ref, lse_ref = orc.sparse_attention(q64, k64, v64, idx, blocks, units=units, counts=cnt)
        rows = [(b, h, blocks[i]) for (b, h, i) in units]
        err_o = max(np.abs(np64(out_o[b, r, h]) - o_ref[b, r, h]).max() for (b, h, r) in rows)
        err_l = max(np.abs(np64(out_l[b, h, r]) - lse_ref[b, h, r]).max() for (b, h, r) in rows)
        if wl.dtype == "bf16":
            assert err_o <= 2e-2 and err_l <= 1e-2, (err_o, err_l)
        else:
            o_s = max(np.abs(o_ref[b, r, h]).max() for (b, h, r) in rows)
            l_s = max(np.abs(lse_ref[b, h, r]).max() for (b, h, r) in rows)
            assert err_o <= 1e-5 * o_s and err_l <= 1e-5 * l_s, (err_o, err_l)


def test_tiled_chain_with_forced_first_frame(sol):
    wl, tile = WORKLOADS[1], (2, 8, 8)
    inp = cpu_inputs(1)
    H = 4
    q_raw, k_raw, v = (inp[n][:, :, :H].contiguous().cuda() for n in ("q", "k", "v"))
    gq, gk = (inp[n][:H * wl.D].contiguous().cuda() for n in ("gamma_q", "gamma_k"))
    q, k, qbar, kbar = sol.sol_qk_prologue_pool_tiled(q_raw, k_raw, gq, gk, wl.grid, tile, wl.rope_split,
                                                      wl.rope_theta, wl.eps)
    topk = 45
    idx, counts = sol.sol_block_select_pooled_ex(qbar, kbar, wl.grid, 128, topk, flags=2 | 4, top_p=0.8,
                                                 softmax_scale=2.0, tile=tile)
    o, lse = sol.sol_sparse_attn_fwd_tiled(q, k, v, idx, wl.grid, tile, counts=counts)
    torch.cuda.synchronize()
    n_first = orc.first_frame_blocks(wl.grid, 128, tile=tile)
    assert n_first == 28
    s64 = orc.block_scores(np64(qbar), np64(kbar))
    idx_n, cnt_n = idx.cpu().numpy(), counts.cpu().numpy()
    check_variant(idx_n, cnt_n, s64, topk, first_blocks=n_first, top_p=0.8, scale=2.0)
    assert (idx_n[..., :n_first] == np.arange(n_first)).all()     # the first-frame tiles lead every row
    blocks = orc.tiled_blocks(wl.grid, tile)
    units = sample_units(1, H, len(blocks), per_head=8)
    q64, k64, v64 = (np64(x) for x in (q, k, v))
    o_ref, lse_ref = orc.sparse_attention(q64, k64, v64, idx_n, blocks, units=units, counts=cnt_n)
    for (b, h, i) in units:
        r = blocks[i]
        assert np.abs(np64(o[b, r, h]) - o_ref[b, r, h]).max() <= 2e-2
        assert np.abs(np64(lse[b, h, r]) - lse_ref[b, h, r]).max() <= 1e-2
