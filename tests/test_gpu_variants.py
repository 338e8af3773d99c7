"""GPU parity of the selection variants (forced blocks, per-head k, top-p) and of
count-limited attention, against the oracle on the same inputs.

Selection: both sides score the same fp32 block means (pooled by the oracle
from the workload's inputs); the oracle scores in fp64.  Rows must match id for
id, except (as for the plain top-k) where the cut falls inside a near tie of
the scores (1e-4 relative), and - with top-p - where the oracle's cumulative
mass at the disputed prefix lengths lies within 1e-5 of top_p (the kernel sums
fp32 exponentials; the oracle fp64 ones).
Attention: O within 2e-2 and LSE within 1e-2 (bf16), 1e-5 relative (fp32).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.gpu_common import NEAR_TIE_REL, cpu_inputs, np64, sample_units, scale_of
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu

MASS_TOL = 1e-5


def oracle_order(row, i, diagonal, first_blocks):
    forced = set(range(min(first_blocks, row.size)))
    if diagonal:
        forced.add(i)
    return sorted(forced) + [j for j in np.argsort(-row, kind="stable") if j not in forced], len(forced)


def check_variant(idx_g, cnt_g, s64, topk, *, diagonal=False, first_blocks=0, top_p=None, scale=1.0, head_k=None):
    """Returns (rows, rows whose count differs, rows whose ids differ)."""
    idx_o, cnt_o = orc.select_variant(s64, topk, diagonal=diagonal, first_blocks=first_blocks, top_p=top_p,
                                      scale=scale, head_k=head_k)
    assert cnt_g.min() >= 1 and cnt_g.max() <= topk
    n_cnt = n_ids = 0
    B, H, nb, _ = s64.shape
    for b, h, i in zip(*np.nonzero((cnt_g != cnt_o) | np.any(idx_g != idx_o, axis=-1))):
        row = s64[b, h, i]
        cg, co = int(cnt_g[b, h, i]), int(cnt_o[b, h, i])
        order, nf = oracle_order(row, i, diagonal, first_blocks)
        if cg != co:
            assert top_p is not None, (b, h, i, cg, co)
            e = np.exp(scale * (row - row.max()))
            cum = np.cumsum(e[order]) / e.sum()
            for L in range(min(cg, co), max(cg, co)):
                assert abs(cum[L - 1] - top_p) <= MASS_TOL, (b, h, i, cg, co, cum[L - 1])
            n_cnt += 1
        got = idx_g[b, h, i]
        assert np.all(got[cg:] == -1) and np.all(np.diff(got[:cg]) > 0)
        want = np.sort(np.asarray(order[:cg]))
        if not np.array_equal(got[:cg], want):
            # the cut at cg falls inside a near tie of the non-forced scores
            assert nf < cg < nb, (b, h, i)
            a, c = row[order[cg - 1]], row[order[cg]]
            band = NEAR_TIE_REL * max(abs(a), abs(c))
            assert abs(a - c) < band, (b, h, i, a, c)
            assert all(abs(row[j] - a) <= 2 * band for j in set(got[:cg]) ^ set(want)), (b, h, i)
            n_ids += 1
    return cnt_g.size, n_cnt, n_ids


@pytest.fixture(scope="module", params=[0, 1], ids=["f32-64x16", "bf16-128x224"])
def pooled(request):
    """fp32 block means of the workload's raw Q and K (the selection's input)."""
    wl = WORKLOADS[request.param]
    inp = cpu_inputs(request.param)
    block = wl.block
    qbar = orc.block_pool(np64(inp["q"]), block).astype(np.float32)
    kbar = orc.block_pool(np64(inp["k"]), block).astype(np.float32)
    return wl, qbar, kbar


CASES = [
    dict(flags=0),
    dict(flags=1),                              # forced diagonal
    dict(flags=2),                              # forced first frame
    dict(flags=3),
    dict(flags=4, top_p=0.5),                   # softmax scale 1/sqrt(D): nearly flat over blocks
    dict(flags=4, top_p=0.5, scale=2.0),        # sharper: counts spread over 1 .. k
    dict(flags=4, top_p=0.9, scale=2.0),
    dict(flags=4, top_p=1.0, scale=2.0),
    dict(flags=7, top_p=0.7, scale=4.0),
    dict(flags=0, per_head=True),
    dict(flags=5, top_p=0.8, scale=2.0, per_head=True),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_selection_variants_match_oracle(sol, pooled, case):
    wl, qbar, kbar = pooled
    grid, block = wl.grid, wl.block
    B, H, nb, D = qbar.shape
    topk = 8 if nb == 16 else min(wl.topk)
    head_k = None
    if case.get("per_head"):
        head_k = np.array([(h * 7) % (topk + 3) for h in range(H)], dtype=np.int32)   # 0 and > topk clamp
    scale = case.get("scale", scale_of(D))
    s64 = orc.block_scores(qbar.astype(np.float64), kbar.astype(np.float64))
    idx, counts, scores = sol.sol_block_select_pooled_ex(
        torch.from_numpy(qbar).cuda(), torch.from_numpy(kbar).cuda(), grid, block, topk, flags=case["flags"],
        top_p=case.get("top_p", 1.0), softmax_scale=case.get("scale", 0.0), head_k=torch.from_numpy(head_k).cuda() if head_k is not None else None,
        return_scores=True)
    torch.cuda.synchronize()
    first = orc.first_frame_blocks(grid, block)
    rows, n_cnt, n_ids = check_variant(
        idx.cpu().numpy(), counts.cpu().numpy(), s64, topk, diagonal=bool(case["flags"] & 1),
        first_blocks=first if case["flags"] & 2 else 0, top_p=case.get("top_p") if case["flags"] & 4 else None,
        scale=scale, head_k=head_k)
    assert n_cnt <= max(2, rows // 1000) and n_ids <= max(2, rows // 1000), (rows, n_cnt, n_ids)
    if case["flags"] == 0 and head_k is None:
        plain = sol.sol_block_select_pooled(torch.from_numpy(qbar).cuda(), torch.from_numpy(kbar).cuda(), grid,
                                            block, topk)
        torch.cuda.synchronize()
        assert torch.equal(plain, idx) and bool((counts == topk).all())


def _attention_inputs(wl_id, H=None):
    """The workload's raw q, k, v (first H heads) on the GPU, in its dtype."""
    wl = WORKLOADS[wl_id]
    inp = cpu_inputs(wl_id)
    return (wl, *(inp[n][:, :, :H].contiguous().cuda() for n in ("q", "k", "v")))


@pytest.mark.parametrize("wl_id", [0, 1])
def test_attention_counts_match_oracle(sol, wl_id):
    wl, qd, kd, vd = _attention_inputs(wl_id, H=None if wl_id == 0 else 4)
    B, N, H, D = qd.shape
    block, nb = wl.block, -(-N // wl.block)
    topk = min(6, nb)
    rng = np.random.default_rng([wl_id, 99])
    # rows of distinct valid ids (entries beyond a row's count stay valid ids, so
    # a kernel that read them would give wrong results rather than bad addresses)
    idx = np.stack([rng.permutation(nb)[:topk] for _ in range(B * H * nb)]).reshape(B, H, nb, topk).astype(np.int32)
    counts = rng.integers(-1, topk + 2, size=(B, H, nb)).astype(np.int32)   # clamped to [1, topk]
    counts[..., 0] = 1
    counts[..., -1] = topk
    dev = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    o, lse = sol.sol_sparse_attn_fwd_counts(qd, kd, vd, dev(idx), dev(counts), wl.grid, block)
    torch.cuda.synchronize()
    eff = np.clip(counts, 1, topk)
    units = sample_units(B, H, nb, per_head=min(nb, 16))
    q64, k64, v64 = (np64(t) for t in (qd, kd, vd))
    o_ref, lse_ref = orc.sparse_attention(q64, k64, v64, idx, block, units=units, counts=eff)
    rows = [(b, h, np.arange(i * block, min(N, (i + 1) * block))) for (b, h, i) in units]
    err_o = max(np.abs(np64(o[b, r, h]) - o_ref[b, r, h]).max() for (b, h, r) in rows)
    err_l = max(np.abs(np64(lse[b, h, r]) - lse_ref[b, h, r]).max() for (b, h, r) in rows)
    if wl.dtype == "bf16":
        assert err_o <= 2e-2 and err_l <= 1e-2, (err_o, err_l)
    else:
        o_s = max(np.abs(o_ref[b, r, h]).max() for (b, h, r) in rows)
        l_s = max(np.abs(lse_ref[b, h, r]).max() for (b, h, r) in rows)
        assert err_o <= 1e-5 * o_s and err_l <= 1e-5 * l_s, (err_o, err_l)
    # all counts equal to topk: the plain call's result, bit for bit
    full = np.full((B, H, nb), topk, dtype=np.int32)
    o2, l2 = sol.sol_sparse_attn_fwd_counts(qd, kd, vd, dev(idx), dev(full), wl.grid, block)
    o3, l3 = sol.sol_sparse_attn_fwd(qd, kd, vd, dev(idx), wl.grid, block)
    torch.cuda.synchronize()
    assert torch.equal(o2, o3) and torch.equal(l2, l3)


def test_top_p_chain_matches_oracle(sol):
    """select_ex (forced diagonal + top-p) feeding count-limited attention."""
    wl, qd, kd, vd = _attention_inputs(1, H=4)
    B, N, H, D = qd.shape
    block, nb, topk = wl.block, -(-N // wl.block), 45
    dev = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    q64, k64, v64 = (np64(t) for t in (qd, kd, vd))
    qbar = orc.block_pool(q64, block).astype(np.float32)
    kbar = orc.block_pool(k64, block).astype(np.float32)
    idx, counts = sol.sol_block_select_pooled_ex(dev(qbar), dev(kbar), wl.grid, block, topk, flags=5, top_p=0.6,
                                                 softmax_scale=2.0)
    o, lse = sol.sol_sparse_attn_fwd_counts(qd, kd, vd, idx, counts, wl.grid, block)
    torch.cuda.synchronize()
    s64 = orc.block_scores(qbar.astype(np.float64), kbar.astype(np.float64))
    idx_n, cnt_n = idx.cpu().numpy(), counts.cpu().numpy()
    check_variant(idx_n, cnt_n, s64, topk, diagonal=True, top_p=0.6, scale=2.0)
    assert cnt_n.min() >= 1 and cnt_n.max() <= topk and len(np.unique(cnt_n)) > 1
    units = sample_units(B, H, nb, per_head=12)
    o_ref, lse_ref = orc.sparse_attention(q64, k64, v64, idx_n, block, units=units, counts=cnt_n)
    for (b, h, i) in units:
        r = np.arange(i * block, min(N, (i + 1) * block))
        assert np.abs(np64(o[b, r, h]) - o_ref[b, r, h]).max() <= 2e-2
        assert np.abs(np64(lse[b, h, r]) - lse_ref[b, h, r]).max() <= 1e-2
