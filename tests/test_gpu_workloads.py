"""GPU parity on the five video-token workloads, at full size.

Workload 0 (fp32, 4x16x16 grid) is checked everywhere against the full oracle,
including k = 16 = nb, which must equal dense attention.  Workloads 1-4 (bf16,
28,672 to 130,560 tokens):

  * staged: the selection on the stored prologue outputs, every row (near-tie
    rule), then attention given the oracle's selection - on every query block
    of every head for workload 1, on sampled blocks (all heads x 16 blocks:
    first, last - the ragged one for workload 3 - and 14 random) for 2-4;
  * chain: raw activations through the whole path, in both launch sequences -
    "fused" (sol_qk_prologue_pool -> sol_block_select_pooled ->
    sol_sparse_attn_fwd, the step the benchmark times) and "split"
    (sol_qk_prologue -> sol_block_select -> sol_sparse_attn_fwd) - against the
    oracle's own chain: prologue on sampled tokens (including every token of
    the last block), the fused path's block means on sampled blocks (including
    the last), the selection on every row, attention on sampled blocks.

Each test writes its counts (rows, near-tie rows, differing rows) and errors to
tests/parity_record.json.
"""
import functools

import numpy as np
import pytest
import torch

import oracle as orc
from tests.gpu_common import (check_attention, check_bf16_prologue, check_selection, cpu_inputs, np32, np64,
                              prologue_flip_size, record_parity, REL_TOL_F32, sample_units,
                              score_perturbation_bound)
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def oracle_prologue_bf16(x32: np.ndarray, gamma, wl, chunk=4096):
    """Oracle prologue over all tokens, rounded to bf16 (stored as float32), and
    the block means of the possible one-step rounding flips of the kernel's
    fp32 result, [B, H, nb, D]."""
    out = np.empty_like(x32)
    flips = np.zeros((wl.B, wl.H, wl.nb, wl.D))
    assert chunk % wl.block == 0
    for t0 in range(0, wl.N, chunk):
        tok = np.arange(t0, min(wl.N, t0 + chunk))
        y = orc.qk_prologue(x32, gamma, wl.grid, wl.rope_split, wl.rope_theta, wl.eps, tokens=tok)
        out[:, t0:t0 + len(tok)] = orc.bf16_round(y)
        b0 = t0 // wl.block
        pooled = orc.block_pool(prologue_flip_size(y), wl.block)
        flips[:, :, b0:b0 + pooled.shape[2]] = pooled
    return out, flips


def test_workload0_fp32_full(sol):
    wl = WORKLOADS[0]
    inp = cpu_inputs(0)
    q_raw, k_raw, v = (inp[n] for n in ("q", "k", "v"))
    gq, gk = inp["gamma_q"], inp["gamma_k"]
    qd, kd, vd = q_raw.cuda(), k_raw.cuda(), v.cuda()
    # prologue, fp32
    q, k = sol.sol_qk_prologue(qd, kd, gq.cuda(), gk.cuda(), wl.grid, wl.rope_split, wl.rope_theta, wl.eps)
    torch.cuda.synchronize()
    for raw, g, out in ((q_raw, gq, q), (k_raw, gk, k)):
        ref = orc.qk_prologue(np64(raw), g.double().numpy(), wl.grid, wl.rope_split, wl.rope_theta, wl.eps)
        assert np.abs(np64(out) - ref).max() <= REL_TOL_F32 * np.abs(ref).max()
    # select + attention on the raw activations, k = 4 and k = 16 (= nb: dense)
    qn, kn, vn = np64(q_raw), np64(k_raw), np64(v)
    units = [(0, h, i) for h in range(wl.H) for i in range(wl.nb)]
    for topk in wl.topk:
        idx, scores = sol.sol_block_select(qd, kd, wl.grid, wl.block, topk, return_scores=True)
        torch.cuda.synchronize()
        idx_ref, s_ref = orc.block_select(qn, kn, wl.block, topk)
        check_selection(idx.cpu().numpy(), s_ref, topk)
        o, lse = sol.sol_sparse_attn_fwd(qd, kd, vd, torch.from_numpy(idx_ref).cuda(), wl.grid, wl.block)
        torch.cuda.synchronize()
        check_attention(o, lse, qn, kn, vn, idx_ref, wl.block, units, fp32=True)
        if topk == wl.nb:
            tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (qn, kn, vn))
            dense = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
            assert np.abs(np64(o) - dense).max() <= REL_TOL_F32 * np.abs(dense).max()


@pytest.mark.parametrize("cfg", [1, 2, 3, 4])
def test_workload_select_and_attention(sol, cfg):
    wl = WORKLOADS[cfg]
    topk = wl.topk[0]
    inp = cpu_inputs(cfg)
    q, k, v = (inp[n] for n in ("q", "k", "v"))
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    q32, k32 = np32(q), np32(k)
    idx, scores = sol.sol_block_select(qd, kd, wl.grid, wl.block, topk, return_scores=True)
    torch.cuda.synchronize()
    idx_ref, s_ref = orc.block_select(q32, k32, wl.block, topk)
    np.testing.assert_allclose(np64(scores), s_ref, rtol=1e-4, atol=1e-5 * np.abs(s_ref).max())
    rows, near, differ = check_selection(idx.cpu().numpy(), s_ref, topk)
    o, lse = sol.sol_sparse_attn_fwd(qd, kd, vd, torch.from_numpy(idx_ref).cuda(), wl.grid, wl.block)
    torch.cuda.synchronize()
    if cfg == 1:    # every query block of every head
        units = [(b, h, i) for b in range(wl.B) for h in range(wl.H) for i in range(wl.nb)]
    else:
        units = sample_units(wl.B, wl.H, wl.nb)
    err_o, err_l = check_attention(o, lse, q32, k32, np32(v), idx_ref, wl.block, units, fp32=False)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    record_parity(f"workload{cfg}/staged", path="sol_block_select on the stored q, k; sol_sparse_attn_fwd given "
                  "the oracle's selection", rows=rows, near_tie_rows=near, differing_rows=differ,
                  attention_units=len(units), attention_units_total=wl.B * wl.H * wl.nb, max_abs_dO=err_o,
                  max_abs_dLSE=err_l, tol_dO=2e-2, tol_dLSE=1e-2)


@functools.lru_cache(maxsize=1)
def oracle_chain(cfg):
    """The oracle's own chain on raw workload inputs: prologue outputs rounded
    to bf16, scores of their block means, and the per-row band within which
    the kernel's prologue (allowed to round a value the other way where the
    exact result sits next to a bf16 midpoint) can move the scores."""
    wl = WORKLOADS[cfg]
    inp = cpu_inputs(cfg)
    q_ref, uq = oracle_prologue_bf16(np32(inp["q"]), inp["gamma_q"].double().numpy(), wl)
    k_ref, uk = oracle_prologue_bf16(np32(inp["k"]), inp["gamma_k"].double().numpy(), wl)
    qbar, kbar = orc.block_pool(q_ref, wl.block), orc.block_pool(k_ref, wl.block)
    s_ref = orc.block_scores(qbar, kbar)
    band = 2 * score_perturbation_bound(qbar, kbar, uq, uk).max(axis=-1)
    return q_ref, k_ref, s_ref, band


def pooled_tolerance(x64: np.ndarray, members) -> tuple[np.ndarray, np.ndarray]:
    """Oracle means of x over the listed blocks and the error bound of an fp32
    running sum of <= 128 values followed by one product with the rounded
    reciprocal of the count: gamma_127 mean|x| (1 + 3u) + 3u |m|, u = 2^-24."""
    u = 2.0 ** -24
    m = orc.block_pool(x64, members)
    mean_abs = orc.block_pool(np.abs(x64), members)
    g = 127 * u / (1 - 127 * u)
    return m, g * mean_abs * (1 + 3 * u) + 3 * u * np.abs(m)


CHAIN_CASES = [(c, ch) for c in (1, 2, 3, 4) for ch in ("fused", "split")]


@pytest.mark.parametrize("cfg,chain", CHAIN_CASES, ids=[f"{c}-{ch}" for c, ch in CHAIN_CASES])
def test_workload_chain(sol, cfg, chain):
    wl = WORKLOADS[cfg]
    topk = wl.topk[0]
    inp = cpu_inputs(cfg)
    q_raw, k_raw, v = (inp[n] for n in ("q", "k", "v"))
    gq, gk = inp["gamma_q"], inp["gamma_k"]
    args = (q_raw.cuda(), k_raw.cuda(), v.cuda(), gq.cuda(), gk.cuda())
    if chain == "fused":
        qd, kd, qbar, kbar = sol.sol_qk_prologue_pool(args[0], args[1], args[3], args[4], wl.grid, wl.block,
                                                      wl.rope_split, wl.rope_theta, wl.eps)
        idx = sol.sol_block_select_pooled(qbar, kbar, wl.grid, wl.block, topk)
        o, lse = sol.sol_sparse_attn_fwd(qd, kd, args[2], idx, wl.grid, wl.block)
    else:
        o, lse, idx = sol.sol_attention_chain(*args, wl.grid, wl.block, topk, wl.rope_split, wl.rope_theta, wl.eps)
        qd, kd = sol.sol_qk_prologue(args[0], args[1], args[3], args[4], wl.grid, wl.rope_split, wl.rope_theta,
                                     wl.eps)
    torch.cuda.synchronize()
    assert sol.sol_check_device_status() == sol.SOL_OK
    del args
    # prologue on sampled tokens: every token of the first and the last block, 4096 random ones
    rng = np.random.default_rng(5)
    last0 = (wl.nb - 1) * wl.block
    tok = np.unique(np.concatenate([np.arange(0, wl.block), np.arange(last0, wl.N), rng.integers(0, wl.N, 4096)]))
    flipped = 0
    for dev, raw, g in ((qd, q_raw, gq), (kd, k_raw, gk)):
        y64 = orc.qk_prologue(np32(raw), g.double().numpy(), wl.grid, wl.rope_split, wl.rope_theta, wl.eps,
                              tokens=tok)
        flipped += check_bf16_prologue(np32(dev[:, tok]), y64)
    # the fused path's block means: the oracle's means of the stored outputs on sampled blocks (last included)
    if chain == "fused":
        blocks = np.unique(np.concatenate([[0, wl.nb - 1], rng.integers(0, wl.nb, 30)]))
        members = [np.arange(i * wl.block, min(wl.N, (i + 1) * wl.block)) for i in blocks]
        for out, bar in ((qd, qbar), (kd, kbar)):
            sub = np.unique(np.concatenate(members))
            pos = {t: j for j, t in enumerate(sub)}
            local = [np.asarray([pos[t] for t in mem]) for mem in members]
            m, tol = pooled_tolerance(np64(out[:, sub]), local)
            err = np.abs(np64(bar[:, :, blocks]) - m)
            assert (err <= tol).all(), float((err - tol).max())
    q_ref, k_ref, s_ref, band = oracle_chain(cfg)
    idx_ref = orc.topk_blocks(s_ref, topk)
    idx_gpu = idx.cpu().numpy()
    rows, near, differ = check_selection(idx_gpu, s_ref, topk, abs_band=band)
    same_rows = np.all(idx_gpu == idx_ref, axis=-1)
    units = [u for u in sample_units(wl.B, wl.H, wl.nb, seed=1) if same_rows[u]]
    err_o, err_l = check_attention(o, lse, q_ref, k_ref, np32(v), idx_ref, wl.block, units, fp32=False)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    seq = ("sol_qk_prologue_pool -> sol_block_select_pooled -> sol_sparse_attn_fwd" if chain == "fused" else
           "sol_qk_prologue -> sol_block_select -> sol_sparse_attn_fwd")
    record_parity(f"workload{cfg}/chain_{chain}", path=seq, rows=rows, near_tie_rows=near, differing_rows=differ,
                  attention_units=len(units), ragged_last_block=bool(wl.N % wl.block),
                  last_block_units=sum(1 for u in units if u[2] == wl.nb - 1), max_abs_dO=err_o, max_abs_dLSE=err_l,
                  prologue_values_checked=2 * len(tok) * wl.H * wl.D, prologue_values_other_neighbour=flipped)
