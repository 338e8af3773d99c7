"""GPU parity of the fused preparation path: sol_qk_prologue_pool followed by
sol_block_select_pooled.

  * Its Q / K outputs are those of sol_qk_prologue, bit for bit.
  * Its block means are the oracle's block means of those stored outputs, within
    the error bound of an fp32 running sum of <= block values followed by one
    multiplication by the rounded reciprocal of the count:
        |r - m| <= gamma_(n-1) * mean|x| * (1 + 3u) + 3u |m|,  u = 2^-24,
    gamma_k = k u / (1 - k u)  (recursive summation bound).
  * Its selection equals sol_block_select's on the same prologue outputs, id for
    id (both pool in ascending token order in fp32), and so passes the same
    oracle selection rule.
Covered: the fp32 workload (4x16x16 grid, block 64, k = 4 and 16), a small bf16
case with a ragged last block, a small bf16 case with 40 heads, and the 896x512
workload at full size.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.gpu_common import check_selection, cpu_inputs, np64
from workloads import WORKLOADS, make_inputs, Workload

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


def pooled_tolerance(x64: np.ndarray, block: int) -> tuple[np.ndarray, np.ndarray]:
    """Oracle block means of x [B, N, H, D] and the fp32 kernel's error bound."""
    m = orc.block_pool(x64, block)
    mean_abs = orc.block_pool(np.abs(x64), block)
    k = block - 1
    gamma = k * U32 / (1 - k * U32)
    return m, gamma * mean_abs * (1 + 3 * U32) + 3 * U32 * np.abs(m)


def run_case(sol, wl: Workload, inp, topks):
    q_raw, k_raw = inp["q"].cuda(), inp["k"].cuda()
    gq, gk = inp["gamma_q"].cuda(), inp["gamma_k"].cuda()
    args = (wl.grid,)
    q_ref, k_ref = sol.sol_qk_prologue(q_raw, k_raw, gq, gk, *args, wl.rope_split, wl.rope_theta, wl.eps)
    q, k, qbar, kbar = sol.sol_qk_prologue_pool(q_raw, k_raw, gq, gk, wl.grid, wl.block, wl.rope_split,
                                                wl.rope_theta, wl.eps)
    torch.cuda.synchronize()
    assert torch.equal(q.view(torch.int16) if q.dtype == torch.bfloat16 else q,
                       q_ref.view(torch.int16) if q_ref.dtype == torch.bfloat16 else q_ref)
    assert torch.equal(k.view(torch.int16) if k.dtype == torch.bfloat16 else k,
                       k_ref.view(torch.int16) if k_ref.dtype == torch.bfloat16 else k_ref)
    assert qbar.shape == (wl.B, wl.H, wl.nb, wl.D)
    for out, bar in ((q, qbar), (k, kbar)):
        m, tol = pooled_tolerance(np64(out), wl.block)
        err = np.abs(np64(bar) - m)
        assert (err <= tol).all(), float((err - tol).max())
    for topk in topks:
        idx_f, s_f = sol.sol_block_select_pooled(qbar, kbar, wl.grid, wl.block, topk, return_scores=True)
        idx_u, s_u = sol.sol_block_select(q, k, wl.grid, wl.block, topk, return_scores=True)
        torch.cuda.synchronize()
        assert torch.equal(s_f, s_u)
        assert torch.equal(idx_f, idx_u)
        if wl.config_id == 0:   # and the oracle's selection rule on the stored outputs
            _, s_ref = orc.block_select(np64(q), np64(k), wl.block, topk)
            check_selection(idx_f.cpu().numpy(), s_ref, topk)


def test_fused_workload0_fp32(sol):
    wl = WORKLOADS[0]
    run_case(sol, wl, cpu_inputs(0), wl.topk)


def test_fused_small_bf16_ragged_block(sol):
    # 3 x 8 x 40 grid = 960 tokens: 7 full blocks of 128 and a last block of 64
    wl = Workload(config_id=90, name="small bf16, ragged last block", dtype="bf16", B=2, H=4, D=128,
                  grid=(3, 8, 40), block=128, topk=(3,))
    assert wl.N % wl.block == 64
    run_case(sol, wl, make_inputs(wl, seed=5), (1, 3, wl.nb))


def test_fused_small_bf16_many_heads(sol):
    # 40 heads: more than the staged kernel's 32 row groups, so both prologue
    # entry points take the register-streaming kernels
    wl = Workload(config_id=91, name="small bf16, 40 heads", dtype="bf16", B=1, H=40, D=128,
                  grid=(2, 8, 24), block=128, topk=(2,))
    run_case(sol, wl, make_inputs(wl, seed=6), (1, 2, wl.nb))


def test_fused_workload1_bf16_full(sol):
    wl = WORKLOADS[1]
    run_case(sol, wl, cpu_inputs(1), wl.topk)


def test_host_pipeline_matches_direct_calls(sol):
    """Clips streamed through HostChainPipeline (three streams, double-buffered
    device buffers) give exactly the outputs of the direct fused chain on each clip."""
    from block_sparse_attention_sol_b200.pipeline import HostChainPipeline
    wl = Workload(config_id=91, name="pipeline check, ragged last block", dtype="bf16", B=1, H=4, D=128,
                  grid=(3, 8, 40), block=128, topk=(3,))
    topk = 3
    clips = [make_inputs(wl, seed=s) for s in range(5)]
    gq, gk = clips[0]["gamma_q"].cuda(), clips[0]["gamma_k"].cuda()
    pipe = HostChainPipeline(wl.B, wl.N, wl.H, wl.D, wl.grid, wl.block, topk, gq, gk, rope_split=wl.rope_split,
                             rope_theta=wl.rope_theta, eps=wl.eps)
    outs = []
    for c in clips:
        host = {n: c[n].pin_memory() for n in ("q", "k", "v")}
        o_host = torch.empty(c["q"].shape, dtype=c["q"].dtype).pin_memory()
        lse_host = torch.empty((wl.B, wl.H, wl.N), dtype=torch.float32).pin_memory()
        pipe.submit(host["q"], host["k"], host["v"], o_host, lse_host)
        outs.append((host, o_host, lse_host))
    pipe.synchronize()
    for c, (_, o_host, lse_host) in zip(clips, outs):
        q, k, qbar, kbar = sol.sol_qk_prologue_pool(c["q"].cuda(), c["k"].cuda(), gq, gk, wl.grid, wl.block,
                                                    wl.rope_split, wl.rope_theta, wl.eps)
        idx = sol.sol_block_select_pooled(qbar, kbar, wl.grid, wl.block, topk)
        o, lse = sol.sol_sparse_attn_fwd(q, k, c["v"].cuda(), idx, wl.grid, wl.block)
        torch.cuda.synchronize()
        assert torch.equal(o.cpu().view(torch.int16), o_host.view(torch.int16))
        assert torch.equal(lse.cpu(), lse_host)
    assert sol.sol_check_device_status() == sol.SOL_OK


def test_chain_graph_matches_direct_calls(sol):
    """The fused chain captured once as a CUDA graph (ChainGraph) and replayed on
    three clips gives exactly the outputs of the direct calls on each clip."""
    from block_sparse_attention_sol_b200.graph import ChainGraph
    wl = Workload(config_id=93, name="graph check, ragged last block", dtype="bf16", B=1, H=4, D=128,
                  grid=(3, 8, 40), block=128, topk=(3,))
    topk = 3
    clips = [make_inputs(wl, seed=s) for s in range(3)]
    gq, gk = clips[0]["gamma_q"].cuda(), clips[0]["gamma_k"].cuda()
    chain = ChainGraph(wl.B, wl.N, wl.H, wl.D, wl.grid, wl.block, topk, gq, gk, rope_split=wl.rope_split,
                       rope_theta=wl.rope_theta, eps=wl.eps).capture()
    for c in clips:
        o_g, lse_g = chain(c["q"].cuda(), c["k"].cuda(), c["v"].cuda())
        o_g, lse_g = o_g.clone(), lse_g.clone()
        q, k, qbar, kbar = sol.sol_qk_prologue_pool(c["q"].cuda(), c["k"].cuda(), gq, gk, wl.grid, wl.block,
                                                    wl.rope_split, wl.rope_theta, wl.eps)
        idx = sol.sol_block_select_pooled(qbar, kbar, wl.grid, wl.block, topk)
        o, lse = sol.sol_sparse_attn_fwd(q, k, c["v"].cuda(), idx, wl.grid, wl.block)
        torch.cuda.synchronize()
        assert torch.equal(o_g.view(torch.int16), o.view(torch.int16))
        assert torch.equal(lse_g, lse)
    assert sol.sol_check_device_status() == sol.SOL_OK
