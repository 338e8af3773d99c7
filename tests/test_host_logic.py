"""Host-side logic of the Python binding and the sequence-parallel runtime (no GPU):
argument checks that must fire before any CUDA call, and buffer planning."""
import pytest
import torch

import block_sparse_attention_sol_b200 as sol
from block_sparse_attention_sol_b200.seqpar import ExchangePlan, LocalTransport, SeqParallelAttention


def test_binding_rejects_host_tensors():
    x = torch.zeros(1, 1024, 2, 64)
    means = torch.zeros(1, 2, 16, 64)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sol.sol_block_select_pooled_ex(means, means, (4, 16, 16), 64, 4)
    with pytest.raises(ValueError, match="CUDA tensor"):
        sol.sol_sparse_attn_fwd_tiled(x, x, x, torch.zeros(1, 2, 16, 4, dtype=torch.int32), (4, 16, 16), (1, 8, 8))
    with pytest.raises(ValueError, match="CUDA tensor"):
        sol.sol_quant_pack(x.to(torch.bfloat16), 1, sol.SOL_SPLIT_HEADS, sol.SOL_CODE_INT8,
                           torch.zeros(10, dtype=torch.uint8), torch.zeros(10))


def test_exchange_plan_offsets():
    p = ExchangePlan(4, 2, 64, 8, 128)
    assert (p.n_local, p.h_local, p.rows) == (16, 2, 2 * 16 * 2)
    assert [p.qkv_offset_rows(t) for t in range(3)] == [0, p.rows, 2 * p.rows]
    assert p.qkv_stride_rows == 3 * p.rows
    assert p.qkv_code_bytes == 4 * 3 * p.rows * 128 and p.qkv_scale_count == 4 * 3 * p.rows
    assert p.wire_bytes() == 3 * 4 * p.rows * (128 + 4)          # three other ranks, four tensors
    assert ExchangePlan(1, 2, 64, 8, 128).wire_bytes() == 0
    for bad in ((0, 1, 64, 8, 128), (3, 1, 64, 8, 128), (4, 1, 66, 8, 128)):
        with pytest.raises(ValueError):
            ExchangePlan(*bad)


def test_seqpar_runtime_validates_and_plans_on_the_host():
    H, D = 8, 128
    g = torch.ones(H * D)
    sp = SeqParallelAttention(1, 2, 1, 1024, H, D, (4, 16, 16), 128, 4, g, g, device="cpu")
    p = sp.plan
    assert sp.send_qkv.numel() == p.qkv_code_bytes and sp.recv_o_s.numel() == p.o_scale_count
    assert tuple(sp.q_h.shape) == (1, 1024, H // 2, D)
    assert sp.gamma_q.numel() == (H // 2) * D
    with pytest.raises(ValueError):
        SeqParallelAttention(2, 2, 1, 1024, H, D, (4, 16, 16), 128, 4, g, g, device="cpu")   # rank out of range
    with pytest.raises(ValueError):
        SeqParallelAttention(0, 2, 1, 1000, H, D, (4, 16, 16), 128, 4, g, g, device="cpu")   # grid != N
    with pytest.raises(ValueError):
        sp.stage_pack(torch.zeros(1, 100, H, D), torch.zeros(1, 100, H, D), torch.zeros(1, 100, H, D))


def test_local_transport_copies():
    src = torch.arange(12, dtype=torch.float32)
    dst = torch.zeros(12)
    LocalTransport().all_to_all(dst, src)
    assert torch.equal(dst, src)


def test_runners_require_gains_on_their_device():
    """HostChainPipeline and ChainGraph check, before allocating anything, that the
    gains live on the device they run on."""
    from block_sparse_attention_sol_b200.graph import ChainGraph
    from block_sparse_attention_sol_b200.pipeline import HostChainPipeline
    gq = gk = torch.ones(2 * 128)
    for runner in (HostChainPipeline, ChainGraph):
        with pytest.raises(ValueError, match="device"):
            runner(1, 1024, 2, 128, (4, 16, 16), 128, 2, gq, gk, device="cuda:0")


def test_chain_graph_replay_needs_capture():
    from block_sparse_attention_sol_b200.graph import ChainGraph
    g = ChainGraph.__new__(ChainGraph)
    g.graph = None
    with pytest.raises(RuntimeError, match="capture"):
        g.replay()
