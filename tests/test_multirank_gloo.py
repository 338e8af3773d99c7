"""The multi-rank host path of bench.py on CPU with the gloo backend (2 ranks).

The Sol-Attn path shards with no data exchange: every rank runs its own clip
(independent (b, h, query block) work), so the only cross-rank steps are the
barrier around the timed region and the max-over-ranks of the device time.
These tests run those steps as two gloo processes, check the reduction, and
check that per-rank work is independent (each rank's oracle result on its own
seeded inputs does not depend on the other rank).
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    import bench
    import oracle as orc
    from workloads import WORKLOADS, make_inputs
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank)
    bench.barrier(w)
    ms = bench.max_over_ranks(10.0 + rank, w)          # rank-dependent "device times"
    # independent work per rank: a tiny clip per rank, seeded by the rank
    wl = WORKLOADS[0]
    inp = make_inputs(wl, seed=rank, names=("q", "k", "v"))
    q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
    idx, _ = orc.block_select(q, k, wl.block, 4)
    o, _ = orc.sparse_attention(q, k, v, idx, wl.block, units=[(0, 0, 0), (0, 1, 5)])
    np.save(os.path.join(out_dir, f"o_{rank}.npy"), np.nan_to_num(o[0, :64, :, :]))
    with open(os.path.join(out_dir, f"ms_{rank}.txt"), "w") as f:
        f.write(str(ms))
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_max_reduction_and_independent_work(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    ms = [float(open(tmp_path / f"ms_{r}.txt").read()) for r in range(2)]
    assert ms == [11.0, 11.0]                           # every rank reports the slowest rank's time
    # each rank's result equals a single-process computation with that rank's seed
    import oracle as orc
    from workloads import WORKLOADS, make_inputs
    wl = WORKLOADS[0]
    for r in range(2):
        inp = make_inputs(wl, seed=r, names=("q", "k", "v"))
        q, k, v = (inp[n].double().numpy() for n in ("q", "k", "v"))
        idx, _ = orc.block_select(q, k, wl.block, 4)
        o, _ = orc.sparse_attention(q, k, v, idx, wl.block, units=[(0, 0, 0), (0, 1, 5)])
        np.testing.assert_array_equal(np.load(tmp_path / f"o_{r}.npy"), np.nan_to_num(o[0, :64, :, :]))
    assert not np.array_equal(np.load(tmp_path / "o_0.npy"), np.load(tmp_path / "o_1.npy"))


def test_weak_scaling_value_counts_all_ranks():
    """value = selected FLOPs of one clip x ranks / max-over-ranks step time."""
    import bench  # noqa: F401  (bench.py computes value = flops * world / (ms * 1e-3) / 1e12)
    from workloads import WORKLOADS
    wl = WORKLOADS[4]
    flops = wl.selected_flops()
    assert flops == 4 * wl.block * 102 * wl.block * wl.D * wl.nb * wl.H   # every block of 130,560 tokens is full
    for world, ms in ((1, 30.0), (8, 31.0)):
        value = flops * world / (ms * 1e-3) / 1e12
        assert abs(value - world * flops / ms / 1e9) < 1e-6


# ----------------------------------------------------------------------------- sequence-parallel exchange
def _pack_np(x, plan, split, G, stride_rows, offset_rows, codes, scales):
    """Host model of sol_quant_pack's documented layout (values copied, no quantisation):
    x [B, Nx, Hx, D] -> slice g at row g * stride_rows + offset_rows + (b * Nc + n) * Hc + h."""
    B, Nx, Hx, D = x.shape
    for b in range(B):
        for n in range(Nx):
            for h in range(Hx):
                if split == "heads":
                    Hc, Nc = Hx // G, Nx
                    g, nc, hc = h // Hc, n, h % Hc
                else:
                    Hc, Nc = Hx, Nx // G
                    g, nc, hc = n // Nc, n % Nc, h
                row = g * stride_rows + offset_rows + (b * Nc + nc) * Hc + hc
                codes[row * D:(row + 1) * D] = x[b, n, h]
                scales[row] = float(x[b, n, h, 0]) + 0.5


def _seqpar_worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import torch.distributed as dist
    from block_sparse_attention_sol_b200.seqpar import CollectiveTransport, ExchangePlan
    dist.init_process_group("gloo", rank=rank, world_size=world, init_method=f"tcp://127.0.0.1:{port}")
    B, N, H, D = 2, 12, 4, 8
    plan = ExchangePlan(world, B, N, H, D)
    Nl, Hg = plan.n_local, plan.h_local

    def code(b, n, h, d):                      # identifies (batch, global token, global head, channel)
        return (b * 101 + n * 7 + h * 13 + d) % 256

    # this rank's token shard of Q, K, V (tensor t adds 50 * t)
    shard = np.zeros((3, B, Nl, H, D), dtype=np.uint8)
    for t in range(3):
        for b in range(B):
            for n in range(Nl):
                for h in range(H):
                    shard[t, b, n, h] = [(code(b, rank * Nl + n, h, d) + 50 * t) % 256 for d in range(D)]
    send = np.zeros(plan.qkv_code_bytes, dtype=np.uint8)
    send_s = np.zeros(plan.qkv_scale_count, dtype=np.float32)
    for t in range(3):
        _pack_np(shard[t], plan, "heads", world, plan.qkv_stride_rows, plan.qkv_offset_rows(t), send, send_s)
    recv = torch.empty(plan.qkv_code_bytes, dtype=torch.uint8)
    recv_s = torch.empty(plan.qkv_scale_count, dtype=torch.float32)
    tr = CollectiveTransport()
    tr.all_to_all(recv, torch.from_numpy(send))
    tr.all_to_all(recv_s, torch.from_numpy(send_s))
    recv, recv_s = recv.numpy(), recv_s.numpy()
    # unpack as sol_dequant_unpack (split heads) documents: slice g -> tokens g * Nl ..
    ok = True
    for t in range(3):
        for g in range(world):
            for b in range(B):
                for n in range(Nl):
                    for h in range(Hg):
                        row = g * plan.qkv_stride_rows + plan.qkv_offset_rows(t) + (b * Nl + n) * Hg + h
                        n_glob, h_glob = g * Nl + n, rank * Hg + h
                        want = [(code(b, n_glob, h_glob, d) + 50 * t) % 256 for d in range(D)]
                        ok &= list(recv[row * D:(row + 1) * D]) == want
                        ok &= recv_s[row] == float(want[0]) + 0.5
    # the way back: this rank's head shard of O (all tokens) -> token shards, split tokens
    o_h = np.zeros((B, N, Hg, D), dtype=np.uint8)
    for b in range(B):
        for n in range(N):
            for h in range(Hg):
                o_h[b, n, h] = [code(b, n, rank * Hg + h, d) for d in range(D)]
    send_o = np.zeros(plan.o_code_bytes, dtype=np.uint8)
    send_os = np.zeros(plan.o_scale_count, dtype=np.float32)
    _pack_np(o_h, plan, "tokens", world, plan.rows, 0, send_o, send_os)
    recv_o = torch.empty(plan.o_code_bytes, dtype=torch.uint8)
    recv_os = torch.empty(plan.o_scale_count, dtype=torch.float32)
    tr.all_to_all(recv_o, torch.from_numpy(send_o))
    tr.all_to_all(recv_os, torch.from_numpy(send_os))
    recv_o = recv_o.numpy()
    for g in range(world):                      # slice g: heads g * Hg .. of this rank's tokens
        for b in range(B):
            for n in range(Nl):
                for h in range(Hg):
                    row = g * plan.rows + (b * Nl + n) * Hg + h
                    want = [code(b, rank * Nl + n, g * Hg + h, d) for d in range(D)]
                    ok &= list(recv_o[row * D:(row + 1) * D]) == want
    with open(os.path.join(out_dir, f"seqpar_{rank}.txt"), "w") as f:
        f.write("ok" if ok else "bad")
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_seqpar_exchange_layout_over_two_gloo_ranks(tmp_path):
    port = _free_port()
    mp.start_processes(_seqpar_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    assert [open(tmp_path / f"seqpar_{r}.txt").read() for r in range(2)] == ["ok", "ok"]


def test_exchange_plan_sizes_and_bytes():
    from block_sparse_attention_sol_b200.seqpar import ExchangePlan
    p = ExchangePlan(8, 1, 130560, 32, 128)
    assert (p.n_local, p.h_local, p.rows) == (16320, 4, 65280)
    assert p.qkv_code_bytes == 8 * 3 * 65280 * 128 and p.o_scale_count == 8 * 65280
    # INT8 / FP8 codes plus one fp32 scale per 128 channels: 132 of every 256 bf16 bytes remain, a reduction
    # by 48.4% (the pages report a reduction by 51.6%, which no 8-bit code of bf16 data with scales reaches)
    assert abs(p.wire_bytes() / p.bf16_wire_bytes() - 132 / 256) < 1e-12
    with pytest.raises(ValueError):
        ExchangePlan(3, 1, 130560, 32, 128)       # 32 heads do not split over 3 ranks
