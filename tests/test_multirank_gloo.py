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
