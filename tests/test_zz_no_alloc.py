"""sol_block_select_noalloc: block selection for callers that cannot allocate.

Some callers of this library cannot call cudaMalloc (a host framework's
launch callback that owns all device memory, or a latency-critical loop where
an allocation's implicit device synchronisation is not acceptable).  For them
libsol keeps the selection scratch in a fixed device array inside the library.
This test calls that entry point through the C ABI twice in a row, on two
different inputs, and checks each result against the workspace-taking
sol_block_select on the same input (same kernels, so ids and scores must be
identical).  It also checks that a shape needing more scratch than the array
holds is refused before any launch.  The file name makes pytest collect it
last; it passes alone in a fresh process and after the other tests.
"""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def _noalloc(sol):
    f = sol.lib.sol_block_select_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, sol.SolShape, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                  ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    return f


def _inputs(seed, B, N, H, D):
    g = torch.Generator().manual_seed(seed)
    ramp = torch.linspace(-1, 1, N).view(1, N, 1, 1)
    q = (torch.randn(B, N, H, D, generator=g) + ramp).to(torch.bfloat16).cuda()
    k = (torch.randn(B, N, H, D, generator=g) - ramp).to(torch.bfloat16).cuda()
    return q, k


def test_noalloc_select_matches_workspace_select_twice(sol):
    f = _noalloc(sol)
    B, H, D, grid, block, topk = 1, 4, 128, (4, 32, 56), 128, 12
    N = grid[0] * grid[1] * grid[2]
    nb = N // block
    shape = sol.SolShape(B, N, H, D, *grid)
    stream = torch.cuda.current_stream()
    for seed in (1, 2):                     # two calls in a row, different data
        q, k = _inputs(seed, B, N, H, D)
        idx = torch.full((B, H, nb, topk), -1, dtype=torch.int32, device="cuda")
        scores = torch.zeros((B, H, nb, nb), dtype=torch.float32, device="cuda")
        st = f(q.data_ptr(), k.data_ptr(), shape, block, topk, 1, idx.data_ptr(), scores.data_ptr(),
               ctypes.c_void_p(stream.cuda_stream))
        assert st == sol.SOL_OK, sol.sol_status_string(st)
        idx_ref, scores_ref = sol.sol_block_select(q, k, grid, block, topk, return_scores=True)
        torch.cuda.synchronize()
        assert sol.sol_check_device_status() == sol.SOL_OK
        assert torch.equal(idx, idx_ref)
        torch.testing.assert_close(scores, scores_ref, rtol=0, atol=0)


def test_noalloc_select_refuses_shapes_beyond_its_scratch(sol):
    f = _noalloc(sol)
    # 2 * B * H * nb * D * 4 bytes = 2 * 64 * 1024 * 128 * 4 = 64 MiB > 40 MiB
    B, H, D, grid, block = 1, 64, 128, (1, 1024, 128), 128
    shape = sol.SolShape(B, grid[1] * grid[2], H, D, *grid)
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    st = f(dummy.data_ptr(), dummy.data_ptr(), shape, block, 8, 1, dummy.data_ptr(), None,
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == sol.SOL_ERR_UNSUPPORTED
