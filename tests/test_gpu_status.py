"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes must give up, be reported as SOL_ERR_TIMEOUT, and leave the CUDA
context usable for the next call."""
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives(sol):
    assert sol.sol_check_device_status() == sol.SOL_OK
    sol.sol_selftest_wait_timeout(20_000)          # 20 ms, nothing ever arrives
    assert sol.sol_check_device_status() == sol.SOL_ERR_TIMEOUT
    assert sol.sol_check_device_status() == sol.SOL_OK      # the word was cleared
    # the context still works: a small attention call succeeds
    B, N, H, D = 1, 256, 1, 128
    q = torch.randn(B, N, H, D, device="cuda").to(torch.bfloat16)
    idx = torch.tensor([[[[0], [1]]]], dtype=torch.int32, device="cuda")
    o, lse = sol.sol_sparse_attn_fwd(q, q, q, idx, (1, 1, N), 128)
    assert sol.sol_check_device_status() == sol.SOL_OK
    assert torch.isfinite(o.float()).all()


def test_bad_arguments_raise_before_launch(sol):
    q = torch.zeros(1, 256, 1, 128, device="cuda", dtype=torch.bfloat16)
    idx = torch.zeros(1, 1, 2, 3, dtype=torch.int32, device="cuda")     # k = 3 > nb = 2
    with pytest.raises(sol.SolError) as e:
        sol.sol_sparse_attn_fwd(q, q, q, idx, (1, 1, 256), 128)
    assert e.value.status == sol.SOL_ERR_INVALID_ARG
    with pytest.raises(sol.SolError) as e:
        sol.sol_sparse_attn_fwd(q, q, q, idx[..., :1].contiguous(), (1, 1, 256), 64)   # bf16 needs block 128
    assert e.value.status == sol.SOL_ERR_UNSUPPORTED
    with pytest.raises(ValueError):
        sol.sol_sparse_attn_fwd(q.cpu(), q, q, idx, (1, 1, 256), 128)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_out_of_range_block_id_is_reported_not_read(sol, dtype):
    """An index list entry outside [0, nb) never addresses memory: the fp32
    kernel skips it, the tensor-core kernel reads block 0 instead, and the call
    is reported as SOL_ERR_INVALID_ARG by the next status check."""
    assert sol.sol_check_device_status() == sol.SOL_OK
    B, N, H, D, block = 1, 512, 2, 128, 128
    g = torch.Generator().manual_seed(3)
    q, k, v = (torch.randn(B, N, H, D, generator=g).to(dtype).cuda() for _ in range(3))
    idx = torch.tensor([0, 2], dtype=torch.int32).repeat(B, H, N // block, 1).contiguous().cuda()
    idx[0, 1, 3, 1] = N // block                    # one past the last block
    sol.sol_sparse_attn_fwd(q, k, v, idx, (1, 4, 128), block)
    assert sol.sol_check_device_status() == sol.SOL_ERR_INVALID_ARG
    idx[0, 1, 3, 1] = 1                             # a valid list: the context and the word are clean again
    sol.sol_sparse_attn_fwd(q, k, v, idx, (1, 4, 128), block)
    assert sol.sol_check_device_status() == sol.SOL_OK


def test_backward_reports_repeated_and_out_of_range_ids(sol):
    """The backward's inverted index records each (query block, key block) pair
    once, so a row that repeats an id cannot be differentiated: it is reported
    (SOL_ERR_INVALID_ARG), as is an id outside [0, nb)."""
    assert sol.sol_check_device_status() == sol.SOL_OK
    B, N, H, D, block = 1, 256, 1, 64, 64
    g = torch.Generator().manual_seed(4)
    q, k, v, dout = (torch.randn(B, N, H, D, generator=g).cuda() for _ in range(4))
    idx = torch.tensor([[[[0, 1], [1, 2], [2, 3], [0, 3]]]], dtype=torch.int32, device="cuda")
    o, lse = sol.sol_sparse_attn_fwd(q, k, v, idx, (1, 1, N), block)
    sol.sol_sparse_attn_bwd(q, k, v, o, lse, dout, idx, (1, 1, N), block)
    assert sol.sol_check_device_status() == sol.SOL_OK
    for bad in (1, 7):                               # a repeat of block 1, then an id past nb = 4
        idx2 = idx.clone()
        idx2[0, 0, 0, 0] = bad
        sol.sol_sparse_attn_bwd(q, k, v, o, lse, dout, idx2, (1, 1, N), block)
        assert sol.sol_check_device_status() == sol.SOL_ERR_INVALID_ARG
