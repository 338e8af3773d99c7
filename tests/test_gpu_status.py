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
