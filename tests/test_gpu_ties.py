"""GPU selection with exact ties, compared id for id with the oracle.

Inputs are small integers (|x| <= 3) over blocks of 64 tokens, so every pooled
mean is an integer / 64 and every score an integer / 4096 below 2^24 / 4096:
all of them exact in fp32, so the kernel's scores equal the oracle's fp64
scores bit for bit and no near-tie tolerance applies.  Key blocks come in
identical pairs (block 2i + 1 repeats block 2i), so odd k cuts through ties,
which must go to the lower block id; a zero Q makes every score tie.
"""
import numpy as np
import pytest
import torch

import oracle as orc

pytestmark = pytest.mark.gpu

GRID = (4, 16, 16)          # 1,024 tokens
BLOCK, H, D = 64, 2, 64


def integer_inputs(seed, zero_q=False):
    rng = np.random.default_rng(seed)
    N = GRID[0] * GRID[1] * GRID[2]
    q = rng.integers(-3, 4, size=(1, N, H, D)).astype(np.float32)
    k = rng.integers(-3, 4, size=(1, N, H, D)).astype(np.float32)
    if zero_q:
        q[:] = 0.0
    kb = k.reshape(1, N // BLOCK, BLOCK, H, D)
    kb[:, 1::2] = kb[:, 0::2]            # identical key blocks in pairs
    return q, kb.reshape(1, N, H, D)


@pytest.mark.parametrize("seed,zero_q", [(0, False), (1, False), (2, True)])
def test_exact_ties_go_to_the_lower_block(sol, seed, zero_q):
    q, k = integer_inputs(seed, zero_q)
    qd, kd = torch.from_numpy(q).cuda(), torch.from_numpy(k).cuda()
    nb = q.shape[1] // BLOCK
    for topk in (1, 3, 5, 8, nb):
        idx, scores = sol.sol_block_select(qd, kd, GRID, BLOCK, topk, return_scores=True)
        torch.cuda.synchronize()
        idx_ref, s_ref = orc.block_select(q.astype(np.float64), k.astype(np.float64), BLOCK, topk)
        assert np.array_equal(scores.cpu().numpy().astype(np.float64), s_ref)      # exact scores
        assert np.array_equal(idx.cpu().numpy(), idx_ref), topk                      # exact ids, ties included
        # and the same from block means given directly
        qbar = torch.from_numpy(orc.block_pool(q.astype(np.float64), BLOCK).astype(np.float32)).cuda()
        kbar = torch.from_numpy(orc.block_pool(k.astype(np.float64), BLOCK).astype(np.float32)).cuda()
        idx_p = sol.sol_block_select_pooled(qbar, kbar, GRID, BLOCK, topk)
        torch.cuda.synchronize()
        assert np.array_equal(idx_p.cpu().numpy(), idx_ref), topk
