"""Pins of the oracle's 3-D tile blocks.

Expected values come from a hand-worked case and from an independent
formulation: reshaping the token grid into tiles with numpy (reshape +
transpose) puts each tile's tokens in one contiguous run, so tiled pooling and
tiled attention must equal run-based pooling and attention on the permuted
tokens.
"""
import numpy as np
import pytest

import oracle as orc


def tile_permutation(grid, tile):
    """Token ids in tile-major order, by reshaping the grid (no index arithmetic)."""
    T, Hg, Wg = grid
    t, h, w = tile
    ids = np.arange(T * Hg * Wg).reshape(T // t, t, Hg // h, h, Wg // w, w)
    return ids.transpose(0, 2, 4, 1, 3, 5).reshape(-1)


def test_tiled_blocks_hand_case():
    blocks = orc.tiled_blocks((2, 4, 4), (1, 2, 2))
    assert len(blocks) == 8
    assert list(blocks[0]) == [0, 1, 4, 5]
    assert list(blocks[1]) == [2, 3, 6, 7]
    assert list(blocks[2]) == [8, 9, 12, 13]
    assert list(blocks[4]) == [16, 17, 20, 21]
    wide = orc.tiled_blocks((1, 4, 4), (1, 2, 4))         # tiles two rows high, four columns wide
    assert [list(b) for b in wide] == [list(range(8)), list(range(8, 16))]
    two_frames = orc.tiled_blocks((2, 2, 3), (2, 1, 3))   # one tile spans both frames
    assert [list(b) for b in two_frames] == [[0, 1, 2, 6, 7, 8], [3, 4, 5, 9, 10, 11]]


@pytest.mark.parametrize("grid,tile", [((4, 16, 16), (1, 8, 8)), ((4, 16, 16), (2, 4, 8)), ((16, 32, 56), (2, 8, 8))])
def test_tiled_blocks_partition_matches_reshape(grid, tile):
    blocks = orc.tiled_blocks(grid, tile)
    flat = np.concatenate(blocks)
    assert np.array_equal(flat, tile_permutation(grid, tile))
    assert np.array_equal(np.sort(flat), np.arange(np.prod(grid)))


def test_tiled_pool_and_attention_equal_runs_on_permuted_tokens():
    rng = np.random.default_rng(3)
    grid, tile = (2, 4, 8), (1, 2, 4)             # 64 tokens, blocks of 8
    B, N, H, D, block = 1, 64, 2, 4, 8
    q, k, v = (rng.standard_normal((B, N, H, D)) for _ in range(3))
    perm = tile_permutation(grid, tile)
    blocks = orc.tiled_blocks(grid, tile)
    assert np.allclose(orc.block_pool(q, blocks), orc.block_pool(q[:, perm], block), rtol=0, atol=1e-14)
    nb = N // block
    idx = np.stack([np.sort(rng.permutation(nb)[:3]) for _ in range(B * H * nb)]).reshape(B, H, nb, 3)
    o_t, l_t = orc.sparse_attention(q, k, v, idx, blocks, 0.5)
    o_p, l_p = orc.sparse_attention(q[:, perm], k[:, perm], v[:, perm], idx, block, 0.5)
    assert np.allclose(o_t[:, perm], o_p, rtol=0, atol=1e-12)
    assert np.allclose(l_t[:, :, perm], l_p, rtol=0, atol=1e-12)


def test_first_frame_blocks_of_tiles():
    assert orc.first_frame_blocks((16, 32, 56), 128, tile=(2, 8, 8)) == 28
    assert orc.first_frame_blocks((4, 16, 16), 64, tile=(1, 8, 8)) == 4
    blocks = orc.tiled_blocks((4, 16, 16), (2, 4, 8))
    n_first = orc.first_frame_blocks((4, 16, 16), 64, tile=(2, 4, 8))
    holds_frame0 = [bool((b < 16 * 16).any()) for b in blocks]
    assert holds_frame0 == [True] * n_first + [False] * (len(blocks) - n_first)
