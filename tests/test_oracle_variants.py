"""Pins of the oracle's selection variants and count-limited attention.

Each expected value comes from an independent formulation: the kept set as the
subset of a given size with the largest score sum (distinct scores), found by
enumerating all subsets; the top-p count as the smallest subset of any kind
whose softmax mass reaches p, found the same way; and count-limited attention
as dense float64 library attention under a key mask.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle as orc


def _scores(seed, B=1, H=2, nb=7):
    rng = np.random.default_rng(seed)
    return rng.standard_normal((B, H, nb, nb))      # continuous: no exact ties


def _best_subset(row, pool, size):
    """The size-subset of `pool` with the largest score sum (unique for distinct scores)."""
    if size <= 0:
        return set()
    return set(max(itertools.combinations(pool, size), key=lambda c: sum(row[j] for j in c)))


def _row_set(idx_row, count):
    got = [int(j) for j in idx_row]
    assert all(j == -1 for j in got[count:])
    assert got[:count] == sorted(got[:count])
    return set(got[:count])


def test_no_options_is_plain_topk():
    s = _scores(0, nb=9)
    for k in (1, 3, 9):
        idx, counts = orc.select_variant(s, k)
        assert np.array_equal(idx, orc.topk_blocks(s, k))
        assert (counts == k).all()


@pytest.mark.parametrize("k", [1, 2, 4])
def test_forced_diagonal_brute_force(k):
    s = _scores(1)
    nb = s.shape[-1]
    idx, counts = orc.select_variant(s, k, diagonal=True)
    for h in range(s.shape[1]):
        for i in range(nb):
            row = s[0, h, i]
            want = {i} | _best_subset(row, [j for j in range(nb) if j != i], k - 1)
            assert _row_set(idx[0, h, i], counts[0, h, i]) == want
            assert counts[0, h, i] == k


@pytest.mark.parametrize("k,first", [(4, 2), (3, 3), (2, 3)])
def test_forced_first_frame_brute_force(k, first):
    s = _scores(2)
    nb = s.shape[-1]
    idx, counts = orc.select_variant(s, k, first_blocks=first)
    for h in range(s.shape[1]):
        for i in range(nb):
            row = s[0, h, i]
            if first >= k:
                want = set(range(k))                 # too many forced blocks: the lowest ids
            else:
                want = set(range(first)) | _best_subset(row, range(first, nb), k - first)
            assert _row_set(idx[0, h, i], counts[0, h, i]) == want


def test_first_frame_block_count():
    assert orc.first_frame_blocks((16, 32, 56), 128) == 14       # 1,792 tokens per frame
    assert orc.first_frame_blocks((4, 16, 16), 64) == 4
    assert orc.first_frame_blocks((31, 48, 84), 128) == 32       # 4,032 tokens: 31.5 blocks


@pytest.mark.parametrize("p", [0.05, 0.3, 0.6, 0.9, 1.0])
def test_top_p_count_is_smallest_subset_reaching_p(p):
    s = _scores(3, nb=7) * 2.0
    nb, k, scale = s.shape[-1], 5, 0.7
    idx, counts = orc.select_variant(s, k, top_p=p, scale=scale)
    for h in range(s.shape[1]):
        for i in range(nb):
            row = s[0, h, i]
            w = np.exp(scale * row)
            w = w / w.sum()
            c_p = min(size for size in range(1, nb + 1) for c in itertools.combinations(range(nb), size)
                      if sum(w[j] for j in c) >= p - 1e-12)
            c = min(k, max(1, c_p))
            assert counts[0, h, i] == c, (h, i)
            assert _row_set(idx[0, h, i], c) == _best_subset(row, range(nb), c)


def test_top_p_with_forced_blocks_keeps_them():
    s = _scores(4, nb=8)
    idx, counts = orc.select_variant(s, 6, diagonal=True, first_blocks=2, top_p=0.01, scale=1.0)
    for i in range(8):
        kept = _row_set(idx[0, 0, i], counts[0, 0, i])
        assert {0, 1, i} <= kept
        assert counts[0, 0, i] == len({0, 1, i})   # a tiny p needs nothing beyond the forced blocks


def test_top_p_limits():
    s = _scores(5, nb=9)
    _, c1 = orc.select_variant(s, 4, top_p=1.0, scale=1.0)
    assert (c1 == 4).all()                         # full mass needs every block: capped at k
    idx, c0 = orc.select_variant(s, 4, top_p=1e-9, scale=1.0)
    assert (c0 == 1).all()
    assert np.array_equal(idx[..., 0], np.argmax(s, axis=-1))


def test_per_head_k():
    s = _scores(6, H=3, nb=8)
    head_k = np.array([1, 5, 99])
    idx, counts = orc.select_variant(s, 6, head_k=head_k)
    for h, kh in enumerate((1, 5, 6)):
        assert (counts[0, h] == kh).all()
        assert np.array_equal(idx[0, h, :, :kh], orc.topk_blocks(s[:, h], kh)[0])
        assert (idx[0, h, :, kh:] == -1).all()


def test_count_limited_attention_matches_masked_library_attention():
    rng = np.random.default_rng(8)
    B, N, H, D, block = 1, 40, 2, 8, 8          # 5 blocks
    q, k, v = (rng.standard_normal((B, N, H, D)) for _ in range(3))
    idx = np.array([[[[3, 0, 4], [1, 2, 0], [2, 4, 1], [0, 3, 2], [4, 1, 3]]] * H], dtype=np.int32)
    counts = np.array([[[1, 3, 2, 1, 2], [3, 1, 1, 2, 3]]], dtype=np.int32)
    scale = 0.3
    o, lse = orc.sparse_attention(q, k, v, idx, block, scale, counts=counts)
    nb = N // block
    for h in range(H):
        mask = np.zeros((N, N), dtype=bool)
        for i in range(nb):
            for j in idx[0, h, i, :counts[0, h, i]]:
                mask[i * block:(i + 1) * block, j * block:(j + 1) * block] = True
        qt, kt, vt = (torch.from_numpy(x[0, :, h]) for x in (q, k, v))
        want = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None],
                                                                attn_mask=torch.from_numpy(mask)[None], scale=scale)[0]
        logits = scale * (qt @ kt.T)
        want_lse = torch.logsumexp(logits.masked_fill(~torch.from_numpy(mask), -np.inf), dim=1)
        assert np.allclose(o[0, :, h], want.numpy(), rtol=0, atol=1e-12)
        assert np.allclose(lse[0, h], want_lse.numpy(), rtol=0, atol=1e-12)
