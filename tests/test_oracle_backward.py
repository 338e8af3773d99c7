"""Pins of the oracle's attention backward against torch autograd in float64
(a library routine) on the dense attention masked to the kept blocks."""
import numpy as np
import pytest
import torch

import oracle as orc


def dense_masked_autograd(q, k, v, do, idx, block, scale, counts=None):
    B, N, H, D = q.shape
    nb = -(-N // block)
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    mask = torch.zeros(B, H, N, N, dtype=torch.bool)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                kept = idx[b, h, i][: None if counts is None else int(counts[b, h, i])]
                for j in kept:
                    mask[b, h, i * block:(i + 1) * block, j * block:(j + 1) * block] = True
    s = scale * torch.einsum("bnhd,bmhd->bhnm", qt, kt)
    p = torch.softmax(s.masked_fill(~mask, float("-inf")), dim=-1)
    o = torch.einsum("bhnm,bmhd->bnhd", p, vt)
    o.backward(torch.tensor(do, dtype=torch.float64))
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


@pytest.mark.parametrize("with_counts", [False, True])
def test_backward_matches_autograd(with_counts):
    rng = np.random.default_rng(21)
    B, N, H, D, block = 2, 36, 2, 8, 8          # 5 blocks, the last one of 4 tokens
    q, k, v, do = (rng.standard_normal((B, N, H, D)) for _ in range(4))
    nb = -(-N // block)
    idx = np.stack([rng.permutation(nb)[:3] for _ in range(B * H * nb)]).reshape(B, H, nb, 3).astype(np.int32)
    counts = rng.integers(1, 4, size=(B, H, nb)) if with_counts else None
    scale = 0.4
    got = orc.sparse_attention_backward(q, k, v, idx, do, block, scale, counts=counts)
    want = dense_masked_autograd(q, k, v, do, idx, block, scale, counts=counts)
    for g, w in zip(got, want):
        assert np.allclose(g, w, rtol=0, atol=1e-12)


def test_backward_dv_closed_form_single_block():
    # one query block keeping one key block: dv = P^T do with P the block softmax
    rng = np.random.default_rng(22)
    q, k, v, do = (rng.standard_normal((1, 4, 1, 3)) for _ in range(4))
    idx = np.array([[[[0]]]], dtype=np.int32)
    _, _, dv = orc.sparse_attention_backward(q, k, v, idx, do, 4, 1.0)
    s = q[0, :, 0] @ k[0, :, 0].T
    p = np.exp(s - s.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert np.allclose(dv[0, :, 0], p.T @ do[0, :, 0], rtol=0, atol=1e-13)


def test_repeated_id_means_the_block_counts_twice():
    """A row that lists a key block twice attends to its keys twice: the
    oracle's forward equals dense attention over the concatenated key list
    (torch SDPA in float64 over [K_0, K_1, K_1], closed form of the multiset),
    and its backward equals autograd of that forward.  The library rejects such
    rows in the backward (its inverted index records each pair once), so this
    pins the definition a caller's repeated id would get, not the kernels."""
    rng = np.random.default_rng(23)
    B, N, H, D, block = 1, 16, 1, 4, 8            # 2 blocks
    q, k, v, do = (rng.standard_normal((B, N, H, D)) for _ in range(4))
    idx = np.array([[[[0, 1, 1], [1, 0, 0]]]], dtype=np.int32)
    scale = 0.5
    o, lse = orc.sparse_attention(q, k, v, idx, block, scale)
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    outs = []
    for i in range(2):
        rows = slice(i * block, (i + 1) * block)
        cols = np.concatenate([np.arange(j * block, (j + 1) * block) for j in idx[0, 0, i]])
        qi = qt[0, rows, 0][None, None]
        kj, vj = kt[0, cols, 0][None, None], vt[0, cols, 0][None, None]
        outs.append(torch.nn.functional.scaled_dot_product_attention(qi, kj, vj, scale=scale)[0, 0])
        logits = scale * (q[0, rows, 0] @ k[0, cols, 0].T)
        m = logits.max(axis=1)
        assert np.allclose(lse[0, 0, rows], m + np.log(np.exp(logits - m[:, None]).sum(axis=1)), rtol=0, atol=1e-13)
    ot = torch.cat(outs)
    assert np.allclose(o[0, :, 0], ot.detach().numpy(), rtol=0, atol=1e-13)
    ot.backward(torch.tensor(do[0, :, 0]))
    got = orc.sparse_attention_backward(q, k, v, idx, do, block, scale)
    for g, t in zip(got, (qt, kt, vt)):
        assert np.allclose(g, t.grad.numpy(), rtol=0, atol=1e-12)
