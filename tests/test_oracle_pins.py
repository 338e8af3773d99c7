"""Pins of the CPU oracle against facts that do not come from the oracle itself.

The Sol-H3 pages print no worked Sol-Attn example, so every pin here is a
hand-derived closed form, a brute-force enumeration on tiny inputs, an
invariant of the mathematics, or an independent library routine
(torch scaled_dot_product_attention / logsumexp in float64).
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle as orc
from workloads import WORKLOADS, make_inputs, rope_split_for

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_round_hand_values():
    u = 2.0 ** -7   # bf16 spacing on [1, 2)
    cases = {
        1.0: 1.0,
        1.0 + u / 2: 1.0,                 # tie -> even mantissa (0)
        1.0 + 3 * u / 2: 1.0 + 2 * u,     # tie -> even mantissa (2)
        1.0 + u / 2 + 2.0 ** -20: 1.0 + u,
        -(1.0 + 3 * u / 2): -(1.0 + 2 * u),
        3.0 * 2.0 ** -130: 3.0 * 2.0 ** -130,   # subnormal, exactly representable
        0.0: 0.0,
    }
    for x, want in cases.items():
        assert orc.bf16_round(np.array([x]))[0] == want, x


def test_bf16_round_matches_torch_from_fp32():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(200_000) * np.exp(rng.uniform(-30, 30, 200_000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = orc.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, want)


# ---------------------------------------------------------------- a1 prologue
def test_prologue_hand_case():
    # D=8 split (4,2,2): pairs 0,1 follow t (freqs 1, theta^-0.5 = 0.01), pair 2 follows y,
    # pair 3 follows x.  Token (t,y,x) = (1,2,3) of a 2x3x4 grid is n = (1*3+2)*4+3 = 23.
    grid, split, theta, eps = (2, 3, 4), (4, 2, 2), 10000.0, 0.25
    x = np.zeros((1, 24, 2, 8))
    raw = np.array([1, 2, 1, 0, 1, 0, 0, 1], dtype=np.float64)
    x[0, 23, 0] = raw
    x[0, 23, 1] = raw
    gamma = np.concatenate([np.ones(8), np.full(8, 3.0)])
    out = orc.qk_prologue(x, gamma, grid, split, theta, eps)
    c = 1.0 / math.sqrt(1.0 + 0.25)         # mean(raw^2) = 1
    want = c * np.array([
        math.cos(1) - 2 * math.sin(1), math.sin(1) + 2 * math.cos(1),   # (1,2) by t=1
        math.cos(0.01), math.sin(0.01),                                 # (1,0) by t*0.01
        math.cos(2), math.sin(2),                                       # (1,0) by y=2
        -math.sin(3), math.cos(3),                                      # (0,1) by x=3
    ])
    np.testing.assert_allclose(out[0, 23, 0], want, rtol=0, atol=1e-14)
    np.testing.assert_allclose(out[0, 23, 1], 3 * want, rtol=0, atol=1e-14)


def _random_prologue_input(grid=(3, 4, 5), H=2, D=16, seed=0):
    rng = np.random.default_rng(seed)
    N = grid[0] * grid[1] * grid[2]
    return rng.standard_normal((1, N, H, D)), grid, rope_split_for(D)


def test_prologue_unit_rms_and_identity_at_origin():
    x, grid, split = _random_prologue_input()
    H, D = x.shape[2], x.shape[3]
    out = orc.qk_prologue(x, np.ones(H * D), grid, split, 10000.0, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(out ** 2, axis=-1)), 1.0, atol=1e-12)
    # token 0 sits at (0,0,0): every angle is 0, so the output is the normalised input
    rms0 = np.sqrt(np.mean(x[0, 0] ** 2, axis=-1, keepdims=True))
    np.testing.assert_allclose(out[0, 0], x[0, 0] / rms0, atol=1e-13)
    # per-pair norms are preserved by the rotation
    rms = np.sqrt(np.mean(x ** 2, axis=-1, keepdims=True))
    y = x / rms
    np.testing.assert_allclose(out[..., 0::2] ** 2 + out[..., 1::2] ** 2,
                               y[..., 0::2] ** 2 + y[..., 1::2] ** 2, atol=1e-12)


def test_prologue_relative_position():
    # <R(p) a, R(p') b> depends only on p - p' (per axis).
    grid = (3, 4, 5)
    D, H = 16, 1
    split = rope_split_for(D)
    rng = np.random.default_rng(3)
    a, b = rng.standard_normal(D), rng.standard_normal(D)

    def tok(t, y, x):
        return (t * grid[1] + y) * grid[2] + x

    def rotated_dot(pa, pb):
        x = np.zeros((1, grid[0] * grid[1] * grid[2], H, D))
        x[0, tok(*pa), 0] = a
        x[0, tok(*pb), 0] = b
        out = orc.qk_prologue(x, np.ones(D), grid, split, 10000.0, 1e-6)
        return out[0, tok(*pa), 0] @ out[0, tok(*pb), 0]

    p1, p2 = (0, 1, 1), (1, 3, 2)
    shift = (1, -1, 2)                        # keeps both tokens on the 3x4x5 grid
    q1 = tuple(u + d for u, d in zip(p1, shift))
    q2 = tuple(u + d for u, d in zip(p2, shift))
    d1 = rotated_dot(p1, p2)
    assert abs(d1 - rotated_dot(q1, q2)) < 1e-12
    assert abs(d1 - rotated_dot(q1, p2)) > 1e-6     # a different offset changes it


def test_prologue_gamma_indexing_and_eps():
    x, grid, split = _random_prologue_input(H=3, D=8, seed=5)
    H, D = 3, 8
    gamma = np.arange(1, H * D + 1, dtype=np.float64)
    eps = 0.7
    out = orc.qk_prologue(x, gamma, grid, split, 10000.0, eps)
    ref = orc.qk_prologue(x, np.ones(H * D), grid, split, 10000.0, eps)
    # RoPE mixes channel pairs, so undo it by checking at the origin token only
    np.testing.assert_allclose(out[0, 0], ref[0, 0] * gamma.reshape(H, D), rtol=1e-13)
    rms = np.sqrt(np.mean(x[0, 0] ** 2, axis=-1, keepdims=True) + eps)
    np.testing.assert_allclose(ref[0, 0], x[0, 0] / rms, rtol=1e-13)


# ---------------------------------------------------------------- a2/a3 pooling + scores
def test_pool_hand_case():
    x = np.arange(10, dtype=np.float64).reshape(1, 10, 1, 1)   # tokens 0..9
    p = orc.block_pool(x, 4)
    np.testing.assert_array_equal(p[0, 0, :, 0], [1.5, 5.5, 8.5])   # last block: (8+9)/2


def test_scores_equal_mean_of_dense_logit_blocks():
    rng = np.random.default_rng(11)
    B, N, H, D, blk = 2, 10, 3, 5, 4
    q = rng.standard_normal((B, N, H, D))
    k = rng.standard_normal((B, N, H, D))
    s = orc.block_scores(orc.block_pool(q, blk), orc.block_pool(k, blk))
    nb = 3
    for b in range(B):
        for h in range(H):
            L = q[b, :, h, :] @ k[b, :, h, :].T          # dense q.k over all tokens
            for i in range(nb):
                for j in range(nb):
                    want = L[i * blk:(i + 1) * blk, j * blk:(j + 1) * blk].mean()
                    assert abs(s[b, h, i, j] - want) < 1e-12


# ---------------------------------------------------------------- a4 top-k
def _brute_force_topk(row, k):
    """The unique k-subset S with: for i in S, j not in S, s_i > s_j or (s_i == s_j and i < j)."""
    n = len(row)
    found = []
    for S in itertools.combinations(range(n), k):
        rest = [j for j in range(n) if j not in S]
        if all(row[i] > row[j] or (row[i] == row[j] and i < j) for i in S for j in rest):
            found.append(S)
    assert len(found) == 1
    return list(found[0])


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(2)
    for trial in range(300):
        n = int(rng.integers(1, 9))
        k = int(rng.integers(1, min(3, n) + 1))
        row = rng.integers(0, 4, size=n).astype(np.float64)     # many exact ties
        got = orc.topk_blocks(row[None], k)[0].tolist()
        assert got == _brute_force_topk(row, k), (row, k)


def test_near_tie_rows_hand_case():
    s = np.array([[5.0, 4.0, 3.0, 2.0],
                  [5.0, 4.0, 4.0 - 1e-5, 1.0],
                  [5.0, 4.0, 4.0, 1.0]])
    np.testing.assert_array_equal(orc.near_tie_rows(s, 2), [False, True, True])
    np.testing.assert_array_equal(orc.near_tie_rows(s, 4), [False, False, False])


def test_selection_permutation_and_scale():
    rng = np.random.default_rng(4)
    B, H, D, blk, nb, k = 1, 2, 8, 4, 7, 3
    N = blk * nb
    q = rng.standard_normal((B, N, H, D))
    kk = rng.standard_normal((B, N, H, D))
    idx, _ = orc.block_select(q, kk, blk, k)
    perm = rng.permutation(nb)                    # new block j holds old block perm[j]
    kp = kk.reshape(B, nb, blk, H, D)[:, perm].reshape(B, N, H, D)
    idx_p, _ = orc.block_select(q, kp, blk, k)
    inv = np.argsort(perm)
    want = np.sort(inv[idx], axis=-1)
    np.testing.assert_array_equal(idx_p, want)
    idx_2, _ = orc.block_select(2.0 * q, kk, blk, k)
    np.testing.assert_array_equal(idx_2, idx)


# ---------------------------------------------------------------- a5 attention
def test_attention_all_blocks_equals_dense_library_attention():
    rng = np.random.default_rng(9)
    B, N, H, D, blk = 1, 10, 2, 6, 4
    q, k, v = (rng.standard_normal((B, N, H, D)) for _ in range(3))
    nb = 3
    idx = np.tile(np.arange(nb, dtype=np.int32), (B, H, nb, 1))
    o, lse = orc.sparse_attention(q, k, v, idx, blk)
    tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)
    lse_ref = torch.logsumexp(tq @ tk.transpose(-1, -2) / math.sqrt(D), dim=-1).numpy()
    np.testing.assert_allclose(lse, lse_ref, atol=1e-12)


def test_attention_workload0_dense_case_matches_library():
    wl = WORKLOADS[0]
    t = make_inputs(wl, names=("q", "k", "v"))
    q, k, v = (t[n].double().numpy() for n in ("q", "k", "v"))
    idx = np.tile(np.arange(wl.nb, dtype=np.int32), (wl.B, wl.H, wl.nb, 1))
    o, lse = orc.sparse_attention(q, k, v, idx, wl.block)
    tq, tk, tv = (torch.from_numpy(a).permute(0, 2, 1, 3) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-11)
    lse_ref = torch.logsumexp(tq @ tk.transpose(-1, -2) / math.sqrt(wl.D), dim=-1).numpy()
    np.testing.assert_allclose(lse, lse_ref, atol=1e-11)


def test_attention_hand_cases():
    # N=4, D=2, block=2.  q = 0 makes every logit 0: O is the mean of the kept V rows.
    v = np.array([[1.0, 0.0], [0.0, 2.0], [4.0, 6.0], [8.0, 10.0]]).reshape(1, 4, 1, 2)
    q = np.zeros((1, 4, 1, 2))
    k = np.ones((1, 4, 1, 2))
    idx = np.array([[[[1], [0]]]], dtype=np.int32)          # block 0 keeps block 1, block 1 keeps block 0
    o, lse = orc.sparse_attention(q, k, v, idx, 2)
    np.testing.assert_allclose(o[0, 0:2, 0], [[6.0, 8.0]] * 2)
    np.testing.assert_allclose(o[0, 2:4, 0], [[0.5, 1.0]] * 2)
    np.testing.assert_allclose(lse, math.log(2.0))
    # two keys with logits s*a, s*b: weight of the first is sigmoid(s*(a-b))
    a, b = 1.5, -0.5
    q = np.array([1.0, 0.0] * 4).reshape(1, 4, 1, 2)
    k = np.array([[a, 0.0], [b, 0.0], [0, 0], [0, 0]]).reshape(1, 4, 1, 2)
    idx = np.array([[[[0], [0]]]], dtype=np.int32)
    o, lse = orc.sparse_attention(q, k, v, idx, 2)
    s = 1 / math.sqrt(2)
    w = 1 / (1 + math.exp(-s * (a - b)))
    np.testing.assert_allclose(o[0, 0, 0], w * v[0, 0, 0] + (1 - w) * v[0, 1, 0], atol=1e-14)
    np.testing.assert_allclose(lse[0, 0, 0], math.log(math.exp(s * a) + math.exp(s * b)), atol=1e-14)


def test_attention_lse_merge_and_order_invariance():
    rng = np.random.default_rng(21)
    B, H, D, blk, nb = 1, 2, 8, 4, 6
    N = blk * nb - 1                          # ragged last block
    q, k, v = (rng.standard_normal((B, N, H, D)) for _ in range(3))
    idx = np.stack([np.stack([np.sort(rng.permutation(nb)[:4]) for _ in range(nb)]) for _ in range(H)])[None]
    idx = idx.astype(np.int32)
    o, lse = orc.sparse_attention(q, k, v, idx, blk)
    oA, lA = orc.sparse_attention(q, k, v, idx[..., :2], blk)
    oB, lB = orc.sparse_attention(q, k, v, idx[..., 2:], blk)
    l_all = np.logaddexp(lA, lB)
    np.testing.assert_allclose(lse, l_all, atol=1e-12)
    wA = np.exp(lA - l_all).transpose(0, 2, 1)[..., None]
    wB = np.exp(lB - l_all).transpose(0, 2, 1)[..., None]
    np.testing.assert_allclose(o, wA * oA + wB * oB, atol=1e-12)
    o_rev, lse_rev = orc.sparse_attention(q, k, v, idx[..., ::-1], blk)
    np.testing.assert_allclose(o_rev, o, atol=1e-12)
    np.testing.assert_allclose(lse_rev, lse, atol=1e-12)
    assert np.all(np.abs(o) <= np.abs(v).max() + 1e-12)    # convex combination of V rows


def test_selected_flops_hand_case():
    N, blk, D = 10, 4, 3
    idx = np.tile(np.arange(3, dtype=np.int32), (1, 1, 3, 1))
    assert orc.selected_flops(idx, N, blk, D) == 4 * D * N * N
    idx1 = np.array([[[[2], [2], [0]]]], dtype=np.int32)      # blocks of size 4, 4, 2
    assert orc.selected_flops(idx1, N, blk, D) == 4 * D * (4 * 2 + 4 * 2 + 2 * 4)
