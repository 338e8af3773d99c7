"""Plant plausible mistakes in the oracle (on the CPU) and check that a pin catches each.

Each mutation replaces one oracle function by a subtly wrong copy; the listed
pin tests must then fail.  This guards the pins themselves: a pin that still
passes with a dropped term, a wrong sign or index, or a transposed operand
would not be pinning anything.
"""
import math

import numpy as np
import pytest

import oracle
import oracle.sol_oracle as so
from tests import test_oracle_pins as pins
from tests import test_oracle_backward as bpins
from tests import test_oracle_quant as qpins
from tests import test_oracle_tiles as tpins
from tests import test_oracle_variants as vpins


def _prologue_rope_sign(x, gamma, grid, split, theta, eps):
    y = np.asarray(x, np.float64)
    H, D = y.shape[2], y.shape[3]
    y = y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps) * np.asarray(gamma).reshape(H, D)
    phi = so.rope_angles(grid, split, theta)
    c, s = np.cos(phi)[None, :, None, :], np.sin(phi)[None, :, None, :]
    out = np.empty_like(y)
    out[..., 0::2] = y[..., 0::2] * c + y[..., 1::2] * s        # rotates the other way
    out[..., 1::2] = -y[..., 0::2] * s + y[..., 1::2] * c
    return out


def _angles_axis_reversed(grid, split, theta):
    T, Hg, Wg = grid
    n = np.arange(T * Hg * Wg)
    pos = (n % Wg, (n // Wg) % Hg, n // (Hg * Wg))               # x, y, t instead of t, y, x
    cols = []
    for axis in range(3):
        for i in range(split[axis] // 2):
            cols.append(pos[axis] * theta ** (-2.0 * i / split[axis]))
    return np.stack(cols, axis=1)


def _prologue_eps_outside(x, gamma, grid, split, theta, eps):
    y = np.asarray(x, np.float64)
    H, D = y.shape[2], y.shape[3]
    y = y / (np.sqrt(np.mean(y * y, axis=-1, keepdims=True)) + eps) * np.asarray(gamma).reshape(H, D)
    phi = so.rope_angles(grid, split, theta)
    c, s = np.cos(phi)[None, :, None, :], np.sin(phi)[None, :, None, :]
    out = np.empty_like(y)
    out[..., 0::2] = y[..., 0::2] * c - y[..., 1::2] * s
    out[..., 1::2] = y[..., 0::2] * s + y[..., 1::2] * c
    return out


def _pool_full_block_divisor(x, block):
    x = np.asarray(x, np.float64)
    B, N, H, D = x.shape
    nb = -(-N // block)
    out = np.empty((B, H, nb, D))
    for i in range(nb):
        out[:, :, i, :] = x[:, i * block:(i + 1) * block].sum(axis=1) / block
    return out



def _topk_ties_high(scores, k):
    s = np.asarray(scores, np.float64)
    n = s.shape[-1]
    rev = s[..., ::-1]
    order = np.argsort(-rev, axis=-1, kind="stable")[..., :k]
    return np.sort(n - 1 - order, axis=-1).astype(np.int32)


def _attention_rows_no_scale(q, k, v, idx, block, scale, b, h, i, count=None):
    return so.__dict__["_orig_rows"](q, k, v, idx, block, 1.0, b, h, i, count)


def _attention_rows_lse_no_max(q, k, v, idx, block, scale, b, h, i, count=None):
    o, lse = so.__dict__["_orig_rows"](q, k, v, idx, block, scale, b, h, i, count)
    members = so._members(q.shape[1], block)
    rows = members[i]
    cols = np.concatenate([members[j] for j in np.asarray(idx[b, h, i])[:count]])
    logits = scale * (np.asarray(q[b, rows, h], np.float64) @ np.asarray(k[b, cols, h], np.float64).T)
    mx = logits.max(axis=1)
    return o, lse - mx


def _variant_diagonal_dropped(scores, topk, **kw):
    return so.__dict__["_orig_variant"](scores, topk, **{**kw, "diagonal": False})


def _variant_scale_ignored(scores, topk, **kw):
    return so.__dict__["_orig_variant"](scores, topk, **{**kw, "scale": 1.0})


def _variant_head_k_ignored(scores, topk, **kw):
    return so.__dict__["_orig_variant"](scores, topk, **{**kw, "head_k": None})


def _tiles_rows_columns_swapped(grid, tile):
    return so.__dict__["_orig_tiles"](grid, (tile[0], tile[2], tile[1]))


def _e4m3_no_subnormals(x):
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, fe = np.frexp(a)
    step = np.exp2(fe.astype(np.float64) - 4.0)         # normal spacing all the way down
    return np.copysign(np.minimum(np.rint(a / step) * step, 448.0), x)


def _quantize_levels_128(x, kind):
    codes, s = oracle.quant_oracle.__dict__["_orig_quant"](x, kind)
    return codes, (s * np.float32(127.0) / np.float32(128.0)).astype(np.float32)


def _backward_softmax_jacobian_dropped(q, k, v, idx, do, block, scale=None, counts=None):
    # dS = P * dP, without subtracting the row's P . dP: a plausible slip in the softmax gradient
    q, k, v, do = (np.asarray(x, np.float64) for x in (q, k, v, do))
    B, N, H, D = q.shape
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    members = so._members(N, block)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            for i, rows in enumerate(members):
                kept = np.asarray(idx[b, h, i])[: None if counts is None else int(counts[b, h, i])]
                cols = np.concatenate([members[j] for j in kept])
                s_ = scale * (q[b, rows, h] @ k[b, cols, h].T)
                p_ = np.exp(s_ - s_.max(axis=1, keepdims=True))
                p_ /= p_.sum(axis=1, keepdims=True)
                ds = p_ * (do[b, rows, h] @ v[b, cols, h].T)
                dq[b, rows, h] += scale * ds @ k[b, cols, h]
                np.add.at(dk[:, :, h], (b, cols), scale * ds.T @ q[b, rows, h])
                np.add.at(dv[:, :, h], (b, cols), p_.T @ do[b, rows, h])
    return dq, dk, dv


MUTATIONS = [
    ("qk_prologue", _prologue_rope_sign, [pins.test_prologue_hand_case]),
    ("rope_angles", _angles_axis_reversed, [pins.test_prologue_hand_case]),
    ("qk_prologue", _prologue_eps_outside, [pins.test_prologue_hand_case, pins.test_prologue_gamma_indexing_and_eps]),
    ("block_pool", _pool_full_block_divisor, [pins.test_pool_hand_case]),
    ("topk_blocks", _topk_ties_high, [pins.test_topk_brute_force_with_ties]),
    ("sparse_attention_rows", _attention_rows_no_scale, [pins.test_attention_all_blocks_equals_dense_library_attention]),
    ("sparse_attention_rows", _attention_rows_lse_no_max, [pins.test_attention_all_blocks_equals_dense_library_attention,
                                                           pins.test_attention_hand_cases]),
    ("select_variant", _variant_diagonal_dropped, [lambda: vpins.test_forced_diagonal_brute_force(2)]),
    ("select_variant", _variant_scale_ignored, [lambda: vpins.test_top_p_count_is_smallest_subset_reaching_p(0.6)]),
    ("select_variant", _variant_head_k_ignored, [vpins.test_per_head_k]),
    ("tiled_blocks", _tiles_rows_columns_swapped, [tpins.test_tiled_blocks_hand_case]),
    ("e4m3_round", _e4m3_no_subnormals, [qpins.test_e4m3_round_matches_torch]),
    ("quantize_rows", _quantize_levels_128, [qpins.test_scales_and_dequantize_hand_case]),
    ("sparse_attention_backward", _backward_softmax_jacobian_dropped,
     [lambda: bpins.test_backward_matches_autograd(False)]),
]


@pytest.mark.parametrize("name,bad,tests", MUTATIONS, ids=[m[1].__name__ for m in MUTATIONS])
def test_pins_catch_planted_mistake(monkeypatch, name, bad, tests):
    monkeypatch.setitem(so.__dict__, "_orig_rows", so.sparse_attention_rows)
    monkeypatch.setitem(so.__dict__, "_orig_variant", so.select_variant)
    monkeypatch.setitem(so.__dict__, "_orig_tiles", so.tiled_blocks)
    monkeypatch.setitem(oracle.quant_oracle.__dict__, "_orig_quant", oracle.quant_oracle.quantize_rows)
    monkeypatch.setattr(so, name, bad, raising=False)
    monkeypatch.setattr(oracle, name, bad)
    for t in tests:
        with pytest.raises(AssertionError):
            t()


def test_scores_transposition_is_caught(monkeypatch):
    # A transposed score matrix (s_ji for s_ij) must fail the dense-block closed form.
    bad = lambda qbar, kbar: np.swapaxes(so.__dict__["_orig_scores"](qbar, kbar), -1, -2)  # noqa: E731
    monkeypatch.setitem(so.__dict__, "_orig_scores", so.block_scores)
    monkeypatch.setattr(so, "block_scores", bad)
    monkeypatch.setattr(oracle, "block_scores", bad)
    with pytest.raises(AssertionError):
        pins.test_scores_equal_mean_of_dense_logit_blocks()
