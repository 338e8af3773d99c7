"""Shared pieces of the GPU parity tests: cached workload inputs, the oracle
run on them, and the comparison rules.

Tolerances (written here once, used by every GPU test):
  * prologue, bf16 out: within 1 bf16 ulp of the fp64 result rounded to bf16
    (the kernel computes in fp32, so only values sitting next to a rounding
    boundary may land on the other side), except values that the rotation
    cancels to near zero, which must be within the fp32 evaluation error
    (2^-20 of the row's largest magnitude); fp32 out: 1e-5 relative to max|ref|.
  * selection: ids bit-exact, except in rows where the oracle's k-th and
    (k+1)-th scores differ by less than 1e-4 relative; there the two id sets
    may differ only among ids whose oracle score lies inside that band.
  * attention, bf16: max |O_gpu - O_oracle| <= 2e-2, |LSE_gpu - LSE_oracle| <= 1e-2;
    fp32: both within 1e-5 relative to max |O_oracle| / max |LSE_oracle|.
"""
from __future__ import annotations

import functools
import math

import numpy as np
import torch

import oracle as orc
from workloads import WORKLOADS, make_inputs

O_TOL_BF16 = 2e-2
LSE_TOL_BF16 = 1e-2
REL_TOL_F32 = 1e-5
NEAR_TIE_REL = 1e-4


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


@functools.lru_cache(maxsize=2)
def cpu_inputs(config_id: int, seed: int = 0):
    return make_inputs(WORKLOADS[config_id], seed=seed)


def bf16_ulps(gpu: np.ndarray, ref64: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place between gpu (bf16 values) and
    the fp64 reference rounded to bf16."""
    def ordered(a):
        bits = (torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
                .view(torch.int16).numpy().astype(np.int32))
        return np.where(bits < 0, -(bits & 0x7FFF), bits)
    return np.abs(ordered(gpu) - ordered(orc.bf16_round(ref64)))


def check_bf16_prologue(gpu: np.ndarray, ref64: np.ndarray) -> int:
    """bf16 prologue outputs: each value within 1 bf16 ulp of the fp64 result
    rounded, or - where the rotation cancels to a value near zero, so that bf16
    ulps become tiny - within the fp32 evaluation error, 2^-20 of the largest
    magnitude in its row.  Returns the number of elements that needed the
    second clause."""
    ulps = bf16_ulps(gpu, ref64)
    floor = 2.0 ** -20 * np.abs(ref64).max(axis=-1, keepdims=True)
    near_zero_ok = np.abs(gpu.astype(np.float64) - ref64) <= floor + 2.0 ** -9 * np.abs(ref64)
    bad = (ulps > 1) & ~near_zero_ok
    assert not bad.any(), f"{int(bad.sum())} prologue values off, first at {np.argwhere(bad)[0]}"
    return int(((ulps > 1) & near_zero_ok).sum())


def check_selection(idx_gpu: np.ndarray, scores_ref: np.ndarray, topk: int, rel=NEAR_TIE_REL):
    """Returns (n_rows, n_near_tie_rows, n_near_tie_rows_differing); asserts
    every other row is identical and differing near-tie rows only swap ids
    inside the tie band."""
    idx_ref = orc.topk_blocks(scores_ref, topk)
    near = orc.near_tie_rows(scores_ref, topk, rel)
    same = np.all(idx_gpu == idx_ref, axis=-1)
    bad = ~same & ~near
    assert not bad.any(), f"{int(bad.sum())} rows differ outside near ties, first at {np.argwhere(bad)[0]}"
    for pos in np.argwhere(~same):
        s = scores_ref[tuple(pos)]
        kth = -np.sort(-s)[topk - 1]
        band = rel * max(abs(kth), 1e-300) * 2
        sym = set(idx_gpu[tuple(pos)]) ^ set(idx_ref[tuple(pos)])
        assert all(abs(s[j] - kth) <= band for j in sym), (pos, sym)
    assert np.all(np.diff(idx_gpu, axis=-1) > 0), "ids must be ascending and distinct"
    return same.size, int(near.sum()), int((~same).sum())


def sample_units(B, H, nb, per_head=16, seed=0):
    """(b, h, query block) units: for every (b, h) the first and last blocks and
    per_head-2 random ones."""
    rng = np.random.default_rng([seed, 7])
    units = []
    for b in range(B):
        for h in range(H):
            blocks = {0, nb - 1}
            while len(blocks) < min(per_head, nb):
                blocks.add(int(rng.integers(0, nb)))
            units += [(b, h, i) for i in sorted(blocks)]
    return units


def check_attention(o_gpu, lse_gpu, q, k, v, idx, block, units, fp32: bool):
    """Compares GPU O / LSE with the oracle on the listed units; returns the max errors."""
    o_ref, lse_ref = orc.sparse_attention(q, k, v, idx, block, units=units)
    N = q.shape[1]
    rows = []
    for (b, h, i) in units:
        r = np.arange(i * block, min(N, (i + 1) * block))
        rows.append((b, h, r))
    err_o = max(np.abs(np64(o_gpu[b, r, h]) - o_ref[b, r, h]).max() for (b, h, r) in rows)
    err_l = max(np.abs(np64(lse_gpu[b, h, r]) - lse_ref[b, h, r]).max() for (b, h, r) in rows)
    if fp32:
        o_scale = max(np.abs(o_ref[b, r, h]).max() for (b, h, r) in rows)
        l_scale = max(np.abs(lse_ref[b, h, r]).max() for (b, h, r) in rows)
        assert err_o <= REL_TOL_F32 * o_scale, (err_o, o_scale)
        assert err_l <= REL_TOL_F32 * l_scale, (err_l, l_scale)
    else:
        assert err_o <= O_TOL_BF16, err_o
        assert err_l <= LSE_TOL_BF16, err_l
    assert np.isfinite(err_o) and np.isfinite(err_l)
    return err_o, err_l


def scale_of(D):
    return 1.0 / math.sqrt(D)
