"""Shared pieces of the GPU parity tests: cached workload inputs, the oracle
run on them, and the comparison rules.

Tolerances (written here once, used by every GPU test):
  * prologue, bf16 out: the bf16 rounding of a value within the kernel's fp32
    error bound (2^-17 of the channel pair's magnitude) of the exact fp64
    result - exactly RN(y) unless y sits that close to a rounding midpoint;
    fp32 out: 1e-5 relative to max|ref|.
  * selection, same inputs on both sides: ids bit-exact, except in rows where
    the oracle's k-th and (k+1)-th scores differ by less than 1e-4 relative;
    there the two id sets may differ only among ids inside that band.
  * selection at the end of the chain (each side selects on its own prologue
    output): the band also covers the score change that the prologue values
    allowed to round the other way can cause (score_perturbation_bound).
  * attention, bf16: max |O_gpu - O_oracle| <= 2e-2, |LSE_gpu - LSE_oracle| <= 1e-2;
    fp32: both within 1e-5 relative to max |O_oracle| / max |LSE_oracle|.
"""
from __future__ import annotations

import functools
import hashlib
import json
import math
import os
import time

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


PROLOGUE_ERR = 2.0 ** -17


def prologue_err_bound(y64: np.ndarray) -> np.ndarray:
    """Largest |fp32 kernel result - exact result| the prologue's arithmetic can
    produce before the final rounding: 2^-17 of the channel pair's magnitude
    (the fp32 sum of squares, reciprocal square root, gains and rotation
    together stay below ~1.5e-6 of it; the cos/sin tables are rounded from
    double-precision angles)."""
    rho = np.sqrt(y64[..., 0::2] ** 2 + y64[..., 1::2] ** 2)
    return np.repeat(rho, 2, axis=-1) * PROLOGUE_ERR


def check_bf16_prologue(gpu: np.ndarray, ref64: np.ndarray) -> int:
    """bf16 prologue outputs: each value must be the bf16 rounding of some value
    within prologue_err_bound of the exact fp64 result, i.e. lie between
    RN(y - E) and RN(y + E).  Where the exact result is not within E of a bf16
    rounding midpoint this is exactly RN(y).  Returns how many values took the
    other neighbour."""
    E = prologue_err_bound(ref64)
    lo, hi = orc.bf16_round(ref64 - E), orc.bf16_round(ref64 + E)
    g = gpu.astype(np.float64)
    bad = (g < lo) | (g > hi)
    assert not bad.any(), f"{int(bad.sum())} prologue values off, first at {np.argwhere(bad)[0]}"
    return int((g != orc.bf16_round(ref64)).sum())


def prologue_flip_size(ref64: np.ndarray) -> np.ndarray:
    """Per value, how far the kernel's bf16 result may lie from RN(y): 0 unless
    y is within the error bound of a rounding midpoint, then one bf16 step."""
    E = prologue_err_bound(ref64)
    return orc.bf16_round(ref64 + E) - orc.bf16_round(ref64 - E)


def score_perturbation_bound(qbar, kbar, uq, uk) -> np.ndarray:
    """Bound on |s_gpu_input - s_oracle_input| [B,H,nb,nb] when each pooled
    channel of q (k) may move by at most uq (uk), the block means of the
    possible prologue flips: |dq|.|k| + |q|.|dk| + |dq|.|dk|."""
    aq, ak = np.abs(qbar), np.abs(kbar)
    T = lambda a: np.swapaxes(a, -1, -2)  # noqa: E731
    return uq @ T(ak) + aq @ T(uk) + uq @ T(uk)


def check_selection(idx_gpu: np.ndarray, scores_ref: np.ndarray, topk: int, rel=NEAR_TIE_REL, abs_band=None):
    """Returns (n_rows, n_near_tie_rows, n_near_tie_rows_differing); asserts
    every other row is identical and differing near-tie rows only swap ids
    inside the tie band.  A row is a near-tie row when the oracle's k-th and
    (k+1)-th scores differ by less than rel times the larger magnitude, or -
    when abs_band [.., rows] is given (inputs that may differ slightly, as in
    the end-to-end chain) - by less than abs_band."""
    idx_ref = orc.topk_blocks(scores_ref, topk)
    srt = -np.sort(-scores_ref, axis=-1)
    if topk < scores_ref.shape[-1]:
        a, b = srt[..., topk - 1], srt[..., topk]
        band = rel * np.maximum(np.abs(a), np.abs(b))
        if abs_band is not None:
            band = np.maximum(band, abs_band)
        near = np.abs(a - b) < band
    else:
        band = np.zeros(scores_ref.shape[:-1])
        near = np.zeros(scores_ref.shape[:-1], dtype=bool)
    same = np.all(idx_gpu == idx_ref, axis=-1)
    bad = ~same & ~near
    assert not bad.any(), f"{int(bad.sum())} rows differ outside near ties, first at {np.argwhere(bad)[0]}"
    for pos in np.argwhere(~same):
        pos = tuple(pos)
        s = scores_ref[pos]
        kth = srt[pos][topk - 1]
        sym = set(idx_gpu[pos]) ^ set(idx_ref[pos])
        assert all(abs(s[j] - kth) <= 2 * band[pos] for j in sym), (pos, sym)
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


# ---------------------------------------------------------------- parity record
# The GPU parity tests write what they measured (rows compared, near-tie rows,
# rows that differ, output errors) to tests/parity_record.json, one entry per
# (workload, path), stamped with a hash of the kernel sources they ran, so the
# counts the selection rule allows are reported and not only asserted.
RECORD_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "parity_record.json")
_ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def kernel_sources_sha256() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(_ROOT, "block_sparse_attention_sol_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + b"\0" + f.read())
    with open(os.path.join(_ROOT, "include", "sol.h"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def record_parity(key: str, **fields) -> None:
    rec = {}
    if os.path.exists(RECORD_PATH):
        with open(RECORD_PATH) as f:
            rec = json.load(f)
    rec.setdefault("about", "written by the -m gpu parity tests (tests/test_gpu_workloads.py): per workload and "
                            "path, the selection rows compared with the oracle, the near-tie rows among them (oracle "
                            "k-th and (k+1)-th scores closer than 1e-4 relative, or than the chain's prologue band), "
                            "the rows whose ids differ (allowed only among near-tie rows), and the attention errors")
    entry = {k: (float(v) if isinstance(v, (np.floating, float)) else int(v) if isinstance(v, (np.integer,)) else v)
             for k, v in fields.items()}
    entry["kernel_sources_sha256"] = kernel_sources_sha256()
    entry["when"] = time.strftime("%Y-%m-%dT%H:%M:%SZ", time.gmtime())
    try:
        entry["device"] = torch.cuda.get_device_name(0)
    except Exception:
        pass
    rec.setdefault("entries", {})[key] = entry
    rec["entries"] = dict(sorted(rec["entries"].items()))
    tmp = RECORD_PATH + ".tmp"
    with open(tmp, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    os.replace(tmp, RECORD_PATH)
