"""Seeded synthetic video-token inputs for the Sol-Attn hot path.

This module holds the workload table and the input generators, and nothing of
the method's arithmetic (no normalisation, rotation, pooling, scoring,
selection or attention).  Both the CPU oracle (``oracle/``) and the CUDA path
consume the tensors it returns, so the two always see identical stored inputs.

Workloads: the shapes are latent video grids (t, h, w) of MiniMax-H3 clips,
flattened in raster order n = (t*Hg + y)*Wg + x.  The 896x512 draft shape and
the 1344x768 / 1920x1088 refinement shapes come from the two-stage H3 pipeline
(ainews.surl.tw, "NVIDIA Adds Two-Stage Generation for MiniMax H3"), the /16
latent grid from the H3 latent layout (Sol-H3-VAE model card, "Usage").

Generator recipe (per tensor q, k, v, drawn independently):
    x[b, n, h, c] = z + sum_{j<4} a_j * sin(w_j . (t, y, x))
    z ~ N(0, 1) i.i.d.;  a_j ~ N(0, variance 0.5);  w_j ~ U(0, 0.5)^3,
    a_j and w_j drawn per (batch, head, channel).
RMSNorm gains gamma_q, gamma_k ~ U(0.8, 1.2), one per (head, channel).
RNG: numpy PCG64 seeded with [seed, config_id, tensor_id], tensor_id
0..4 = q, k, v, gamma_q, gamma_k.  Values are produced in fp32 and, for bf16
workloads, rounded once (round to nearest even) to bf16.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "make_inputs", "make_field", "rope_split_for", "random_index_lists"]


def rope_split_for(D: int) -> tuple[int, int, int]:
    """Channel split of the 3D rotary embedding over (t, h, w).

    For D=128 this is the 44/42/42 split of the workloads; the same rule
    (h and w get 2*floor(D/6) channels each, t the rest) gives 24/20/20 at D=64.
    """
    dh = 2 * (D // 6)
    return (D - 2 * dh, dh, dh)


@dataclasses.dataclass(frozen=True)
class Workload:
    config_id: int
    name: str
    dtype: str            # "f32" or "bf16"
    B: int
    H: int
    D: int
    grid: tuple[int, int, int]   # (T, Hg, Wg) latent grid
    block: int
    topk: tuple[int, ...]
    rope_theta: float = 10000.0
    eps: float = 1e-6

    @property
    def N(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def nb(self) -> int:
        return -(-self.N // self.block)

    @property
    def rope_split(self) -> tuple[int, int, int]:
        return rope_split_for(self.D)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def selected_flops(self, topk: int | None = None) -> int:
        """Selected attention FLOPs: 4 * n_q * n_k * D summed over selected block pairs.

        Every query block keeps exactly ``topk`` key blocks; a pair that involves the
        ragged last block counts only its valid tokens.  With the selection unknown,
        this assumes every selected key block is full (upper bound when N % block != 0).
        """
        k = self.topk[0] if topk is None else topk
        total = 0
        full = self.N // self.block
        tail = self.N - full * self.block
        for nq in [self.block] * full + ([tail] if tail else []):
            total += 4 * nq * k * self.block * self.D
        return total * self.B * self.H


WORKLOADS: dict[int, Workload] = {
    0: Workload(0, "tiny fp32 correctness case, 4x16x16 grid", "f32", 1, 2, 64, (4, 16, 16), 64, (4, 16)),
    1: Workload(1, "896x512 draft-stage shape, 16x32x56 grid", "bf16", 1, 32, 128, (16, 32, 56), 128, (45,)),
    2: Workload(2, "1344x768 5 s clip shape, 16x48x84 grid", "bf16", 1, 32, 128, (16, 48, 84), 128, (76,)),
    3: Workload(3, "1344x768 10 s clip shape, 31x48x84 grid (ragged last block)", "bf16", 1, 32, 128, (31, 48, 84), 128, (98,)),
    4: Workload(4, "1920x1088 refinement-stage chain, 16x68x120 grid", "bf16", 1, 32, 128, (16, 68, 120), 128, (102,)),
}

_TENSOR_ID = {"q": 0, "k": 1, "v": 2, "gamma_q": 3, "gamma_k": 4}
_J = 4  # number of sinusoidal terms in the smooth field


def make_field(grid, a: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Smooth field sum_j a_j sin(w_j . (t, y, x)) over the raster-ordered grid.

    a: [C, J], w: [C, J, 3] -> returns [N, C] float64.  Evaluated with the angle
    addition identity sin(u + v) = sin u cos v + cos u sin v, u = w_t t + w_y y,
    v = w_x x, which turns the sum over j into a small matrix product per channel.
    """
    T, Hg, Wg = grid
    t = np.arange(T, dtype=np.float64)
    y = np.arange(Hg, dtype=np.float64)
    x = np.arange(Wg, dtype=np.float64)
    # u[c, j, t, y] and v[c, j, x]
    u = w[:, :, 0, None, None] * t[None, None, :, None] + w[:, :, 1, None, None] * y[None, None, None, :]
    u = u.reshape(w.shape[0], w.shape[1], T * Hg)
    v = w[:, :, 2, None] * x[None, None, :]
    left = np.concatenate([a[:, :, None] * np.sin(u), a[:, :, None] * np.cos(u)], axis=1)   # [C, 2J, T*Hg]
    right = np.concatenate([np.cos(v), np.sin(v)], axis=1)                                    # [C, 2J, Wg]
    f = np.matmul(left.transpose(0, 2, 1), right)                                              # [C, T*Hg, Wg]
    return f.reshape(w.shape[0], T * Hg * Wg).T


def _activation(wl: Workload, seed: int, name: str) -> np.ndarray:
    rng = np.random.default_rng([seed, wl.config_id, _TENSOR_ID[name]])
    B, N, H, D = wl.B, wl.N, wl.H, wl.D
    a = rng.normal(0.0, math.sqrt(0.5), size=(B, H * D, _J))
    w = rng.uniform(0.0, 0.5, size=(B, H * D, _J, 3))
    out = rng.standard_normal(size=(B, N, H * D), dtype=np.float32)
    hd_chunk = 512
    for b in range(B):
        for c0 in range(0, H * D, hd_chunk):
            c1 = min(H * D, c0 + hd_chunk)
            out[b, :, c0:c1] += make_field(wl.grid, a[b, c0:c1], w[b, c0:c1]).astype(np.float32)
    return out.reshape(B, N, H, D)


def make_inputs(wl: Workload | int, seed: int = 0, names=("q", "k", "v", "gamma_q", "gamma_k")) -> dict:
    """Returns CPU torch tensors: q, k, v as [B, N, H, D] in the workload dtype
    (these are the raw, pre-prologue activations), gamma_q / gamma_k as fp32 [H*D]."""
    if isinstance(wl, int):
        wl = WORKLOADS[wl]
    out = {}
    for name in names:
        if name.startswith("gamma"):
            rng = np.random.default_rng([seed, wl.config_id, _TENSOR_ID[name]])
            out[name] = torch.from_numpy(rng.uniform(0.8, 1.2, size=wl.H * wl.D).astype(np.float32))
        else:
            t = torch.from_numpy(_activation(wl, seed, name))
            out[name] = t.to(wl.torch_dtype) if wl.dtype == "bf16" else t
    return out


def random_index_lists(B: int, H: int, nb: int, k: int, seed: int) -> torch.Tensor:
    """Seeded random selections: k distinct ascending key-block ids per (b, h, query block).

    Used to drive the attention stage with selections that do not come from any
    scoring rule (any valid index list is a legal input)."""
    rng = np.random.default_rng([seed, 99])
    keys = rng.random(size=(B, H, nb, nb))
    idx = np.sort(np.argsort(keys, axis=-1)[..., :k], axis=-1).astype(np.int32)
    return torch.from_numpy(np.ascontiguousarray(idx))
