"""The fused Sol-Attn chain captured once as a CUDA graph and replayed.

One step of the chain is three launches (prologue with block means, selection
from the means, attention).  For short clips or few heads the launch overhead
is a visible share of the step, so ChainGraph runs the three libsol calls once
outside capture (which sets the kernels' one-time attributes), captures them
into a CUDA graph over static device buffers, and replays that graph: one
graph launch per step.  Inputs go into the static buffers (`q_raw`, `k_raw`,
`v`; copied by __call__, or written there directly by the caller); O and LSE
stay in `o` and `lse`, overwritten by each replay.

Only orchestration lives here; every computation is a libsol call, captured as
it is issued.
"""
from __future__ import annotations

import torch

from . import sol_block_select_pooled, sol_qk_prologue_pool, sol_sparse_attn_fwd


class ChainGraph:
    def __init__(self, B, N, H, D, grid, block, topk, gamma_q, gamma_k, dtype=torch.bfloat16, rope_split=None,
                 rope_theta=10000.0, eps=1e-6, softmax_scale=0.0, device=None):
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        if gamma_q.device != dev or gamma_k.device != dev:
            raise ValueError("gamma_q and gamma_k must live on the graph's device")
        self.dev, self.grid, self.block, self.topk = dev, tuple(grid), int(block), int(topk)
        self.rope_split, self.rope_theta, self.eps, self.scale = rope_split, rope_theta, eps, softmax_scale
        self.gamma_q, self.gamma_k = gamma_q, gamma_k
        nb = -(-N // block)
        act = (B, N, H, D)
        mk = lambda shape, dt: torch.zeros(shape, dtype=dt, device=dev)  # noqa: E731
        self.q_raw, self.k_raw, self.v = mk(act, dtype), mk(act, dtype), mk(act, dtype)
        self.q, self.k = mk(act, dtype), mk(act, dtype)
        self.qbar, self.kbar = mk((B, H, nb, D), torch.float32), mk((B, H, nb, D), torch.float32)
        self.idx = mk((B, H, nb, topk), torch.int32)
        self.o, self.lse = mk(act, dtype), mk((B, H, N), torch.float32)
        self.graph = None

    def _step(self):
        sol_qk_prologue_pool(self.q_raw, self.k_raw, self.gamma_q, self.gamma_k, self.grid, self.block,
                             self.rope_split, self.rope_theta, self.eps, q_out=self.q, k_out=self.k,
                             qbar_out=self.qbar, kbar_out=self.kbar)
        sol_block_select_pooled(self.qbar, self.kbar, self.grid, self.block, self.topk, idx_out=self.idx)
        sol_sparse_attn_fwd(self.q, self.k, self.v, self.idx, self.grid, self.block, self.scale, o=self.o,
                            lse=self.lse)

    def capture(self):
        """Run the step once on a side stream, then capture it.  Returns self."""
        cur = torch.cuda.current_stream(self.dev)
        side = torch.cuda.Stream(self.dev)
        side.wait_stream(cur)
        with torch.cuda.stream(side):
            self._step()
        cur.wait_stream(side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            self._step()
        self.graph = g
        return self

    def replay(self):
        """One step over the current contents of the static input buffers."""
        if self.graph is None:
            raise RuntimeError("capture() first")
        self.graph.replay()

    def __call__(self, q_raw, k_raw, v):
        """Copy the inputs into the static buffers, replay; returns (o, lse), the static outputs."""
        for dst, src in ((self.q_raw, q_raw), (self.k_raw, k_raw), (self.v, v)):
            if src.shape != dst.shape or src.dtype != dst.dtype:
                raise ValueError(f"expected {tuple(dst.shape)} {dst.dtype}, got {tuple(src.shape)} {src.dtype}")
            dst.copy_(src, non_blocking=True)
        self.replay()
        return self.o, self.lse
