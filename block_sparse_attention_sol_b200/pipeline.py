"""A stream of clips through the Sol-Attn chain from and to host memory.

Each submitted clip is copied from pinned host memory to the device, runs the
fused chain (prologue with block means -> selection from the means ->
attention), and its O and LSE are copied back to pinned host memory.  Three CUDA
streams carry the three kinds of work: inputs in, kernels, outputs out.  Input
and output device buffers are double-buffered, so clip i + 1's inputs cross PCIe
while clip i computes and clip i - 1's outputs come back.  Events order each
buffer's reuse: a clip's inputs overwrite a device buffer only after the chain
that read it finished, and the chain writes an output buffer only after that
buffer's previous contents reached the host.  Steady-state time per clip is the
longest of the three lanes.

Only orchestration lives here (copies, streams, events); every computation is a
libsol call.
"""
from __future__ import annotations

import torch

from . import sol_block_select_pooled, sol_qk_prologue_pool, sol_sparse_attn_fwd


class HostChainPipeline:
    def __init__(self, B, N, H, D, grid, block, topk, gamma_q, gamma_k, dtype=torch.bfloat16, rope_split=None,
                 rope_theta=10000.0, eps=1e-6, softmax_scale=0.0, device=None):
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        if gamma_q.device != dev or gamma_k.device != dev:
            raise ValueError("gamma_q and gamma_k must live on the pipeline's device")
        self.dev, self.grid, self.block, self.topk = dev, tuple(grid), int(block), int(topk)
        self.rope_split, self.rope_theta, self.eps, self.scale = rope_split, rope_theta, eps, softmax_scale
        self.gamma_q, self.gamma_k = gamma_q, gamma_k
        nb = -(-N // block)
        act = (B, N, H, D)
        mk = lambda shape, dt: torch.empty(shape, dtype=dt, device=dev)  # noqa: E731
        self.inp = [{n: mk(act, dtype) for n in ("q", "k", "v")} for _ in range(2)]
        self.out = [{"o": mk(act, dtype), "lse": mk((B, H, N), torch.float32)} for _ in range(2)]
        self.q, self.k = mk(act, dtype), mk(act, dtype)
        self.qbar, self.kbar = mk((B, H, nb, D), torch.float32), mk((B, H, nb, D), torch.float32)
        self.idx = mk((B, H, nb, topk), torch.int32)
        self.s_in = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.in_ready = [torch.cuda.Event() for _ in range(2)]
        self.in_free = [None, None]      # chain that last read input buffer b
        self.out_ready = [torch.cuda.Event() for _ in range(2)]
        self.out_free = [None, None]     # copy-out that last read output buffer b
        self.count = 0

    def submit(self, q_host, k_host, v_host, o_host, lse_host):
        """Queue one clip.  The host tensors must be pinned and stay untouched
        until synchronize() (or a later submit's completion) shows it done."""
        for t in (q_host, k_host, v_host, o_host, lse_host):
            if t.device.type != "cpu" or not t.is_pinned():
                raise ValueError("host tensors must be pinned CPU tensors")
        b = self.count % 2
        self.count += 1
        inp, out = self.inp[b], self.out[b]
        with torch.cuda.stream(self.s_in):
            if self.in_free[b] is not None:
                self.s_in.wait_event(self.in_free[b])
            inp["q"].copy_(q_host, non_blocking=True)
            inp["k"].copy_(k_host, non_blocking=True)
            inp["v"].copy_(v_host, non_blocking=True)
            self.in_ready[b].record(self.s_in)
        with torch.cuda.stream(self.s_comp):
            self.s_comp.wait_event(self.in_ready[b])
            if self.out_free[b] is not None:
                self.s_comp.wait_event(self.out_free[b])
            s = self.s_comp
            sol_qk_prologue_pool(inp["q"], inp["k"], self.gamma_q, self.gamma_k, self.grid, self.block,
                                 self.rope_split, self.rope_theta, self.eps, q_out=self.q, k_out=self.k,
                                 qbar_out=self.qbar, kbar_out=self.kbar, stream=s)
            sol_block_select_pooled(self.qbar, self.kbar, self.grid, self.block, self.topk, idx_out=self.idx,
                                    stream=s)
            sol_sparse_attn_fwd(self.q, self.k, inp["v"], self.idx, self.grid, self.block, self.scale,
                                o=out["o"], lse=out["lse"], stream=s)
            done = torch.cuda.Event()
            done.record(s)
            self.in_free[b] = done
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(done)
            o_host.copy_(out["o"], non_blocking=True)
            lse_host.copy_(out["lse"], non_blocking=True)
            freed = torch.cuda.Event()
            freed.record(self.s_out)
            self.out_free[b] = freed

    def synchronize(self):
        for s in (self.s_in, self.s_comp, self.s_out):
            s.synchronize()
