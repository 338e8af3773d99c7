"""Sequence-parallel Sol-Attn: G ranks hold token shards; the attention runs on head shards.

Multi-GPU runs of the Sol-H3 runtime move Q, K and V between GPUs as INT8 and
the attention output as FP8, about half the inter-GPU bytes of bf16
(ai-feiten.nl, "Videomodel MiniMax-H3 rendert sneller dan afspelen", section
"Waar de snelheidswinst vandaan komt").  Per rank r of G:

    q_raw, k_raw, v   [B, N/G, H, D] bf16   tokens r N/G .. (r+1) N/G - 1, all heads
      -> sol_quant_pack (INT8, split heads)       one slice per destination rank
      -> all-to-all                               slice g of every rank lands on rank g
      -> sol_dequant_unpack                       [B, N, H/G, D]: all tokens, heads r H/G ..
      -> sol_qk_prologue_pool -> sol_block_select_pooled -> sol_sparse_attn_fwd
      -> sol_quant_pack (e4m3, split tokens) -> all-to-all -> sol_dequant_unpack
    o                 [B, N/G, H, D] bf16   (and lse [B, H/G, N] of the local heads)

Every scale belongs to one (token, head) row, so the values that reach the
attention do not depend on G.  The exchange itself goes through a Transport:
CollectiveTransport (torch.distributed all_to_all_single: NCCL over NVLink on
GPUs), HostStagedTransport (the same collective on host copies, for gloo) or
LocalTransport (G = 1).  Each exchange buffer is laid out
[G][...] so that slice g is exactly what rank g receives (ExchangePlan).
"""
from __future__ import annotations

import dataclasses

import torch

from . import (SOL_CODE_E4M3, SOL_CODE_INT8, SOL_SPLIT_HEADS, SOL_SPLIT_TOKENS, sol_block_select_pooled,
               sol_dequant_unpack, sol_qk_prologue_pool, sol_quant_pack, sol_sparse_attn_fwd)

__all__ = ["ExchangePlan", "Transport", "CollectiveTransport", "HostStagedTransport", "LocalTransport",
           "SeqParallelAttention"]


@dataclasses.dataclass(frozen=True)
class ExchangePlan:
    """Sizes and offsets of the exchange buffers of one rank.

    rows: (token, head) rows of one tensor that one rank sends to one
    destination, B * (N/G) * (H/G).  The Q/K/V buffer holds, per destination g,
    Q then K then V (3 * rows rows); the O buffer holds rows rows per
    destination.  Codes are D bytes per row, scales 4 bytes per row.
    """
    G: int
    B: int
    N: int
    H: int
    D: int

    def __post_init__(self):
        if self.G < 1 or self.N % self.G or self.H % self.G:
            raise ValueError(f"N={self.N} and H={self.H} must be multiples of G={self.G}")

    @property
    def n_local(self) -> int:
        return self.N // self.G

    @property
    def h_local(self) -> int:
        return self.H // self.G

    @property
    def rows(self) -> int:
        return self.B * self.n_local * self.h_local

    @property
    def qkv_stride_rows(self) -> int:      # rows between destination slices of the Q/K/V buffer
        return 3 * self.rows

    def qkv_offset_rows(self, t: int) -> int:   # tensor t (0 q, 1 k, 2 v) inside each slice
        return t * self.rows

    @property
    def qkv_code_bytes(self) -> int:
        return self.G * self.qkv_stride_rows * self.D

    @property
    def qkv_scale_count(self) -> int:
        return self.G * self.qkv_stride_rows

    @property
    def o_code_bytes(self) -> int:
        return self.G * self.rows * self.D

    @property
    def o_scale_count(self) -> int:
        return self.G * self.rows

    def wire_bytes(self) -> int:
        """Bytes one rank sends to other ranks per step (its own slice stays local)."""
        per_dest = (3 + 1) * self.rows * (self.D + 4)
        return (self.G - 1) * per_dest

    def bf16_wire_bytes(self) -> int:
        return (self.G - 1) * (3 + 1) * self.rows * self.D * 2


class Transport:
    """Moves slice g of `send` (dim 0 split into G equal parts) to rank g, into slice r of its `recv`."""

    def all_to_all(self, recv: torch.Tensor, send: torch.Tensor) -> None:
        raise NotImplementedError


class CollectiveTransport(Transport):
    """torch.distributed all_to_all_single over a process group (NCCL on GPUs; gloo on CPU)."""

    def __init__(self, group=None):
        self.group = group

    def all_to_all(self, recv, send):
        torch.distributed.all_to_all_single(recv, send, group=self.group)


class HostStagedTransport(Transport):
    """all_to_all through host memory: a device -> host copy of `send`,
    torch.distributed all_to_all_single on the host tensors, a host -> device
    copy into `recv`.  For process groups whose backend moves only host memory
    (gloo), e.g. ranks that share one GPU; no peer memory is touched."""

    def __init__(self, group=None):
        self.group = group

    def all_to_all(self, recv, send):
        host_send = send.cpu()
        host_recv = torch.empty_like(host_send)
        torch.distributed.all_to_all_single(host_recv, host_send, group=self.group)
        recv.copy_(host_recv)


class LocalTransport(Transport):
    """G = 1: the only slice stays on this rank."""

    def all_to_all(self, recv, send):
        recv.copy_(send)


class SeqParallelAttention:
    """One rank's part of sequence-parallel Sol-Attn (module docstring).

    gamma_q, gamma_k: the full fp32 [H * D] gains (this rank uses its heads' slice).
    """

    def __init__(self, rank, world, B, N, H, D, grid, block, topk, gamma_q, gamma_k, rope_split=None,
                 rope_theta=10000.0, eps=1e-6, softmax_scale=0.0, device=None):
        self.plan = ExchangePlan(world, B, N, H, D)
        if not 0 <= rank < world:
            raise ValueError("rank out of range")
        if int(grid[0]) * int(grid[1]) * int(grid[2]) != N:
            raise ValueError("grid does not match N")
        self.rank = rank
        self.grid, self.block, self.topk = tuple(int(g) for g in grid), int(block), int(topk)
        self.rope_split, self.rope_theta, self.eps, self.softmax_scale = rope_split, rope_theta, eps, softmax_scale
        dev = torch.device(device) if device is not None else gamma_q.device
        p = self.plan
        h0 = rank * p.h_local
        self.gamma_q = gamma_q[h0 * D:(h0 + p.h_local) * D].contiguous()
        self.gamma_k = gamma_k[h0 * D:(h0 + p.h_local) * D].contiguous()
        u8, f32 = torch.uint8, torch.float32
        self.send_qkv = torch.empty(p.qkv_code_bytes, dtype=u8, device=dev)
        self.recv_qkv = torch.empty_like(self.send_qkv)
        self.send_qkv_s = torch.empty(p.qkv_scale_count, dtype=f32, device=dev)
        self.recv_qkv_s = torch.empty_like(self.send_qkv_s)
        self.send_o = torch.empty(p.o_code_bytes, dtype=u8, device=dev)
        self.recv_o = torch.empty_like(self.send_o)
        self.send_o_s = torch.empty(p.o_scale_count, dtype=f32, device=dev)
        self.recv_o_s = torch.empty_like(self.send_o_s)
        heads = (B, N, p.h_local, D)
        self.q_h = torch.empty(heads, dtype=torch.bfloat16, device=dev)
        self.k_h = torch.empty_like(self.q_h)
        self.v_h = torch.empty_like(self.q_h)
        self.lse = None

    # -- stages --------------------------------------------------------------
    def stage_pack(self, q_raw, k_raw, v, stream=None):
        """Quantise this rank's token shard [B, N/G, H, D] into the Q/K/V send buffer."""
        p = self.plan
        for t, x in enumerate((q_raw, k_raw, v)):
            if tuple(x.shape) != (p.B, p.n_local, p.H, p.D):
                raise ValueError(f"expected a token shard of shape {(p.B, p.n_local, p.H, p.D)}")
            r0 = p.qkv_offset_rows(t)
            sol_quant_pack(x, p.G, SOL_SPLIT_HEADS, SOL_CODE_INT8, self.send_qkv[r0 * p.D:], self.send_qkv_s[r0:],
                           g_stride_rows=p.qkv_stride_rows, stream=stream)

    def stage_compute(self, stream=None):
        """Dequantise the received head shard, run the path, quantise O into the O send buffer.
        Returns lse [B, H/G, N] of this rank's heads."""
        p = self.plan
        for t, out in enumerate((self.q_h, self.k_h, self.v_h)):
            r0 = p.qkv_offset_rows(t)
            sol_dequant_unpack(self.recv_qkv[r0 * p.D:], self.recv_qkv_s[r0:], p.B, p.n_local, p.h_local, p.D, p.G,
                               SOL_SPLIT_HEADS, SOL_CODE_INT8, out, g_stride_rows=p.qkv_stride_rows, stream=stream)
        q, k, qbar, kbar = sol_qk_prologue_pool(self.q_h, self.k_h, self.gamma_q, self.gamma_k, self.grid, self.block,
                                                self.rope_split, self.rope_theta, self.eps, stream=stream)
        idx = sol_block_select_pooled(qbar, kbar, self.grid, self.block, self.topk, stream=stream)
        o_h, lse = sol_sparse_attn_fwd(q, k, self.v_h, idx, self.grid, self.block, self.softmax_scale, stream=stream)
        sol_quant_pack(o_h, p.G, SOL_SPLIT_TOKENS, SOL_CODE_E4M3, self.send_o, self.send_o_s, stream=stream)
        self.lse = lse
        return lse

    def stage_unpack(self, out=None, stream=None):
        """O of this rank's token shard, [B, N/G, H, D] bf16."""
        p = self.plan
        if out is None:
            out = torch.empty((p.B, p.n_local, p.H, p.D), dtype=torch.bfloat16, device=self.send_o.device)
        sol_dequant_unpack(self.recv_o, self.recv_o_s, p.B, p.n_local, p.h_local, p.D, p.G, SOL_SPLIT_TOKENS,
                           SOL_CODE_E4M3, out, stream=stream)
        return out

    def exchange_qkv(self, transport: Transport):
        transport.all_to_all(self.recv_qkv, self.send_qkv)
        transport.all_to_all(self.recv_qkv_s, self.send_qkv_s)

    def exchange_o(self, transport: Transport):
        transport.all_to_all(self.recv_o, self.send_o)
        transport.all_to_all(self.recv_o_s, self.send_o_s)

    def forward(self, q_raw, k_raw, v, transport: Transport, out=None):
        """The whole step on this rank: returns (o [B, N/G, H, D], lse [B, H/G, N])."""
        self.stage_pack(q_raw, k_raw, v)
        self.exchange_qkv(transport)
        lse = self.stage_compute()
        self.exchange_o(transport)
        return self.stage_unpack(out), lse
