"""GPU parity of the quantised exchange kernels and of sequence-parallel Sol-Attn.

  * sol_quant_pack: codes and scales bit for bit equal to the oracle's
    quantisation (both decide each code in fp32), placed where the documented
    layout puts them, for INT8 / e4m3, split heads / split tokens, several G.
  * sol_dequant_unpack: bit for bit equal to the oracle's dequantisation of the
    same (seeded) codes, concatenated along tokens or heads.
  * SeqParallelAttention run as G = 2 and 4 ranks on one GPU (each stage runs
    for every rank in turn and the exchange is done by copying slices, so no
    kernel waits on another): the head-shard inputs each rank receives equal
    the oracle's INT8 round trip of the raw tensors; the result is bit for bit
    the G = 1 result (scales are per (token, head) row, so G cannot matter);
    and the G = 1 result differs from the plain chain on the same dequantised
    inputs only by the FP8 rounding of O (at most 2^-4 of each value, plus the
    e4m3 subnormal step and the bf16 rounding).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.gpu_common import cpu_inputs, np64
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def seeded_rows(shape, seed):
    rng = np.random.default_rng([seed, 17])
    x = rng.standard_normal(shape) * np.exp2(rng.uniform(-6, 6, shape[:-1] + (1,)))
    x[0, 0, 0] = 0.0                                     # an all-zero row
    x[0, -1, -1, :3] = [448.0, -1000.0, 3e-5]            # large and tiny values in one row
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def code_values(codes_u8: torch.Tensor, kind: str) -> np.ndarray:
    if kind == "int8":
        return codes_u8.view(torch.int8).cpu().numpy().astype(np.float64)
    return codes_u8.view(torch.float8_e4m3fn).cpu().to(torch.float64).numpy()


@pytest.mark.parametrize("kind", ["int8", "e4m3"])
@pytest.mark.parametrize("split,G", [("heads", 1), ("heads", 2), ("heads", 4), ("tokens", 2), ("tokens", 3)])
def test_quant_pack_matches_oracle(sol, kind, split, G):
    B, N, H, D = 2, 96, 4, 128
    x = seeded_rows((B, N, H, D), seed=G)
    rows = B * N * H
    codes = torch.empty(rows * D, dtype=torch.uint8, device="cuda")
    scales = torch.empty(rows, dtype=torch.float32, device="cuda")
    sol.sol_quant_pack(x.cuda(), G, sol.SOL_SPLIT_HEADS if split == "heads" else sol.SOL_SPLIT_TOKENS,
                       sol.SOL_CODE_INT8 if kind == "int8" else sol.SOL_CODE_E4M3, codes, scales)
    torch.cuda.synchronize()
    want_c, want_s = orc.quantize_rows(x.float().numpy(), kind)          # [B, N, H, D], [B, N, H]
    if split == "heads":                                                  # -> [G, B, N, H/G]
        want_c = want_c.reshape(B, N, G, H // G, D).transpose(2, 0, 1, 3, 4)
        want_s = want_s.reshape(B, N, G, H // G).transpose(2, 0, 1, 3)
    else:                                                                 # -> [G, B, N/G, H]
        want_c = want_c.reshape(B, G, N // G, H, D).transpose(1, 0, 2, 3, 4)
        want_s = want_s.reshape(B, G, N // G, H).transpose(1, 0, 2, 3)
    got_c = code_values(codes, kind).reshape(want_c.shape)
    got_s = scales.cpu().numpy().reshape(want_s.shape)
    assert np.array_equal(got_s, want_s)
    assert np.array_equal(got_c, want_c)


@pytest.mark.parametrize("kind", ["int8", "e4m3"])
@pytest.mark.parametrize("split,G", [("heads", 2), ("tokens", 4)])
def test_dequant_unpack_matches_oracle(sol, kind, split, G):
    B, Nc, Hc, D = 2, 40, 3, 128
    rng = np.random.default_rng([G, 23])
    if kind == "int8":
        codes = torch.from_numpy(rng.integers(-127, 128, size=(G, B, Nc, Hc, D)).astype(np.int8)).view(torch.uint8)
    else:
        vals = orc.e4m3_round(rng.standard_normal((G, B, Nc, Hc, D)) * 100)
        codes = torch.from_numpy(vals.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)
    scales = torch.from_numpy((rng.uniform(0.0, 2.0, (G, B, Nc, Hc)) ** 3).astype(np.float32))
    out_shape = (B, G * Nc, Hc, D) if split == "heads" else (B, Nc, G * Hc, D)
    out = torch.empty(out_shape, dtype=torch.bfloat16, device="cuda")
    sol.sol_dequant_unpack(codes.contiguous().cuda(), scales.cuda(), B, Nc, Hc, D, G,
                           sol.SOL_SPLIT_HEADS if split == "heads" else sol.SOL_SPLIT_TOKENS,
                           sol.SOL_CODE_INT8 if kind == "int8" else sol.SOL_CODE_E4M3, out)
    torch.cuda.synchronize()
    want = orc.dequantize_rows(code_values(codes, kind).reshape(G, B, Nc, Hc, D), scales.numpy())
    if split == "heads":
        want = want.transpose(1, 0, 2, 3, 4).reshape(out_shape)
    else:
        want = want.transpose(1, 2, 0, 3, 4).reshape(out_shape)
    assert np.array_equal(np64(out), want)


def run_ranks(sol, G, wl, inp, H):
    """Every stage for every rank in turn; the exchange copies slices (slice g of
    rank r's send buffer -> slice r of rank g's receive buffer)."""
    from block_sparse_attention_sol_b200.seqpar import SeqParallelAttention
    q, k, v = (inp[n][:, :, :H].contiguous().cuda() for n in ("q", "k", "v"))
    gq, gk = (inp[n][:H * wl.D].contiguous().cuda() for n in ("gamma_q", "gamma_k"))
    ranks = [SeqParallelAttention(r, G, wl.B, wl.N, H, wl.D, wl.grid, wl.block, min(wl.topk), gq, gk,
                                  wl.rope_split, wl.rope_theta, wl.eps) for r in range(G)]
    Nl = wl.N // G
    for r, rk in enumerate(ranks):
        rk.stage_pack(*(x[:, r * Nl:(r + 1) * Nl].contiguous() for x in (q, k, v)))

    def exchange(send_name, recv_name):
        for r, rk in enumerate(ranks):
            for g, dst in enumerate(ranks):
                src = getattr(rk, send_name).view(G, -1)[g]
                getattr(dst, recv_name).view(G, -1)[r].copy_(src)

    exchange("send_qkv", "recv_qkv")
    exchange("send_qkv_s", "recv_qkv_s")
    lses = [rk.stage_compute() for rk in ranks]
    exchange("send_o", "recv_o")
    exchange("send_o_s", "recv_o_s")
    o = torch.cat([rk.stage_unpack() for rk in ranks], dim=1)
    torch.cuda.synchronize()
    return ranks, o, torch.cat(lses, dim=1), (q, k, v, gq, gk)


def test_seqpar_ranks_on_one_gpu(sol):
    wl = WORKLOADS[1]
    inp = cpu_inputs(1)
    H = 8
    ranks1, o1, lse1, (q, k, v, gq, gk) = run_ranks(sol, 1, wl, inp, H)
    # what the attention received: the oracle's INT8 round trip of the raw tensors
    for name, x in (("q_h", q), ("k_h", k), ("v_h", v)):
        assert np.array_equal(np64(getattr(ranks1[0], name)), orc.quant_roundtrip(np64(x), "int8")), name
    for G in (2, 4):
        ranks, o, lse, _ = run_ranks(sol, G, wl, inp, H)
        for r, rk in enumerate(ranks):                    # each rank's head shard of all tokens
            h0 = r * (H // G)
            assert torch.equal(rk.v_h, ranks1[0].v_h[:, :, h0:h0 + H // G])
        assert torch.equal(o, o1) and torch.equal(lse, lse1), G
    # against the plain chain on the same dequantised inputs: only O's FP8 round trip differs
    qq, kk, qbar, kbar = sol.sol_qk_prologue_pool(ranks1[0].q_h, ranks1[0].k_h, gq, gk, wl.grid, wl.block,
                                                  wl.rope_split, wl.rope_theta, wl.eps)
    idx = sol.sol_block_select_pooled(qbar, kbar, wl.grid, wl.block, min(wl.topk))
    o_ref, lse_ref = sol.sol_sparse_attn_fwd(qq, kk, ranks1[0].v_h, idx, wl.grid, wl.block)
    torch.cuda.synchronize()
    assert torch.equal(lse1, lse_ref)
    ref = np64(o_ref)
    amax = np.abs(ref).max(axis=-1, keepdims=True)
    bound = 2.0 ** -4 * np.abs(ref) + 2.0 ** -10 * amax / 448.0 + 2.0 ** -8 * (np.abs(ref) * (1 + 2.0 ** -4))
    assert (np.abs(np64(o1) - ref) <= bound + 1e-30).all()
