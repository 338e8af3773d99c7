"""GPU parity of the FP8 (e4m3) attention and its input quantiser.

  * sol_quant_attn_fp8: Q/K codes and row scales, V^T codes (keys permuted in
    groups of 16 as documented) and head scales bit for bit equal to the
    oracle's quantisation (both decide each code in fp32).
  * sol_sparse_attn_fwd_fp8, fed the ORACLE's codes and scales: O and LSE
    against the oracle's exact attention of the dequantised values.  The
    kernel's products are exact up to fp32 accumulation (e4m3 x e4m3 products
    are exact in fp32); its one approximation is rounding the softmax weights
    to e4m3 for the P V product (relative 2^-4 at most, normaliser unrounded),
    so each output channel may differ by 2^-4 * sum_m p_m |v_m,d| / sum_m p_m,
    plus the final bf16 rounding (2^-8 relative) and 2e-3 for weights in the
    e4m3 subnormal range and accumulation order.  LSE within 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from tests.gpu_common import cpu_inputs, np64, sample_units
from workloads import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu


def vt_layout(v_codes):
    """[B, N, H, D] codes -> the documented V^T layout [B, H, D, N] (keys permuted per 16)."""
    B, N, H, D = v_codes.shape
    perm = np.concatenate([16 * g + np.asarray(orc.VT_KEY_ORDER) for g in range(N // 16)])
    return np.ascontiguousarray(v_codes.transpose(0, 2, 3, 1)[..., perm])


def e4m3_bytes(values: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(values, dtype=np.float32)).to(torch.float8_e4m3fn).view(torch.uint8)


def e4m3_values(codes_u8: torch.Tensor) -> np.ndarray:
    return codes_u8.view(torch.float8_e4m3fn).cpu().to(torch.float64).numpy()


CASES = [("w1", 1, 4), ("ragged", None, 4)]


def case_inputs(kind):
    if kind == "w1":
        wl = WORKLOADS[1]
        inp = cpu_inputs(1)
        return wl, {n: inp[n][:, :, :4].contiguous() for n in ("q", "k", "v")}
    # 3 x 8 x 40 grid = 960 tokens: 7 full blocks of 128 and a last block of 64
    wl = Workload(config_id=91, name="small bf16, ragged last block", dtype="bf16", B=2, H=2, D=128,
                  grid=(3, 8, 40), block=128, topk=(3,))
    return wl, make_inputs(wl, seed=9, names=("q", "k", "v"))


@pytest.mark.parametrize("kind", ["w1", "ragged"])
def test_quant_attn_fp8_matches_oracle(sol, kind):
    wl, inp = case_inputs(kind)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    out = sol.sol_quant_attn_fp8(q, k, v, wl.grid)
    torch.cuda.synchronize()
    ref = orc.fp8_attention_inputs(*(inp[n].float().numpy() for n in ("q", "k", "v")))
    assert np.array_equal(e4m3_values(out["q8"]), ref["q_codes"])
    assert np.array_equal(e4m3_values(out["k8"]), ref["k_codes"])
    assert np.array_equal(out["q_scale"].cpu().numpy(), ref["q_scales"])
    assert np.array_equal(out["k_scale"].cpu().numpy(), ref["k_scales"])
    assert np.array_equal(out["v_scale"].cpu().numpy(), ref["v_scales"])
    assert np.array_equal(e4m3_values(out["vt8"]), vt_layout(ref["v_codes"]))


def fp8_tolerance(q, k, v, idx, blocks, units, scale, counts=None):
    """Per (unit row, channel) bound of the e4m3 rounding of P (module docstring)."""
    bounds = {}
    N = q.shape[1]
    for (b, h, i) in units:
        rows = np.arange(i * blocks, min(N, (i + 1) * blocks))
        kept = idx[b, h, i][: None if counts is None else int(counts[b, h, i])]
        cols = np.concatenate([np.arange(j * blocks, min(N, (j + 1) * blocks)) for j in kept])
        logits = scale * (q[b, rows, h] @ k[b, cols, h].T)
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        bounds[(b, h, i)] = 2.0 ** -4 * (p @ np.abs(v[b, cols, h])) / p.sum(axis=1, keepdims=True)
    return bounds


@pytest.mark.parametrize("kind,with_counts", [("w1", False), ("w1", True), ("ragged", False)])
def test_attention_fp8_matches_oracle(sol, kind, with_counts):
    wl, inp = case_inputs(kind)
    ref = orc.fp8_attention_inputs(*(inp[n].float().numpy() for n in ("q", "k", "v")))
    B, N, H, D = ref["q_codes"].shape
    nb = -(-N // wl.block)
    topk = min(12, nb)
    rng = np.random.default_rng([N, 3])
    idx = np.stack([np.sort(rng.permutation(nb)[:topk]) for _ in range(B * H * nb)]).reshape(B, H, nb, topk)
    idx = idx.astype(np.int32)
    idx[:, :, :, -1] = np.where((idx[:, :, :, :-1] == nb - 1).any(-1), idx[:, :, :, -1], nb - 1)   # the last block
    idx = np.sort(idx, axis=-1)
    counts = rng.integers(1, topk + 1, size=(B, H, nb)).astype(np.int32) if with_counts else None
    fp8 = {"q8": e4m3_bytes(ref["q_codes"]).cuda(), "k8": e4m3_bytes(ref["k_codes"]).cuda(),
           "vt8": e4m3_bytes(vt_layout(ref["v_codes"])).cuda(),
           "q_scale": torch.from_numpy(ref["q_scales"]).cuda(), "k_scale": torch.from_numpy(ref["k_scales"]).cuda(),
           "v_scale": torch.from_numpy(ref["v_scales"]).cuda()}
    o, lse = sol.sol_sparse_attn_fwd_fp8(fp8, torch.from_numpy(idx).cuda(), wl.grid, wl.block,
                                         counts=torch.from_numpy(counts).cuda() if counts is not None else None)
    torch.cuda.synchronize()
    units = sample_units(B, H, nb, per_head=min(nb, 10))
    scale = 1.0 / np.sqrt(D)
    o_ref, lse_ref = orc.sparse_attention(ref["q_deq"], ref["k_deq"], ref["v_deq"], idx, wl.block, scale,
                                          units=units, counts=counts)
    bounds = fp8_tolerance(ref["q_deq"], ref["k_deq"], ref["v_deq"], idx, wl.block, units, scale, counts)
    worst = 0.0
    for (b, h, i) in units:
        r = np.arange(i * wl.block, min(N, (i + 1) * wl.block))
        got = np64(o[b, r, h])
        err = np.abs(got - o_ref[b, r, h])
        tol = bounds[(b, h, i)] + 2.0 ** -8 * np.abs(o_ref[b, r, h]) + 2e-3
        assert (err <= tol).all(), (b, h, i, float((err - tol).max()))
        worst = max(worst, float(err.max()))
        assert np.abs(np64(lse[b, h, r]) - lse_ref[b, h, r]).max() <= 1e-3
    assert worst < 0.1
    if counts is None:   # every count equal to topk gives the same result, bit for bit
        full = torch.full((B, H, nb), topk, dtype=torch.int32, device="cuda")
        o2, lse2 = sol.sol_sparse_attn_fwd_fp8(fp8, torch.from_numpy(idx).cuda(), wl.grid, wl.block, counts=full)
        torch.cuda.synchronize()
        assert torch.equal(o, o2) and torch.equal(lse, lse2)
