"""Oracle of the quantised token <-> head exchange around the Sol-Attn path.

TEST INFRASTRUCTURE ONLY (like sol_oracle): imported by tests/ and nothing in
the product path.  It shares no code with the CUDA path.

Source.  For multi-GPU runs the Sol-H3 runtime moves Q, K and V between GPUs
as INT8 and the attention output as FP8, cutting inter-GPU traffic by about a
half (ai-feiten.nl, "Videomodel MiniMax-H3 rendert sneller dan afspelen",
section "Waar de snelheidswinst vandaan komt").  The pages give no format
details; the readings written out here are:

  - one scale per (token, head) row of D channels, symmetric, in fp32:
    s = max_d |x_d| / L with L = 127 (INT8) or 448 (FP8 e4m3, its largest
    finite value); a row of zeros gets s = 0 and all-zero codes;
  - the codes use the row's reciprocal scale r = L / max_d |x_d| (one IEEE
    fp32 division per row): INT8 code = clamp(round_half_even(x * r), -127,
    127); e4m3 code = x * r rounded to the nearest e4m3 value (ties to even),
    saturating at +-448; x * r is one fp32 product, and max, division,
    product and rounding decide the code in fp32 exactly as written;
  - dequantised value = bf16_round(fp32(code * s)).
  - sequence-parallel layout: G ranks; rank r owns tokens [r N/G, (r+1) N/G)
    of all heads before the attention and heads [r H/G, (r+1) H/G) of all
    tokens during it.  Because every scale belongs to one (token, head) row,
    the quantised values do not depend on G.
"""
from __future__ import annotations

import numpy as np

from .sol_oracle import bf16_round

__all__ = ["INT8_LEVELS", "E4M3_MAX", "e4m3_round", "quantize_rows", "dequantize_rows", "quant_roundtrip"]

INT8_LEVELS = 127.0
E4M3_MAX = 448.0


def e4m3_round(x) -> np.ndarray:
    """Nearest FP8 e4m3 value (ties to even), saturating at +-448; float64 result.

    e4m3: 1 sign, 4 exponent bits (bias 7), 3 mantissa bits, no infinities.
    Normal numbers m * 2^e with 1 <= m < 2 and e >= -6 are spaced 2^(e-3);
    below 2^-6 the subnormals are spaced 2^-9.  The largest finite value is
    1.75 * 2^8 = 448.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, fe = np.frexp(a)                           # a = f * 2^fe, 0.5 <= f < 1: exponent fe - 1
    e = np.maximum(fe.astype(np.float64) - 1.0, -6.0)   # subnormal range keeps the 2^-9 spacing
    step = np.exp2(e - 3.0)
    r = np.rint(a / step) * step                  # np.rint: half to even (in units of the step)
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def quantize_rows(x, kind: str):
    """Codes and scales of rows x[..., D] (stored bf16 / fp32 values).

    kind "int8" or "e4m3".  Returns (codes float64 [..., D] holding the code
    values, scales float32 [...]).
    """
    x32 = np.asarray(x, dtype=np.float32)
    levels = np.float32(INT8_LEVELS if kind == "int8" else E4M3_MAX)
    amax = np.max(np.abs(x32), axis=-1)
    s = (amax / levels).astype(np.float32)                       # one fp32 division
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    recip = (levels / safe).astype(np.float32)                   # one fp32 division per row
    quo = (x32 * recip[..., None]).astype(np.float32)            # one fp32 product per value
    if kind == "int8":
        codes = np.clip(np.rint(quo.astype(np.float64)), -127.0, 127.0)
    elif kind == "e4m3":
        codes = e4m3_round(quo.astype(np.float64))
    else:
        raise ValueError(kind)
    codes = np.where(s[..., None] > 0, codes, 0.0)
    return codes, s


def dequantize_rows(codes, scales) -> np.ndarray:
    """bf16_round(fp32(code * s)), float64 result."""
    prod = np.asarray(codes, np.float32) * np.asarray(scales, np.float32)[..., None]
    return bf16_round(prod.astype(np.float32).astype(np.float64))


def quant_roundtrip(x, kind: str) -> np.ndarray:
    """The values a tensor [..., D] arrives with after quantisation and dequantisation."""
    codes, s = quantize_rows(x, kind)
    return dequantize_rows(codes, s)


# ----------------------------------------------------------------------------- FP8 attention inputs
# Readings for the FP8 (e4m3) variant of the attention (the pages say only that
# the runtime uses FP8; the formats are this library's): Q rows are quantised
# like the exchange rows above (one scale per (token, head) row); K gets one
# scale per (batch, head, block of 128 tokens) and V one per (batch, head):
# s = max |x| over the group / 448, codes x * (448 / max |x|) rounded to
# nearest e4m3.  (e4m3 keeps values down to 2^-14 of a group's maximum normal,
# so block- and head-wide scales cost no precision on these inputs, and a block
# scale folds into the softmax's per-row factor.)  The
# attention is then the exact softmax attention of the dequantised values
# (code * scale, in fp64 here); the kernel's further rounding of P to e4m3 is
# an approximation that the tests bound.
__all__ += ["quantize_heads_e4m3", "quantize_blocks_e4m3", "fp8_attention_inputs", "VT_KEY_ORDER"]

# V is stored transposed, [B, H, D, N], with the keys of every aligned group of
# 16 in this order (position j of the group holds key VT_KEY_ORDER[j]).
VT_KEY_ORDER = (0, 1, 8, 9, 2, 3, 10, 11, 4, 5, 12, 13, 6, 7, 14, 15)


def quantize_heads_e4m3(v):
    """v [B, N, H, D] -> (codes float64 [B, N, H, D], scales float32 [B, H]), one scale per (b, h)."""
    v32 = np.asarray(v, dtype=np.float32)
    amax = np.max(np.abs(v32), axis=(1, 3))                       # [B, H]
    s = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
    recip = (np.float32(E4M3_MAX) / safe).astype(np.float32)
    quo = (v32 * recip[:, None, :, None]).astype(np.float32)
    codes = e4m3_round(quo.astype(np.float64))
    codes = np.where(s[:, None, :, None] > 0, codes, 0.0)
    return codes, s


def quantize_blocks_e4m3(x, block: int = 128):
    """x [B, N, H, D] -> (codes float64 [B, N, H, D], scales float32 [B, H, nb]), one scale per
    (b, h, block of `block` consecutive tokens; the last block may be short)."""
    x32 = np.asarray(x, dtype=np.float32)
    B, N, H, D = x32.shape
    nb = -(-N // block)
    codes = np.zeros(x32.shape)
    scales = np.zeros((B, H, nb), dtype=np.float32)
    for i in range(nb):
        seg = x32[:, i * block:(i + 1) * block]                      # [B, n_i, H, D]
        c, sc = quantize_heads_e4m3(seg)
        codes[:, i * block:(i + 1) * block] = c
        scales[:, :, i] = sc
    return codes, scales


def fp8_attention_inputs(q, k, v):
    """Codes, scales and the dequantised (exact, fp64) Q, K, V of the FP8 attention.

    Returns dict with q_codes, q_scales [B, H, N], k_codes, k_scales [B, H, nb]
    (blocks of 128 tokens), v_codes [B, N, H, D], v_scales [B, H], and q_deq,
    k_deq, v_deq (float64 [B, N, H, D], code * scale without further rounding)."""
    qc, qs = quantize_rows(q, "e4m3")                               # scales [B, N, H]
    kc, ks = quantize_blocks_e4m3(k, 128)
    vc, vs = quantize_heads_e4m3(v)
    N = kc.shape[1]
    ks_tok = np.repeat(ks, 128, axis=2)[:, :, :N]                   # [B, H, N]
    return {
        "q_codes": qc, "q_scales": np.ascontiguousarray(np.swapaxes(qs, 1, 2)),
        "k_codes": kc, "k_scales": ks,
        "v_codes": vc, "v_scales": vs,
        "q_deq": qc * qs.astype(np.float64)[..., None],
        "k_deq": kc * np.swapaxes(ks_tok, 1, 2).astype(np.float64)[..., None],
        "v_deq": vc * vs.astype(np.float64)[:, None, :, None],
    }
