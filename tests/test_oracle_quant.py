"""Pins of the oracle's quantisers (INT8 and FP8 e4m3 rows, per-row fp32 scale).

Independent references: torch's float8_e4m3fn conversion (a library routine),
a brute-force nearest-level search over all 255 INT8 levels, hand values, and
the error bounds the formats imply.
"""
import numpy as np
import pytest
import torch

import oracle as orc


def test_e4m3_round_matches_torch():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(200_000) * np.exp2(rng.uniform(-14, 9, 200_000))).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(orc.e4m3_round(x.astype(np.float64)), want)


def test_e4m3_hand_values_and_saturation():
    cases = {0.0: 0.0, 1.0: 1.0, 1.0625: 1.0, 1.1875: 1.25, 448.0: 448.0, 460.0: 448.0, 1e6: 448.0,
             -1e6: -448.0, 2.0 ** -9: 2.0 ** -9, 2.0 ** -10: 0.0, 3 * 2.0 ** -10: 2.0 ** -8, 0.3: 0.3125}
    for x, want in cases.items():
        assert orc.e4m3_round(np.array([x]))[0] == want, x


def test_int8_codes_brute_force():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((64, 16)).astype(np.float32)
    x[3] = 0.0                                            # an all-zero row
    x[5, 2] = -x[5].__abs__().max() * 1.0                  # the extreme is negative
    codes, s = orc.quantize_rows(x, "int8")
    levels = np.arange(-127, 128, dtype=np.float64)
    for r in range(x.shape[0]):
        if s[r] == 0:
            assert (codes[r] == 0).all()
            continue
        recip = np.float32(127.0) / np.abs(x[r]).max()
        quo = (x[r] * recip).astype(np.float32).astype(np.float64)
        for d in range(x.shape[1]):
            dist = np.abs(levels - quo[d])
            best = levels[dist == dist.min()]
            want = best[0] if len(best) == 1 else best[best % 2 == 0][0]   # ties to the even level
            assert codes[r, d] == want
        assert np.abs(codes[r]).max() == 127                # the row's extreme maps to +-127


def test_scales_and_dequantize_hand_case():
    x = np.array([[254.0, -127.0, 1.0, 0.0]], dtype=np.float32)
    codes, s = orc.quantize_rows(x, "int8")
    assert s[0] == np.float32(2.0)
    assert list(codes[0]) == [127.0, -64.0, 0.0, 0.0]       # -63.5 -> -64 (even), 0.5 -> 0 (even)
    assert list(orc.dequantize_rows(codes, s)[0]) == [254.0, -128.0, 0.0, 0.0]
    c8, s8 = orc.quantize_rows(np.array([[448.0, 1.0, -224.0]], dtype=np.float32), "e4m3")
    assert s8[0] == np.float32(1.0) and list(c8[0]) == [448.0, 1.0, -224.0]


@pytest.mark.parametrize("kind,rel", [("int8", 0.5 / 127), ("e4m3", 2.0 ** -4)])
def test_roundtrip_error_bounds(kind, rel):
    rng = np.random.default_rng(13)
    x = orc.bf16_round(rng.standard_normal((500, 128)) * np.exp2(rng.uniform(-4, 4, (500, 1))))
    y = orc.quant_roundtrip(x, kind)
    amax = np.abs(x).max(axis=-1, keepdims=True)
    # quantisation error <= rel of the row maximum (int8: half a level; e4m3: half a
    # mantissa step of the value, at most 2^-4 of it, plus the subnormal floor), then
    # one bf16 rounding (2^-8 relative)
    if kind == "int8":
        bound = rel * amax * (1 + 1e-6) + 2.0 ** -8 * np.abs(y)
    else:
        bound = rel * np.abs(x) + 2.0 ** -10 * amax / 448.0 + 2.0 ** -8 * np.abs(y)
    assert (np.abs(y - x) <= bound + 1e-12).all()


def test_head_scales_fp8_inputs():
    rng = np.random.default_rng(14)
    v = rng.standard_normal((2, 48, 3, 16)).astype(np.float32)
    v[1, :, 2] = 0.0                                          # an all-zero head
    codes, s = orc.quantize_heads_e4m3(v)
    for b in range(2):
        for h in range(3):
            a = np.abs(v[b, :, h]).max()
            assert s[b, h] == np.float32(a / np.float32(448.0))
            if a == 0:
                assert (codes[b, :, h] == 0).all()
                continue
            # codes are the e4m3 values nearest to v * (448 / amax), checked against torch's cast
            quo = (v[b, :, h] * (np.float32(448.0) / np.float32(a))).astype(np.float32)
            want = torch.from_numpy(np.clip(quo, -448, 448)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
            assert np.array_equal(codes[b, :, h], want)
            assert np.abs(codes[b, :, h]).max() == 448.0
    d = orc.fp8_attention_inputs(v, v, v)
    assert d["q_scales"].shape == (2, 3, 48) and d["v_scales"].shape == (2, 3) and d["k_scales"].shape == (2, 3, 1)
    # K blocks of 128 tokens: with 48 tokens one block, so K's scales are V's and its codes too
    assert np.array_equal(d["k_scales"][:, :, 0], s) and np.array_equal(d["k_codes"], codes)
    kc, ks = orc.quantize_blocks_e4m3(np.concatenate([v, 2 * v, v], axis=1), 48)   # 3 blocks of 48
    assert np.array_equal(ks[:, :, 1], 2 * s) and np.array_equal(kc[:, 48:96], codes)
    assert np.allclose(d["v_deq"], v, rtol=2.0 ** -4, atol=2.0 ** -10 * np.abs(v).max() / 448 * 2)


def test_vt_key_order_is_a_permutation_of_each_16_group():
    order = orc.VT_KEY_ORDER
    assert sorted(order) == list(range(16))
    # position 4 c + e of a group (TMEM column c, byte e) holds key 2 c + (e & 1) + 8 (e >> 1)
    for pos in range(16):
        c, e = pos // 4, pos % 4
        assert order[pos] == 2 * c + (e & 1) + 8 * (e >> 1)
