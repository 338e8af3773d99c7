"""The attention kernel's FMA-pipe exponential: its polynomial constants (read
from the CUDA header) evaluated step by step in fp32, against 2^x in float64.
The kernel's results feed P, which is rounded to bf16 (relative step 2^-8),
so a relative error below 1e-4 is far inside what the output tolerance needs."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_sol_b200", "csrc", "sm100_ptx.cuh")


def constants():
    text = open(HDR).read()
    vals = {}
    for name in ("kExp2C1", "kExp2C2", "kExp2C3"):
        m = re.search(name + r"\s*=\s*(0x[0-9a-fA-Fp.+-]+)f;", text)
        vals[name] = np.float32(float.fromhex(m.group(1)))
    return vals["kExp2C1"], vals["kExp2C2"], vals["kExp2C3"]


def emulate(x):
    """The kernel's steps in fp32: clamp, floor, fraction, Horner, exponent add."""
    c1, c2, c3 = constants()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    n = np.floor(x).astype(np.float32)               # add.rm + sub of 1.5*2^23 is exact floor here
    f = (x - n).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    bits = p.view(np.int32) + (n.astype(np.int32) << 23)
    return bits.view(np.float32)


def test_constants_match_the_fit_script():
    import importlib.util
    spec = importlib.util.spec_from_file_location("fit", os.path.join(os.path.dirname(HDR), "fit_exp2_poly.py"))
    fit = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(fit)
    c, _ = fit.fit()
    np.testing.assert_array_equal(np.array(constants()), c)


def test_relative_error_over_the_softmax_range():
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float32)
    got = emulate(x).astype(np.float64)
    want = 2.0 ** x.astype(np.float64)
    assert np.max(np.abs(got / want - 1.0)) < 1e-4


def test_special_values():
    np.testing.assert_array_equal(emulate([0.0, 1.0, 8.0, -1.0, -3.0]), [1.0, 2.0, 256.0, 0.5, 0.125])
    assert emulate([-127.0])[0] == 0.0
    assert emulate([-np.inf])[0] == 0.0
    assert 0.0 <= emulate([-200.0])[0] < 2.0 ** -126
