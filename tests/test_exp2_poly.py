"""Host checks of the exp2 approximation the prefill attention kernel uses for part of P.

The kernel computes 2^x = 2^n * 2^f with n = round(x), f = x - n in [-1/2, 1/2], and 2^f by a
cubic whose coefficients (kP0..kP3) and rounding constant live in csrc/flash_attn.cuh.  These
tests read those constants from the header and check the arithmetic the kernel performs, in
float32, against numpy's exp2: the relative error must stay below 7.6e-5 (the minimax bound the
fit was made for, well under the 2^-9 rounding of the bf16 P it feeds), the exponent assembly
must be exact, and inputs at or below -125 (masked keys are -inf) must give at most 2^-124.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(__file__), "..", "tensor_transformer_matmul_b200", "csrc",
                   "flash_attn.cuh")


def _constants():
    src = open(HDR).read()
    vals = {}
    for name in ("kP0", "kP1", "kP2", "kP3", "kRoundMagic"):
        m = re.search(name + r"\s*=\s*([0-9.eE+-]+)f", src)
        assert m, name
        vals[name] = np.float32(float(m.group(1)))
    return vals


def _exp2_poly(x):
    """float32 restatement of the kernel's exp2_poly_x2 (one lane)."""
    c = _constants()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    j = (x + c["kRoundMagic"]).astype(np.float32)
    n = (j - c["kRoundMagic"]).astype(np.float32)
    f = (x - n).astype(np.float32)
    q = (c["kP3"] * f + c["kP2"]).astype(np.float32)
    q = (q * f + c["kP1"]).astype(np.float32)
    q = (q * f + c["kP0"]).astype(np.float32)
    bits = q.view(np.uint32).astype(np.uint64) + j.view(np.uint32).astype(np.uint64) * (1 << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-100.0, 8.5, 400001, dtype=np.float32)
    ref = np.exp2(x.astype(np.float64))
    got = _exp2_poly(x).astype(np.float64)
    rel = np.abs(got - ref) / ref
    assert rel.max() < 7.6e-5, rel.max()


def test_integer_inputs_are_close_to_powers_of_two():
    for n in range(-120, 9):
        got = float(_exp2_poly(np.float32(n)))
        assert abs(got / 2.0 ** n - 1.0) < 7.6e-5


def test_reduction_uses_round_to_nearest():
    # f = x - round(x) stays in [-1/2, 1/2], the interval the cubic was fitted on
    c = _constants()
    x = np.linspace(-60.0, 8.0, 100001, dtype=np.float32)
    j = (x + c["kRoundMagic"]).astype(np.float32)
    f = x - (j - c["kRoundMagic"]).astype(np.float32)
    assert np.abs(f).max() <= 0.5


def test_masked_keys_vanish():
    got = _exp2_poly(np.array([-np.inf, -1e30, -200.0, -125.0], np.float32))
    assert np.all(got > 0) and np.all(got <= 2.0 ** -124)
