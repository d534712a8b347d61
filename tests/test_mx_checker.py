"""The MXFP8 parity checker (parity.check_mx) on the CPU: it accepts the
oracle's own quantisation of a matrix and rejects plausible kernel mistakes
(a scale off by one, a code off by one step, a flipped sign, a missing NaN
scale, codes of the wrong block)."""
import numpy as np
import pytest

import oracle
from parity import check_mx


def _matrix(seed=5):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((9, 128)) * np.exp2(rng.integers(-30, 30, (9, 1)))
    v[2, 3] = np.nan
    v[4, 64:96] = 0.0
    return v


@pytest.mark.parametrize("rule", [oracle.MX_RULE_OCP, oracle.MX_RULE_CEIL])
def test_checker_accepts_the_oracle(rule):
    o = oracle.load()
    v = _matrix()
    codes, scales = o.mxfp8_quantize(v, rule)
    rep = check_mx("oracle", codes, scales, v, 1e-6 * np.abs(np.nan_to_num(v)), rule)
    assert rep["exact"] == rep["codes"]


@pytest.mark.parametrize("mistake", ["scale+1", "code+1", "sign", "nan_scale", "block_swap"])
def test_checker_rejects_mistakes(mistake):
    o = oracle.load()
    v = _matrix()
    rule = oracle.MX_RULE_OCP
    codes, scales = o.mxfp8_quantize(v, rule)
    codes, scales = codes.copy(), scales.copy()
    if mistake == "scale+1":
        scales[1, 2] += 1
    elif mistake == "code+1":
        mag = int(codes[5, 10]) & 0x7F
        codes[5, 10] = (int(codes[5, 10]) & 0x80) | (mag + 1 if mag < 0x7E else mag - 1)
    elif mistake == "sign":
        codes[6, 40] ^= 0x80
        if v[6, 40] == 0:
            pytest.skip("zero element")
    elif mistake == "nan_scale":
        scales[2, 0] = 127
    elif mistake == "block_swap":
        codes[7, 0:32], codes[7, 32:64] = codes[7, 32:64].copy(), codes[7, 0:32].copy()
    with pytest.raises(AssertionError):
        check_mx("mutated", codes, scales, v, 1e-6 * np.abs(np.nan_to_num(v)), rule)
