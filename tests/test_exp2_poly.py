"""The FMA-pipe exp2 used for part of the softmax: its coefficients come from
the committed generator, and the float32 operation sequence of ex2_poly stays
within the fitted relative-error bound of 2^x (far below bf16's 2^-9)."""
import os
import re
import sys

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "long_context_prefill_trianglemix_b200", "csrc")


def coefficients():
    text = open(os.path.join(CSRC, "tm_exp2_poly.h")).read()
    c = [float(re.search(rf"TM_EXP2_C{i} ([-0-9.e]+)f", text).group(1)) for i in range(4)]
    bound = float(re.search(r"TM_EXP2_MAX_REL_ERR ([-0-9.e]+)", text).group(1))
    return np.array(c, np.float32), bound


def fma32(a, b, c):
    return (a.astype(np.float64) * b + c).astype(np.float32)


def ex2_poly(x):
    """float32 emulation of the device routine, step by step."""
    c0, c1, c2, c3 = coefficients()[0]
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    p = fma32(fma32(fma32(np.full_like(f, c3), f, c2), f, c1), f, c0)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_header_matches_generator(tmp_path):
    sys.path.insert(0, CSRC)
    try:
        import gen_exp2_poly
        c, err = gen_exp2_poly.fit()
    finally:
        sys.path.remove(CSRC)
    have, bound = coefficients()
    np.testing.assert_array_equal(c, have)
    assert abs(err - bound) <= 1e-3 * bound


def test_relative_error_bound():
    _, bound = coefficients()
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001, dtype=np.float64),
                        np.arange(-125, 9, dtype=np.float64) + 0.5]).astype(np.float32)
    got = ex2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() <= bound + 2e-7, rel.max()
    assert bound < 2.0 ** -9 / 10


def test_clamp_and_masked_scores():
    out = ex2_poly(np.array([-np.inf, -1000.0, -125.0], np.float32))
    assert np.all(out > 0) and np.all(out < 2.0 ** -124)
    assert ex2_poly(np.array([0.0], np.float32))[0] == np.float32(coefficients()[0][0])
