"""The FMA-pipe exp2 the prefill kernel can use for a share of the softmax
(a compile-time share: a quarter of the keys by default):
range reduction x = n + f with the 1.5*2^23 shifter, a degree-3 polynomial
for 2^f on [-1/2, 1/2], n added to the exponent field.  The constants are
read from the kernel source and the routine is replayed in fp32 numpy, op
for op, against exp2 (fp64): relative error must stay below 1.1e-4 (under
the 2^-9 rounding of the bf16 P it feeds), and inputs below -127 give 0."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_attention_layerrouter_b200", "csrc", "fa_prefill.cu")


def _coeffs():
    text = open(SRC).read()
    return [np.float32(float(re.search(r"kExp2C%d = ([0-9.eE+-]+)f;" % i, text).group(1)))
            for i in (1, 2, 3)]


def ex2_poly(x):
    c1, c2, c3 = _coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = (c3 * f + c2).astype(np.float32)
    p = (p * f + c1).astype(np.float32)
    p = (p * f + np.float32(1.0)).astype(np.float32)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 1_000_001).astype(np.float32)
    rel = np.abs(ex2_poly(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < 1.1e-4, rel.max()


def test_exact_at_integers_and_underflow():
    ints = np.arange(-120, 9).astype(np.float32)
    np.testing.assert_array_equal(ex2_poly(ints), np.exp2(ints))
    assert np.all(ex2_poly(np.array([-127.0, -200.0, -np.inf], np.float32)) == 0.0)


def test_continuity_across_half_integers():
    x = np.array([k + 0.5 for k in range(-20, 8)], np.float32)
    lo = ex2_poly(np.nextafter(x, np.float32(-1e9)))
    hi = ex2_poly(x)
    assert np.max(np.abs(hi / lo - 1)) < 3e-4
