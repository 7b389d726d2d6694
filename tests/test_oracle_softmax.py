"""Pins of the oracle's softmax pieces against what the pages fix.

Newsletter on Softmax and FlashAttention 1-4: the worked example, fp16
overflow, max-subtraction invariance and the online (blockwise) form.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def test_worked_example_exact_and_printed(golden_dir):
    g = _load(golden_dir, "softmax_worked_example.json")
    x = g["scores"]
    p = oracle.softmax(x)
    z = math.exp(2.0) + math.exp(1.0) + math.exp(0.5)
    exact = [math.exp(2.0) / z, math.exp(1.0) / z, math.exp(0.5) / z]
    np.testing.assert_allclose(p, exact, rtol=0, atol=1e-12)
    # The printed softmax vector is approximate on the page (off by up to
    # 0.0202 from the exact value); it must still be within 0.025.
    printed = np.array(g["printed_softmax"])
    dev = np.max(np.abs(p - printed))
    assert dev < 0.025, dev
    assert dev > 0.005  # the discrepancy is real; recorded, not hidden
    # Softmax concentrates more mass on the largest score than x/sum(x).
    plain = np.array(x) / np.sum(x)
    np.testing.assert_allclose(plain, g["printed_plain_normalisation"], atol=0.005)
    assert p[0] > plain[0] and p[2] < plain[2]


def test_rows_sum_to_one_and_shift_invariance():
    rng = np.random.default_rng(0)
    x = rng.normal(size=(64, 37)) * 5
    p = oracle.softmax(x)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(p > 0)
    for c in (-1e3, -1.0, 1.0, 1e3):
        np.testing.assert_allclose(oracle.softmax(x + c), p, atol=1e-12)


def test_fp16_overflow_threshold(golden_dir):
    g = _load(golden_dir, "fp16_overflow.json")
    thr = math.log(g["fp16_max_finite"])
    assert abs(thr - g["printed_threshold_approx"]) < 0.1
    with np.errstate(over="ignore"):
        assert np.isfinite(np.exp(np.float16(11.0)))
        assert np.isinf(np.exp(np.float16(11.25)))
        # naive softmax in fp16 breaks, the max-subtracted one does not
        x16 = np.array([12.0, 11.0, 10.0], dtype=np.float16)
        naive = np.exp(x16) / np.sum(np.exp(x16))
        assert not np.all(np.isfinite(naive))
        stable = np.exp(x16 - x16.max()) / np.sum(np.exp(x16 - x16.max()))
    assert np.all(np.isfinite(stable))
    np.testing.assert_allclose(stable.astype(np.float64),
                               oracle.softmax([12.0, 11.0, 10.0]), atol=2e-3)


def test_online_softmax_example(golden_dir):
    g = _load(golden_dir, "online_softmax_example.json")
    # Eight scores, two blocks of four, block maxima 4.1 then 5.0.
    x = np.array([1.0, 4.1, -2.0, 0.5, 3.0, 5.0, 2.0, -1.0])
    assert x[:4].max() == g["m_block1"] and x[4:].max() == g["m_block2"]
    p, m, l, factors = oracle.online_softmax(x, g["block"])
    assert m == 5.0
    assert abs(factors[1] - math.exp(-0.9)) < 1e-15
    assert abs(factors[1] - 0.4065696597405991) < 1e-12
    np.testing.assert_allclose(p, oracle.softmax(x), atol=1e-15)
    np.testing.assert_allclose(l, np.sum(np.exp(x - 5.0)), atol=1e-13)


@pytest.mark.parametrize("n,block", [(1, 1), (7, 3), (64, 64), (100, 7), (333, 64)])
def test_online_equals_one_pass(n, block):
    rng = np.random.default_rng(n * 31 + block)
    x = rng.normal(size=n) * 4
    p, m, l, _ = oracle.online_softmax(x, block)
    np.testing.assert_allclose(p, oracle.softmax(x), atol=1e-14)
    assert m == x.max()
    v = rng.normal(size=(n, 5))
    o = oracle.online_attention_row(x, v, block)
    np.testing.assert_allclose(o, oracle.softmax(x) @ v, atol=1e-13)


def test_online_catches_a_missing_rescale():
    """A blockwise form that forgets the exp(m_old - m_new) factor is wrong
    whenever a later block raises the maximum: the pin is sensitive."""
    x = np.array([0.0, 1.0, 5.0, 2.0])
    m, l = -math.inf, 0.0
    for s in range(0, 4, 2):
        c = x[s:s + 2]
        m_new = max(m, c.max())
        l = l + np.sum(np.exp(c - m_new))      # rescale dropped on purpose
        m = m_new
    assert abs(l - np.sum(np.exp(x - m))) > 1e-3
