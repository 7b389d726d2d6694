"""Pins of the soft-routing forward ('Flux Attention', router paragraph on
training: Gumbel-softmax relaxation r_soft = exp((pi_FA + g_FA)/tau) /
sum_i exp((pi_i + g_i)/tau); the full and sparse outputs are mixed by r)."""
import math

import numpy as np
import pytest

import oracle


def test_two_way_softmax_is_a_sigmoid_of_the_logit_gap():
    logits = np.array([[0.3, -0.2], [1.0, 1.0], [-2.0, 5.0]])
    r = oracle.router_soft(logits)
    gap = logits[:, 0] - logits[:, 1]
    np.testing.assert_allclose(r, 1 / (1 + np.exp(-gap)), atol=1e-15)
    assert r[1] == 0.5


def test_gumbel_noise_and_temperature():
    logits = np.array([[0.1, 0.4]])
    g = np.array([[0.7, -0.1]])
    tau = 0.5
    want = math.exp((0.1 + 0.7) / tau) / (math.exp((0.1 + 0.7) / tau) + math.exp((0.4 - 0.1) / tau))
    assert abs(oracle.router_soft(logits, g, tau)[0] - want) < 1e-15
    # tau -> 0 recovers the hard decision on the noisy logits; large tau -> 1/2
    assert oracle.router_soft(logits, g, 1e-3)[0] > 1 - 1e-12
    assert abs(oracle.router_soft(logits, g, 1e6)[0] - 0.5) < 1e-6
    # hard routing on the same (noise-free) logits picks SPARSE here
    assert oracle.router_argmax(logits)[0] == oracle.MODE_SPARSE
    assert oracle.router_soft(logits, None, 1e-3)[0] < 1e-12


@pytest.mark.parametrize("r", [0.0, 0.25, 1.0])
def test_soft_mix_endpoints_and_linearity(r):
    rng = np.random.default_rng(7)
    a, b = rng.normal(size=(1, 5, 2, 3)), rng.normal(size=(1, 5, 2, 3))
    y = oracle.soft_mix(a, b, np.array([r]))
    np.testing.assert_allclose(y, r * a + (1 - r) * b, atol=1e-15)
    if r == 1.0:
        np.testing.assert_array_equal(y, a)
    if r == 0.0:
        np.testing.assert_array_equal(y, b)
