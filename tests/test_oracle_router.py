"""Pins of the oracle's router (pooling -> MLP -> argmax) by closed forms.

'Flux Attention' router paragraphs: the first and last 100 query tokens are
compressed from [200 x h x d'] to [1 x h x d'], an MLP context encoder and a
router head give pi_FA and pi_SA, and inference takes the argmax.  The pages
print no numeric router example, so the pins are closed forms that a dropped
term, a wrong window, a transposed weight or a flipped comparison would fail.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import inputs


def _bits(x: np.ndarray) -> np.ndarray:
    return inputs.bits(torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16))


def test_constants_match_pages(golden_dir):
    with open(os.path.join(golden_dir, "flux_constants.json")) as f:
        g = json.load(f)
    assert oracle.N_HEAD_TOKENS == g["pool_head_tokens"]
    assert oracle.N_TAIL_TOKENS == g["pool_tail_tokens"]
    assert oracle.N_HEAD_TOKENS + oracle.N_TAIL_TOKENS == g["pooled_rows"]
    assert oracle.BLOCK == g["sparsity_block"]
    assert oracle.SINK_TOKENS == g["sink_tokens"]


def test_pool_closed_form_token_ramp():
    # Q[t, h, d] = (t mod 8) + h: the mean over tokens 0..99 and S-100..S-1
    # has a closed form that depends on which tokens are taken.
    B, S, Hq, D = 2, 300, 3, 4
    t = np.arange(S)[None, :, None, None]
    h = np.arange(Hq)[None, None, :, None]
    q = np.broadcast_to((t % 8) + h + 0 * np.arange(D), (B, S, Hq, D)).astype(np.float32)
    x = oracle.router_pool(_bits(q))
    sel = list(range(100)) + list(range(S - 100, S))
    expect_t = np.mean([s % 8 for s in sel])
    for hh in range(Hq):
        np.testing.assert_allclose(x[:, hh * D:(hh + 1) * D], expect_t + hh, atol=1e-12)
    # a wrong window (e.g. the first 200 tokens) gives another value
    assert abs(np.mean([s % 8 for s in range(200)]) - expect_t) > 1e-3


def test_pool_ignores_middle_tokens_and_is_head_major():
    B, S, Hq, D = 1, 260, 2, 8
    q = np.zeros((B, S, Hq, D), np.float32)
    q[0, 150, :, :] = 100.0           # middle token: not pooled
    q[0, 5, 1, 3] = 2.0               # head 1, dim 3, in the head window
    q[0, S - 1, 0, 6] = -4.0          # head 0, dim 6, in the tail window
    x = oracle.router_pool(_bits(q))
    expect = np.zeros(Hq * D)
    expect[1 * D + 3] = 2.0 / 200
    expect[0 * D + 6] = -4.0 / 200
    np.testing.assert_allclose(x[0], expect, atol=1e-15)


def test_pool_rejects_overlapping_windows():
    with pytest.raises(ValueError):
        oracle.router_pool(np.zeros((1, 199, 1, 4), np.uint16))


def test_mlp_closed_form_selection_weights():
    # W1 picks coordinates 0 and 2 with signs; ReLU zeroes the negative one;
    # W2 routes hidden unit 0 to pi_FA and unit 1 to pi_SA.
    x = np.array([[0.5, -7.0, -0.25, 3.0]])
    w1 = np.array([[1.0, 0, 0, 0], [0, 0, 1.0, 0], [0, 0, 0, 2.0]])
    b1 = np.array([0.0, 0.0, -10.0])
    w2 = np.array([[1.0, 0.0, 1.0], [0.0, -1.0, 0.0]])
    b2 = np.array([0.125, 0.0])
    logits = oracle.router_mlp(x, w1, b1, w2, b2)
    # h = relu([0.5, -0.25, 6 - 10]) = [0.5, 0, 0]
    np.testing.assert_allclose(logits, [[0.5 + 0.125, 0.0]], atol=1e-15)


def test_mlp_linear_regime_matches_matrix_product():
    # With a bias large enough to keep every hidden unit positive, the MLP
    # is the affine map W2 (W1 x + b1) + b2.
    rng = np.random.default_rng(3)
    x = rng.normal(size=(3, 16))
    w1 = rng.normal(size=(8, 16)) * 0.1
    b1 = np.full(8, 100.0)
    w2 = rng.normal(size=(2, 8))
    b2 = rng.normal(size=2)
    expect = (w2 @ w1) @ x.T + (w2 @ b1 + b2)[:, None]
    np.testing.assert_allclose(oracle.router_mlp(x, w1, b1, w2, b2), expect.T, atol=1e-10)


def test_argmax_and_tie_rule():
    logits = np.array([[0.2, 0.1], [0.1, 0.2], [0.3, 0.3], [-1.0, -0.5]])
    np.testing.assert_array_equal(oracle.router_argmax(logits), [0, 1, 0, 1])
    assert oracle.MODE_FULL == 0 and oracle.MODE_SPARSE == 1


def test_router_decide_bias_forces_mode():
    # A bias on pi_SA much larger than the logit spread of N(0, 0.02) weights
    # forces SPARSE, and on pi_FA forces FULL (used by the 32-layer stack).
    q, _, _ = inputs.qkv(1, 256, 4, 4, 128, seed=5)
    qb = inputs.bits(q)
    for b2, want in (((0.0, 0.1), 1), ((0.1, 0.0), 0)):
        w1, b1, w2, b2t = inputs.router_weights(4 * 128, 64, seed=5, b2=b2)
        logits, mode, _ = oracle.router_decide(qb, w1.numpy(), b1.numpy(), w2.numpy(), b2t.numpy())
        assert mode[0] == want
        assert abs(logits[0, 1] - logits[0, 0]) > 0.05
