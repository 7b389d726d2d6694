"""Pins of the oracle's backward functions (CPU only).

The gradients are checked against things other than themselves: central
finite differences of a pure-Python forward (tests/brute.py), the adjoint
identity of the pooling, conservation laws of the softmax Jacobian, and the
reduction of GQA to per-head sums."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import inputs
from tests import brute


def _tiny(B, S, Hq, Hkv, D, seed):
    q, k, v = inputs.qkv(B, S, Hq, Hkv, D, seed)
    do = inputs.randn_bf16((B, S, Hq, D), seed + 400)
    return [inputs.bits(t) for t in (q, k, v, do)]


def _f(bits):
    return oracle.bf16_bits_to_f64(bits)


def _brute_loss(q, k, v, do, scale, mode, block, sink, window):
    """sum(dO * O) with O from the pure-Python forward (fp64 floats)."""
    B, S, Hq, D = q.shape
    G = Hq // k.shape[2]
    total = 0.0
    for b in range(B):
        for h in range(Hq):
            K = [list(k[b, j, h // G]) for j in range(S)]
            V = [list(v[b, j, h // G]) for j in range(S)]
            for t in range(S):
                allowed = [brute.key_allowed(t, j, mode, block, sink, window) for j in range(S)]
                out, _ = brute.attention_row(list(q[b, t, h]), K, V, scale, allowed)
                total += sum(a * g for a, g in zip(out, do[b, t, h]))
    return total


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_backward_matches_central_differences(mode):
    B, S, Hq, Hkv, D = 1, 12, 2, 1, 3
    block, sink, window = 4, 4, 4
    qb, kb, vb, dob = _tiny(B, S, Hq, Hkv, D, seed=501)
    scale = 1 / math.sqrt(D)
    mask = None
    if mode == "sparse":
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, block, sink, window))
    dq, dk, dv = oracle.attention_backward(qb, kb, vb, dob, scale, mask, block)
    base = [_f(x) for x in (qb, kb, vb, dob)]
    eps = 1e-5
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        arr = base[which]
        for idx in np.ndindex(*arr.shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            fd = (_brute_loss(*plus, scale, mode, block, sink, window) -
                  _brute_loss(*minus, scale, mode, block, sink, window)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-7 * max(1.0, abs(fd)), (which, idx, fd, grad[idx])


def test_softmax_jacobian_conservation():
    """Rows of dS sum to 0, so sum_k dK_k = 0 per kv head; rows of P sum to
    1, so sum_k dV_k = sum over the group's query rows of dO."""
    B, S, Hq, Hkv, D = 2, 200, 4, 2, 16
    qb, kb, vb, dob = _tiny(B, S, Hq, Hkv, D, seed=502)
    for mask in (None, oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 64, 64))):
        dq, dk, dv = oracle.attention_backward(qb, kb, vb, dob, 0.25, mask, 64)
        np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-9)
        do = _f(dob).reshape(B, S, Hkv, Hq // Hkv, D).sum(axis=(1, 3))
        np.testing.assert_allclose(dv.sum(axis=1), do, atol=1e-9)
        # Row 0 attends one key: its softmax is constant, so dQ is 0 there.
        np.testing.assert_allclose(dq[:, 0], 0.0, atol=1e-12)


def test_gqa_sums_the_heads_of_a_group():
    """GQA on K/V equals MHA on the same K/V replicated per head, with the
    replicated heads' dK/dV summed."""
    B, S, Hq, Hkv, D = 1, 96, 4, 2, 8
    qb, kb, vb, dob = _tiny(B, S, Hq, Hkv, D, seed=503)
    G = Hq // Hkv
    k_rep = np.repeat(kb, G, axis=2)
    v_rep = np.repeat(vb, G, axis=2)
    dq_g, dk_g, dv_g = oracle.attention_backward(qb, kb, vb, dob, 0.3)
    dq_m, dk_m, dv_m = oracle.attention_backward(qb, k_rep, v_rep, dob, 0.3)
    np.testing.assert_allclose(dq_g, dq_m, atol=1e-12)
    np.testing.assert_allclose(dk_g, dk_m.reshape(B, S, Hkv, G, D).sum(axis=3), atol=1e-12)
    np.testing.assert_allclose(dv_g, dv_m.reshape(B, S, Hkv, G, D).sum(axis=3), atol=1e-12)


def test_all_ones_mask_equals_full():
    B, S, Hq, Hkv, D = 1, 128, 2, 2, 8
    qb, kb, vb, dob = _tiny(B, S, Hq, Hkv, D, seed=504)
    full = oracle.attention_backward(qb, kb, vb, dob, 0.35)
    ones = oracle.attention_backward(qb, kb, vb, dob, 0.35, np.ones((2, 2), np.uint8), 64)
    for a, b in zip(full, ones):
        np.testing.assert_allclose(a, b, atol=0)


def test_row_variants_agree_with_full_backward():
    B, S, Hq, Hkv, D = 2, 160, 4, 2, 16
    qb, kb, vb, dob = _tiny(B, S, Hq, Hkv, D, seed=505)
    mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 32, 32, 64))
    dq, dk, dv = oracle.attention_backward(qb, kb, vb, dob, 0.25, mask, 32)
    rows = np.array([(0, 0, 0), (1, 3, 159), (0, 2, 63), (1, 1, 64)], np.int64)
    got = oracle.attention_backward_qrows(qb, kb, vb, dob, 0.25, rows, mask, 32)
    np.testing.assert_allclose(got, dq[rows[:, 0], rows[:, 2], rows[:, 1]], atol=1e-12)
    keys = np.array([0, 31, 32, 100, 159], np.int64)
    gk, gv = oracle.attention_backward_keyrows(qb, kb, vb, dob, 0.25, 1, 1, keys, mask, 32)
    np.testing.assert_allclose(gk, dk[1, keys, 1], atol=1e-12)
    np.testing.assert_allclose(gv, dv[1, keys, 1], atol=1e-12)


def test_pool_backward_is_the_adjoint_of_pooling():
    """<pool^T(dx), Q> = <dx, pool(Q)> for any Q and dx."""
    B, S, Hq, D = 2, 300, 3, 8
    qb = inputs.bits(inputs.randn_bf16((B, S, Hq, D), 506))
    dx = np.random.default_rng(506).standard_normal((B, Hq * D))
    g = oracle.router_pool_backward(dx, S, Hq, D)
    lhs = (g * _f(qb)).sum()
    rhs = (dx * oracle.router_pool(qb)).sum()
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(rhs))
    # Tokens outside the first and last 100 receive nothing.
    assert np.all(g[:, 100:S - 100] == 0.0)


def test_soft_routed_backward_matches_central_differences():
    rng = np.random.default_rng(507)
    B, IN, H1 = 3, 12, 7
    x = rng.standard_normal((B, IN))
    w1 = rng.standard_normal((H1, IN)) * 0.5
    b1 = rng.standard_normal(H1) * 0.1
    w2 = rng.standard_normal((2, H1)) * 0.5
    b2 = rng.standard_normal(2) * 0.1
    g = rng.standard_normal((B, 2))
    tau = 0.7
    of = rng.standard_normal((B, 5, 2))
    osp = rng.standard_normal((B, 5, 2))
    dy = rng.standard_normal((B, 5, 2))

    def loss(x, w1, b1, w2, b2):
        lg = oracle.router_mlp(x, w1, b1, w2, b2)
        r = oracle.router_soft(lg, g, tau)
        return float((dy * oracle.soft_mix(of, osp, r)).sum())

    out = oracle.soft_routed_backward(x, w1, b1, w2, b2, g, tau, of, osp, dy)
    args = [x, w1, b1, w2, b2]
    eps = 1e-6
    for i, name in enumerate(["dx", "dw1", "db1", "dw2", "db2"]):
        for idx in np.ndindex(*args[i].shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[i][idx] += eps
            minus[i][idx] -= eps
            fd = (loss(*plus) - loss(*minus)) / (2 * eps)
            assert abs(fd - out[name][idx]) < 1e-7, (name, idx, fd, out[name][idx])
    # The two attention paths receive r dy and (1 - r) dy: the mix is linear.
    r = out["r"]
    np.testing.assert_allclose(out["dr"], (dy * (of - osp)).sum(axis=(1, 2)), atol=1e-12)
    assert np.all((r > 0) & (r < 1))
