"""GPU: attention backward (dQ, dK, dV) against the oracle's chain-rule
gradients, full and block-sparse, GQA, ragged lengths, per-batch modes, and
sampled rows at the full Qwen3-4B layer size."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import assert_close_grad, to_f64, zero_status

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)


def _setup(B, S, Hq, Hkv, seed, cfg=None, modes=None):
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, seed, device="cuda")
    do = inputs.randn_bf16((B, S, Hq, 128), seed + 400, device="cuda")
    lse = torch.empty(B, Hq, S, device="cuda")
    status = zero_status()
    rp = ci = None
    if cfg is not None:
        rp, ci = capi.blocksparse_index(S, cfg)
    o = torch.empty_like(q)
    if modes is None:
        capi.attn_prefill_full(q, k, v, o=o, lse=lse, status=status)
    else:
        # Per-batch modes through the varlen-free routed path: one launch per mode.
        for b, m in enumerate(modes):
            sl = slice(b, b + 1)
            if m == 0:
                capi.attn_prefill_full(q[sl], k[sl], v[sl], o=o[sl], lse=lse[sl], status=status)
            else:
                capi.attn_prefill_blocksparse(q[sl], k[sl], v[sl], rp, ci, o=o[sl], lse=lse[sl],
                                              status=status)
    return q, k, v, do, o, lse, rp, ci, status


def _oracle_grads(q, k, v, do, mask):
    return oracle.attention_backward(inputs.bits(q), inputs.bits(k), inputs.bits(v),
                                     inputs.bits(do), SCALE, mask)


def _check_all(got, want, tag):
    for name, g, w in zip(("dq", "dk", "dv"), got, want):
        assert_close_grad(to_f64(g), w, "%s %s" % (tag, name))


@pytest.mark.parametrize("B,S,Hq,Hkv", [(2, 320, 8, 2), (1, 200, 2, 2), (1, 1024, 4, 1),
                                         (1, 2560, 2, 1)])
def test_backward_full(B, S, Hq, Hkv):
    q, k, v, do, o, lse, _, _, status = _setup(B, S, Hq, Hkv, seed=601 + S)
    # Attention of the full path: recompute the forward into o/lse first.
    capi.attn_prefill_full(q, k, v, o=o, lse=lse, status=status)
    dq, dk, dv = capi.attn_prefill_backward(q, k, v, o, lse, do, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    _check_all((dq, dk, dv), _oracle_grads(q, k, v, do, None), "full B%d S%d" % (B, S))


@pytest.mark.parametrize("B,S,Hq,Hkv,sink,window", [(2, 320, 8, 2, 64, 128),
                                                    (1, 1000, 4, 2, 128, 256),
                                                    (1, 640, 2, 1, 0, 64),
                                                    (1, 2560, 2, 1, 128, 256)])
def test_backward_sparse(B, S, Hq, Hkv, sink, window):
    c = capi.cfg(64, sink, window)
    q, k, v, do, o, lse, rp, ci, status = _setup(B, S, Hq, Hkv, seed=611 + S, cfg=c)
    capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o, lse=lse, status=status)
    dq, dk, dv = capi.attn_prefill_backward(q, k, v, o, lse, do, rp, ci, mode=1, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, sink, window))
    _check_all((dq, dk, dv), _oracle_grads(q, k, v, do, mask), "sparse S%d W%d" % (S, window))


def test_backward_per_batch_modes_on_device():
    B, S, Hq, Hkv, W = 2, 384, 4, 2, 128
    c = capi.cfg(64, 64, W)
    modes = [1, 0]
    q, k, v, do, o, lse, rp, ci, status = _setup(B, S, Hq, Hkv, seed=621, cfg=c, modes=modes)
    mode_dev = torch.tensor(modes, dtype=torch.int32, device="cuda")
    dq, dk, dv = capi.attn_prefill_backward(q, k, v, o, lse, do, rp, ci, mode_dev=mode_dev,
                                            status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 64, W))
    for b, m in enumerate(modes):
        sl = slice(b, b + 1)
        want = _oracle_grads(q[sl], k[sl], v[sl], do[sl], mask if m else None)
        _check_all((dq[sl], dk[sl], dv[sl]), want, "batch %d mode %d" % (b, m))


def test_backward_is_deterministic_in_dk_dv():
    """With no key tile split into chunks (S = 512: at most 32 query blocks
    per tile), dK/dV accumulate in one CTA's TMEM in a fixed order: repeat
    calls give identical bits (dQ is summed with reductions in varying
    order)."""
    q, k, v, do, o, lse, _, _, status = _setup(1, 512, 4, 2, seed=631)
    capi.attn_prefill_full(q, k, v, o=o, lse=lse, status=status)
    a = capi.attn_prefill_backward(q, k, v, o, lse, do, status=status)
    a = [t.clone() for t in a]
    b = capi.attn_prefill_backward(q, k, v, o, lse, do, status=status)
    torch.cuda.synchronize()
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert int(status.item()) == 0


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_backward_qwen3_4b_layer_sampled(mode):
    """Full Qwen3-4B layer (S = 8192, 32/8 heads): dQ on seeded sampled rows
    and dK/dV on seeded key rows of one KV head, against the oracle."""
    wl = inputs.WORKLOADS["qwen3-4b-layer-s8192"]
    S, Hq, Hkv = wl.S, wl.Hq, wl.Hkv
    c = capi.cfg(64, wl.sink, wl.window)
    q, k, v, do, o, lse, rp, ci, status = _setup(1, S, Hq, Hkv, seed=wl.seed, cfg=c)
    sparse = mode == "sparse"
    if sparse:
        capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o, lse=lse, status=status)
    dq, dk, dv = capi.attn_prefill_backward(q, k, v, o, lse, do, rp, ci, mode=int(sparse),
                                            status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    mask = (oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, wl.sink, wl.window))
            if sparse else None)
    qb, kb, vb, dob = (inputs.bits(t) for t in (q, k, v, do))
    rows = inputs.sample_rows(1, S, Hq, Hkv, seed=wl.seed + 7, n_random=48, n_boundary=4,
                              n_groups=1)
    rng = np.random.default_rng(wl.seed + 7)
    rows = rows[np.sort(rng.choice(len(rows), size=min(160, len(rows)), replace=False))]
    want_q = oracle.attention_backward_qrows(qb, kb, vb, dob, SCALE, rows, mask)
    rt = torch.from_numpy(rows).cuda()
    assert_close_grad(to_f64(dq[rt[:, 0], rt[:, 2], rt[:, 1]]), want_q, "%s dq rows" % mode)
    kvh = int(rng.integers(0, Hkv))
    keys = np.unique(np.concatenate([[0, 63, 64, 127, 128, S - 1, S - 64],
                                     rng.integers(0, S, size=9)])).astype(np.int64)
    want_k, want_v = oracle.attention_backward_keyrows(qb, kb, vb, dob, SCALE, 0, kvh, keys, mask)
    kt = torch.from_numpy(keys).cuda()
    assert_close_grad(to_f64(dk[0, kt, kvh]), want_k, "%s dk rows" % mode)
    assert_close_grad(to_f64(dv[0, kt, kvh]), want_v, "%s dv rows" % mode)


def test_soft_routed_layer_backward_matches_oracle():
    """Router weights and attention inputs' gradients through the soft-routed
    layer y = r O_FA + (1 - r) O_SA, against the oracle's chain rule."""
    B, S, Hq, Hkv, H1, W, tau = 2, 384, 4, 2, 32, 128, 1.5
    c = capi.cfg(64, 64, W)
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, 641, device="cuda")
    dy = inputs.randn_bf16((B, S, Hq, 128), 1041, device="cuda")
    rp, ci = capi.blocksparse_index(S, c)
    status = zero_status()
    lse_f = torch.empty(B, Hq, S, device="cuda")
    lse_s = torch.empty(B, Hq, S, device="cuda")
    o_f = capi.attn_prefill_full(q, k, v, lse=lse_f, status=status)
    o_s = capi.attn_prefill_blocksparse(q, k, v, rp, ci, lse=lse_s, status=status)
    w1, b1, w2, b2 = inputs.router_weights(Hq * 128, H1, 641, b2=(0.02, -0.01), std=0.05)
    g = inputs.gumbel(B, 641)
    out = capi.soft_routed_layer_backward(q, k, v, o_f, lse_f, o_s, lse_s, dy, w1.cuda(),
                                          b1.cuda(), w2.cuda(), b2.cuda(), rp, ci,
                                          gumbel=g.cuda(), tau=tau, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0

    qb, kb, vb, dyb = (inputs.bits(t) for t in (q, k, v, dy))
    mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 64, W))
    x = oracle.router_pool(qb)
    o_full, _ = oracle.attention(qb, kb, vb, SCALE)
    o_sparse, _ = oracle.attention(qb, kb, vb, SCALE, mask)
    rb = oracle.soft_routed_backward(x, w1.double().numpy(), b1.double().numpy(),
                                     w2.double().numpy(), b2.double().numpy(),
                                     g.double().numpy(), tau, o_full, o_sparse,
                                     oracle.bf16_bits_to_f64(dyb))
    np.testing.assert_allclose(out["r"].cpu().double().numpy(), rb["r"], atol=1e-5)
    for name in ("dw1", "db1", "dw2", "db2"):
        assert_close_grad(to_f64(out[name]), rb[name], "soft " + name)
    gf = oracle.attention_backward(qb, kb, vb, dyb, SCALE)
    gs = oracle.attention_backward(qb, kb, vb, dyb, SCALE, mask)
    r = rb["r"][:, None, None, None]
    want = [r * a + (1 - r) * b for a, b in zip(gf, gs)]
    want[0] = want[0] + oracle.router_pool_backward(rb["dx"], S, Hq, 128)
    for name, w in zip(("dq", "dk", "dv"), want):
        assert_close_grad(to_f64(out[name]), w, "soft " + name)
