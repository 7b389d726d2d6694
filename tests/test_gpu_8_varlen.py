"""GPU: packed variable-length batches (the serving form of the routed layer:
one launch, every sequence in its own mode) against the oracle per sequence,
and bit-for-bit against per-sequence fixed-length launches."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import LSE_ABS_TOL, assert_close_attention, to_f64, zero_status

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)


def _packed(lengths, Hq, Hkv, seed):
    T = int(sum(lengths))
    q = inputs.randn_bf16((T, Hq, 128), seed)
    k = inputs.randn_bf16((T, Hkv, 128), seed + 100)
    v = inputs.randn_bf16((T, Hkv, 128), seed + 200)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return q, k, v, cu


def _oracle_seq(q, k, v, cu, b, sparse, window):
    t0, t1 = int(cu[b]), int(cu[b + 1])
    L = t1 - t0
    mask = None
    if sparse:
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(L, 64, 128, window))
    return oracle.attention(inputs.bits(q[t0:t1][None]), inputs.bits(k[t0:t1][None]),
                            inputs.bits(v[t0:t1][None]), SCALE, mask)


@pytest.mark.parametrize("modes", [[0, 0, 0, 0, 0], [1, 1, 1, 1, 1], [1, 0, 1, 0, 1]])
def test_varlen_matches_oracle_per_sequence(modes):
    lengths = [1000, 64, 1, 0, 513]
    Hq, Hkv, W = 8, 2, 256
    q, k, v, cu = _packed(lengths, Hq, Hkv, seed=91)
    T, maxL = int(cu[-1]), max(lengths)
    c = capi.cfg(64, 128, W)
    rp, ci = capi.blocksparse_index(maxL, c)
    lse = torch.full((Hq, T), 7.0, device="cuda")
    status = zero_status()
    o = capi.attn_prefill_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu).cuda(), maxL,
                                 rp, ci, mode_dev=torch.tensor(modes, dtype=torch.int32).cuda(),
                                 lse=lse, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for b, L in enumerate(lengths):
        if L == 0:
            continue
        t0 = int(cu[b])
        ref, ref_lse = _oracle_seq(q, k, v, cu, b, modes[b] == 1, W)
        assert_close_attention(to_f64(o[t0:t0 + L]), ref[0], "varlen seq %d" % b)
        np.testing.assert_allclose(to_f64(lse[:, t0:t0 + L]), ref_lse[0], atol=LSE_ABS_TOL)


def test_varlen_equals_fixed_length_launches_bitwise():
    lengths = [700, 129, 2048, 64]
    Hq, Hkv = 16, 4
    q, k, v, cu = _packed(lengths, Hq, Hkv, seed=92)
    maxL = max(lengths)
    c = capi.cfg(64, 128, 512)
    rp, ci = capi.blocksparse_index(maxL, c)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    cud = torch.from_numpy(cu).cuda()
    for mode in (capi.FA_MODE_FULL, capi.FA_MODE_SPARSE):
        o = capi.attn_prefill_varlen(qd, kd, vd, cud, maxL, rp, ci, mode=mode)
        for b, L in enumerate(lengths):
            t0 = int(cu[b])
            sl = slice(t0, t0 + L)
            qs, ks, vs = qd[sl][None].contiguous(), kd[sl][None].contiguous(), vd[sl][None].contiguous()
            if mode == capi.FA_MODE_FULL:
                ref = capi.attn_prefill_full(qs, ks, vs)
            else:
                rpb, cib = capi.blocksparse_index(L, c)
                ref = capi.attn_prefill_blocksparse(qs, ks, vs, rpb, cib)
            torch.cuda.synchronize()
            assert torch.equal(o[sl], ref[0]), "sequence %d mode %d" % (b, mode)


def test_hybrid_layer_varlen_routes_each_sequence():
    lengths = [300, 1200, 256, 777]
    Hq, Hkv, W = 8, 2, 256
    q, k, v, cu = _packed(lengths, Hq, Hkv, seed=93)
    maxL = max(lengths)
    w1, b1, w2, b2 = inputs.router_weights(Hq * 128, 64, seed=93)
    c = capi.cfg(64, 128, W)
    rp, ci = capi.blocksparse_index(maxL, c)
    status = zero_status()
    o, logits, mode = capi.hybrid_layer_varlen(q.cuda(), k.cuda(), v.cuda(),
                                               torch.from_numpy(cu).cuda(), maxL, w1.cuda(),
                                               b1.cuda(), w2.cuda(), b2.cuda(), rp, ci, c,
                                               status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    mode = mode.cpu().numpy()
    for b, L in enumerate(lengths):
        t0 = int(cu[b])
        qb = inputs.bits(q[t0:t0 + L][None])
        ref_logits, ref_mode, _ = oracle.router_decide(qb, w1.double().numpy(), b1.double().numpy(),
                                                       w2.double().numpy(), b2.double().numpy())
        np.testing.assert_allclose(logits[b].cpu().double().numpy(), ref_logits[0], atol=1e-5)
        if abs(ref_logits[0, 0] - ref_logits[0, 1]) >= 1e-3:
            assert mode[b] == ref_mode[0]
        ref, _ = _oracle_seq(q, k, v, cu, b, mode[b] == 1, W)
        assert_close_attention(to_f64(o[t0:t0 + L]), ref[0], "hybrid varlen seq %d" % b)


def test_serving_varlen_full_size_sampled():
    """The packed serving batch at its full size (8 requests of seeded
    lengths up to 32768, Qwen3-4B heads), through the hybrid varlen entry in
    the benchmark's launch configuration: every routing decision matches the
    oracle's, and seeded sampled rows of each request match the oracle in the
    mode the router chose for that request."""
    wl = inputs.WORKLOADS["serving-varlen-qwen3-4b"]
    lengths = inputs.varlen_lengths(wl.B, wl.S, wl.seed)
    T = int(lengths.sum())
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    q = inputs.randn_bf16((T, wl.Hq, 128), wl.seed, device="cuda")
    k = inputs.randn_bf16((T, wl.Hkv, 128), wl.seed + 100, device="cuda")
    v = inputs.randn_bf16((T, wl.Hkv, 128), wl.seed + 200, device="cuda")
    w1, b1, w2, b2 = inputs.router_weights(wl.Hq * 128, wl.hidden, wl.seed)
    c = capi.cfg(64, wl.sink, wl.window)
    rp, ci = capi.blocksparse_index(wl.S, c)
    lse = torch.empty(wl.Hq, T, device="cuda")
    status = zero_status()
    o, logits, mode = capi.hybrid_layer_varlen(q, k, v, torch.from_numpy(cu).cuda(), wl.S,
                                               w1.cuda(), b1.cuda(), w2.cuda(), b2.cuda(), rp, ci,
                                               c, lse=lse, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    mode = mode.cpu().numpy()
    qh, kh, vh = q.cpu(), k.cpu(), v.cpu()
    for b, L in enumerate(lengths.tolist()):
        t0 = int(cu[b])
        qb = inputs.bits(qh[t0:t0 + L][None])
        ref_logits, ref_mode, _ = oracle.router_decide(qb, w1.double().numpy(), b1.double().numpy(),
                                                       w2.double().numpy(), b2.double().numpy())
        np.testing.assert_allclose(logits[b].cpu().double().numpy(), ref_logits[0], atol=1e-5)
        assert mode[b] == ref_mode[0], "request %d routed differently" % b
        rows = inputs.sample_rows(1, L, wl.Hq, wl.Hkv, seed=wl.seed + b, n_random=24,
                                  n_boundary=4, n_groups=1)
        if mode[b] == 0:
            rng = np.random.default_rng(wl.seed + b)
            rows = rows[np.sort(rng.choice(len(rows), size=min(96, len(rows)), replace=False))]
            mask = None
        else:
            mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(L, 64, wl.sink, wl.window))
        ref, ref_lse = oracle.attention_rows(qb, inputs.bits(kh[t0:t0 + L][None]),
                                             inputs.bits(vh[t0:t0 + L][None]), SCALE, rows, mask)
        rt = torch.from_numpy(rows).cuda()
        got = o[t0 + rt[:, 2], rt[:, 1]]
        got_lse = lse[rt[:, 1], t0 + rt[:, 2]]
        assert_close_attention(to_f64(got), ref, "serving request %d mode %d" % (b, mode[b]))
        np.testing.assert_allclose(to_f64(got_lse), ref_lse, atol=LSE_ABS_TOL)
