"""GPU: parity at the workloads' full sizes, in the launch configuration the
benchmark times, on seeded sampled rows the oracle computes one by one (each
output row depends only on its own query row and the keys it may attend)."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import LSE_ABS_TOL, assert_close_attention, to_f64, zero_status

pytestmark = pytest.mark.gpu
W = inputs.WORKLOADS


def _prefill_sampled(wl, mode, n_random, n_groups=2, full_rows_cap=None):
    B, S, Hq, Hkv = wl.B, wl.S, wl.Hq, wl.Hkv
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, wl.seed, device="cuda")
    lse = torch.empty(B, Hq, S, device="cuda", dtype=torch.float32)
    status = zero_status()
    c = capi.cfg(64, wl.sink, wl.window)
    if mode == "full":
        o = capi.attn_prefill_full(q, k, v, lse=lse, status=status)
        mask = None
    else:
        rp, ci = capi.blocksparse_index(S, c)
        o = capi.attn_prefill_blocksparse(q, k, v, rp, ci, lse=lse, status=status)
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, wl.sink, wl.window))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = inputs.sample_rows(B, S, Hq, Hkv, seed=wl.seed, n_random=n_random, n_groups=n_groups)
    if full_rows_cap is not None and mode == "full":
        rng = np.random.default_rng(wl.seed)
        keep = rng.choice(len(rows), size=min(full_rows_cap, len(rows)), replace=False)
        rows = rows[np.sort(keep)]
    ref, ref_lse = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v),
                                         1 / math.sqrt(128), rows, mask)
    rt = torch.from_numpy(rows).cuda()
    got = o[rt[:, 0], rt[:, 2], rt[:, 1]]
    got_lse = lse[rt[:, 0], rt[:, 1], rt[:, 2]]
    assert_close_attention(to_f64(got), ref, "%s %s" % (wl.name, mode))
    np.testing.assert_allclose(to_f64(got_lse), ref_lse, atol=LSE_ABS_TOL)


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_qwen3_4b_layer_s8192(mode):
    _prefill_sampled(W["qwen3-4b-layer-s8192"], mode, n_random=256)


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_llama_layer_s32768(mode):
    _prefill_sampled(W["llama3.1-8b-32l-s32768"], mode, n_random=128, full_rows_cap=600)


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_qwen3_8b_layer_s262144(mode):
    _prefill_sampled(W["qwen3-8b-layer-s262144"], mode, n_random=64, n_groups=1,
                     full_rows_cap=120)


def test_llama_32_layer_router_decisions():
    """32 layers, per-layer Q and router; b2 biases a seeded half of the
    layers to SPARSE.  Decisions match the oracle exactly."""
    wl = W["llama3.1-8b-32l-s32768"]
    rng = np.random.default_rng(wl.seed)
    sparse_layers = set(rng.choice(wl.layers, size=wl.layers // 2, replace=False).tolist())
    got, want = [], []
    for layer in range(wl.layers):
        bias = (0.0, 0.1) if layer in sparse_layers else (0.1, 0.0)
        q = inputs.randn_bf16((1, wl.S, wl.Hq, 128), wl.seed + 1000 * layer, device="cuda")
        w1, b1, w2, b2 = inputs.router_weights(wl.Hq * 128, wl.hidden, wl.seed, layer, b2=bias)
        logits, mode = capi.router_decide(q, w1.cuda(), b1.cuda(), w2.cuda(), b2.cuda())
        ref_logits, ref_mode, _ = oracle.router_decide(inputs.bits(q), w1.double().numpy(),
                                                       b1.double().numpy(), w2.double().numpy(),
                                                       b2.double().numpy())
        np.testing.assert_allclose(logits.cpu().double().numpy(), ref_logits, atol=1e-5)
        got.append(int(mode.item()))
        want.append(int(ref_mode[0]))
    assert got == want
    assert sum(got) == wl.layers // 2


@pytest.mark.parametrize("mode", [capi.FA_MODE_FULL, capi.FA_MODE_SPARSE])
def test_decode_b8_l131072(mode):
    wl = W["decode-b8-l131072-32l"]
    B, L, Hq, Hkv = wl.B, wl.decode_len, wl.Hq, wl.Hkv
    q, kc, vc = inputs.decode_inputs(B, L, Hq, Hkv, 128, wl.seed, device="cuda")
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    lse = torch.empty(B, Hq, device="cuda", dtype=torch.float32)
    status = zero_status()
    o = capi.attn_decode(q, kc, vc, sl, mode, capi.cfg(64, wl.sink, wl.window), lse=lse,
                         status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    bs = list(range(B)) if mode == capi.FA_MODE_SPARSE else [0, B - 1]
    qb, kb, vb = inputs.bits(q), inputs.bits(kc[bs]), inputs.bits(vc[bs])
    ref, ref_lse = oracle.decode(qb[bs], kb, vb, np.full(len(bs), L, np.int32),
                                 1 / math.sqrt(128), mode, 64, wl.sink, wl.window)
    assert_close_attention(to_f64(o[bs]), ref, "decode mode=%d" % mode)
    np.testing.assert_allclose(to_f64(lse[bs]), ref_lse, atol=LSE_ABS_TOL)


def test_bench_step_qwen3_4b_routed_layers():
    """The benchmark's step at full size: CSR, two routed layers (router head
    bias -> FULL, -> SPARSE) reading the mode on the device, and one decode
    token per layer with the device-side mode; sampled rows vs the oracle."""
    wl = W["qwen3-4b-layer-s8192"]
    B, S, Hq, Hkv = wl.B, wl.S, wl.Hq, wl.Hkv
    c = capi.cfg(64, wl.sink, wl.window)
    rp, ci = capi.blocksparse_index(S, c)
    mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, wl.sink, wl.window))
    rows = inputs.sample_rows(B, S, Hq, Hkv, seed=wl.seed + 5, n_random=128, n_groups=1)
    rt = torch.from_numpy(rows).cuda()
    for li, (bias, want) in enumerate((((0.1, 0.0), 0), ((0.0, 0.1), 1))):
        q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, wl.seed + 7919 * li, device="cuda")
        w1, b1, w2, b2 = inputs.router_weights(Hq * 128, wl.hidden, wl.seed, li, b2=bias)
        status = zero_status()
        o, logits, mode = capi.hybrid_layer(q, k, v, w1.cuda(), b1.cuda(), w2.cuda(), b2.cuda(),
                                            rp, ci, c, status=status)
        qd = inputs.randn_bf16((B, Hq, 128), wl.seed + 31 * li + 5, device="cuda")
        sl = torch.full((B,), S, dtype=torch.int32, device="cuda")
        od = capi.attn_decode(qd, k, v, sl, mode_dev=mode, c=c, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0 and int(mode.item()) == want
        qb, kb, vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
        ref, _ = oracle.attention_rows(qb, kb, vb, 1 / math.sqrt(128), rows,
                                       mask if want == 1 else None)
        assert_close_attention(to_f64(o[rt[:, 0], rt[:, 2], rt[:, 1]]), ref, "routed layer %d" % li)
        ref_d, _ = oracle.decode(inputs.bits(qd), kb, vb, np.full(B, S, np.int32),
                                 1 / math.sqrt(128), want, 64, wl.sink, wl.window)
        assert_close_attention(to_f64(od), ref_d, "decode layer %d" % li)
