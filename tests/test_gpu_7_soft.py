"""GPU: soft-routing forward ('Flux Attention', training-time relaxation):
r = Gumbel-softmax weight of the full path, y = r O_FA + (1 - r) O_SA, with
the mix fused into the sparse launch's epilogue; against the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import assert_close_attention, to_f64, zero_status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("tau", [0.05, 1.0, 7.0])
def test_router_soft_matches_oracle(tau):
    rng = np.random.default_rng(3)
    logits = rng.normal(size=(64, 2)).astype(np.float32)
    g = inputs.gumbel(64, seed=9)
    r = capi.router_soft(torch.from_numpy(logits).cuda(), g.cuda(), tau)
    torch.cuda.synchronize()
    want = oracle.router_soft(logits.astype(np.float64), g.double().numpy(), tau)
    np.testing.assert_allclose(r.cpu().numpy(), want, atol=2e-6, rtol=1e-5)


@pytest.mark.parametrize("B,S,Hq,Hkv,W", [(1, 1024, 4, 4, 128), (2, 1024, 8, 2, 256),
                                          (1, 777, 4, 2, 192)])
def test_soft_routed_layer_matches_oracle(B, S, Hq, Hkv, W):
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, seed=81 + S)
    w1, b1, w2, b2 = inputs.router_weights(Hq * 128, 64, seed=81)
    g = inputs.gumbel(B, seed=82)
    tau = 4.0   # keeps both paths weighted for these noise draws
    c = capi.cfg(64, 128, W)
    rp, ci = capi.blocksparse_index(S, c)
    status = zero_status()
    y, logits, r = capi.soft_routed_layer(q.cuda(), k.cuda(), v.cuda(), w1.cuda(), b1.cuda(),
                                          w2.cuda(), b2.cuda(), rp, ci, c, gumbel=g.cuda(),
                                          tau=tau, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    qb, kb, vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
    ref_logits, _, _ = oracle.router_decide(qb, w1.double().numpy(), b1.double().numpy(),
                                            w2.double().numpy(), b2.double().numpy())
    ref_r = oracle.router_soft(ref_logits, g.double().numpy(), tau)
    np.testing.assert_allclose(r.cpu().double().numpy(), ref_r, atol=1e-5)
    assert np.all((ref_r > 0.05) & (ref_r < 0.95)), "both paths must carry weight"
    scale = 1 / math.sqrt(128)
    mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 128, W))
    o_full, _ = oracle.attention(qb, kb, vb, scale)
    o_sparse, _ = oracle.attention(qb, kb, vb, scale, mask)
    ref = oracle.soft_mix(o_full, o_sparse, ref_r)
    assert_close_attention(to_f64(y), ref, "soft routed layer")
    # the mix is not either endpoint
    assert np.abs(to_f64(y) - o_full).max() > 1e-2 and np.abs(to_f64(y) - o_sparse).max() > 1e-2


def test_soft_mix_matches_oracle():
    """fa_soft_mix against the oracle's mix of the same bf16 outputs."""
    of = inputs.randn_bf16((3, 200, 4, 128), 851, device="cuda")
    osp = inputs.randn_bf16((3, 200, 4, 128), 852, device="cuda")
    r = torch.tensor([0.1, 0.5, 0.93], device="cuda")
    y = capi.soft_mix(of, osp, r)
    torch.cuda.synchronize()
    want = oracle.soft_mix(oracle.bf16_bits_to_f64(inputs.bits(of)),
                           oracle.bf16_bits_to_f64(inputs.bits(osp)), r.cpu().double().numpy())
    got = y.float().cpu().double().numpy()
    # one bf16 rounding of the fp32 result: half an ulp, relative 2^-9
    assert np.all(np.abs(got - want) <= np.abs(want) * 2.0 ** -8 + 1e-6)
