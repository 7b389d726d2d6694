"""GPU: one routed layer (router on device -> mode read by the attention
kernel) equals the standalone call of the chosen path, bit for bit, and the
decision matches the oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import assert_close_attention, to_f64, zero_status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bias,want", [((0.0, 0.1), 1), ((0.1, 0.0), 0), ((0.0, 0.0), None)])
def test_hybrid_layer_routes_and_matches(bias, want):
    B, S, Hq, Hkv, W = 2, 1024, 8, 2, 256
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, seed=61)
    w1, b1, w2, b2 = inputs.router_weights(Hq * 128, 64, seed=61, b2=bias)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    c = capi.cfg(64, 128, W)
    rp, ci = capi.blocksparse_index(S, c)
    status = zero_status()
    o, logits, mode = capi.hybrid_layer(qd, kd, vd, w1.cuda(), b1.cuda(), w2.cuda(), b2.cuda(),
                                        rp, ci, c, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_logits, ref_mode, _ = oracle.router_decide(inputs.bits(q), w1.double().numpy(),
                                                   b1.double().numpy(), w2.double().numpy(),
                                                   b2.double().numpy())
    mode = mode.cpu().numpy()
    tie = np.abs(ref_logits[:, 0] - ref_logits[:, 1]) < 1e-3
    assert np.array_equal(mode[~tie], ref_mode[~tie])
    if want is not None:
        assert np.all(mode == want)
    full = capi.attn_prefill_full(qd, kd, vd)
    sparse = capi.attn_prefill_blocksparse(qd, kd, vd, rp, ci)
    torch.cuda.synchronize()
    for b in range(B):
        expect = sparse[b] if mode[b] == 1 else full[b]
        assert torch.equal(o[b], expect)
    mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 128, W))
    for b in range(B):
        ref, _ = oracle.attention(inputs.bits(q[b:b + 1]), inputs.bits(k[b:b + 1]),
                                  inputs.bits(v[b:b + 1]), 1 / math.sqrt(128),
                                  mask if mode[b] == 1 else None)
        assert_close_attention(to_f64(o[b:b + 1]), ref, "hybrid b=%d" % b)


def test_hybrid_layer_reports_a_csr_built_for_another_window():
    """The routed layer reads the CSR on the device only; one built for
    another window (a different entry count) is reported as
    FA_DEV_BAD_INDEX, and the one built for its own window is not."""
    B, S, Hq, Hkv = 1, 1024, 4, 2
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, seed=62)
    w1, b1, w2, b2 = [t.cuda() for t in inputs.router_weights(Hq * 128, 64, seed=62,
                                                               b2=(0.0, 0.1))]
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    c = capi.cfg(64, 128, 256)
    rp_own, ci_own = capi.blocksparse_index(S, c)
    rp_other, ci_other = capi.blocksparse_index(S, capi.cfg(64, 128, 512))
    st = zero_status()
    capi.hybrid_layer(qd, kd, vd, w1, b1, w2, b2, rp_own, ci_own, c, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    capi.hybrid_layer(qd, kd, vd, w1, b1, w2, b2, rp_other, ci_other, c, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) & capi.FA_DEV_BAD_INDEX
