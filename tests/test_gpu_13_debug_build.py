"""GPU: the debug build (libfa_hybrid_debug.so, -DFA_DEBUG=1), whose kernels
check the flattened index of every direct output store against the tensor's
element count (computed from the shape, apart from the index arithmetic) and
report FA_DEV_DEBUG_BOUNDS instead of storing.  On the paths with hand-written
index arithmetic -- both prefill kernels with ragged lengths, packed
variable-length batches, decode split partials with lengths below the cache's,
the backward with split key tiles -- no check may fire, and the results must
still be the oracle's."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import build, capi, inputs
from tests.gpu_util import (LSE_ABS_TOL, assert_close_attention, assert_close_grad, to_f64,
                            zero_status)

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)


@pytest.fixture(scope="module", autouse=True)
def debug_library():
    old = capi.use_library(build.build(debug=True))
    yield
    capi.use_library(old)


def _clean(status):
    torch.cuda.synchronize()
    v = int(status.item())
    assert v & capi.FA_DEV_DEBUG_BOUNDS == 0, "a debug bounds check fired (status %d)" % v
    assert v == 0, "device status %d" % v


@pytest.mark.parametrize("Hq,Hkv,S", [(4, 1, 1025), (3, 3, 255), (8, 2, 1536)])
@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_prefill_stores_in_bounds(Hq, Hkv, S, mode):
    B = 2
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, seed=1400 + S + Hq)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    lse = torch.empty(B, Hq, S, device="cuda")
    st = zero_status()
    c = capi.cfg(64, 128, 256)
    if mode == "full":
        o = capi.attn_prefill_full(qd, kd, vd, lse=lse, status=st)
        mask = None
    else:
        rp, ci = capi.blocksparse_index(S, c)
        o = capi.attn_prefill_blocksparse(qd, kd, vd, rp, ci, lse=lse, status=st)
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 128, 256))
    _clean(st)
    ref, ref_lse = oracle.attention(inputs.bits(q), inputs.bits(k), inputs.bits(v), SCALE, mask)
    assert_close_attention(to_f64(o), ref, "debug prefill %s" % mode)
    np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL)


def test_varlen_stores_in_bounds():
    lengths = [1, 64, 200, 1000, 129]
    T, Hq, Hkv = sum(lengths), 8, 2
    q, k, v = inputs.qkv(1, T, Hq, Hkv, 128, seed=1410)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")
    st = zero_status()
    lse = torch.empty(Hq, T, device="cuda")
    o = capi.attn_prefill_varlen(q[0].cuda(), k[0].cuda(), v[0].cuda(), cu, max(lengths), lse=lse,
                                 status=st)
    _clean(st)
    got = to_f64(o)
    for i, L in enumerate(lengths):
        a = int(cu[i].item())
        sl = slice(a, a + L)
        ref, _ = oracle.attention(inputs.bits(q[:, sl]), inputs.bits(k[:, sl]),
                                  inputs.bits(v[:, sl]), SCALE, None)
        assert_close_attention(got[sl][None], ref, "debug varlen sequence %d" % i)


@pytest.mark.parametrize("mode", [capi.FA_MODE_FULL, capi.FA_MODE_SPARSE])
def test_decode_partials_in_bounds(mode):
    B, Lmax, Hq, Hkv = 3, 5000, 16, 2
    seqlens = np.array([5000, 1, 3333], np.int32)
    q, kc, vc = inputs.decode_inputs(B, Lmax, Hq, Hkv, 128, 1420 + mode)
    c = capi.cfg(64, 128, 1024)
    st = zero_status()
    lse = torch.empty(B, Hq, device="cuda")
    o = capi.attn_decode(q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(seqlens).cuda(), mode, c,
                         lse=lse, status=st)
    _clean(st)
    ref, ref_lse = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), seqlens, SCALE,
                                 mode, 64, 128, 1024)
    assert_close_attention(to_f64(o), ref, "debug decode")
    np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL)


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_backward_gradient_stores_in_bounds(mode):
    """S = 4608 (72 query blocks): on the sparse path the sink tile (which
    every query block attends) is cut into chunks whose dK/dV go through the
    fp32 partial sums."""
    B, S, Hq, Hkv = 1, 4608, 4, 2
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, 1430, device="cuda")
    do = inputs.randn_bf16((B, S, Hq, 128), 1431, device="cuda")
    c = capi.cfg(64, 128, 512)
    rp, ci = capi.blocksparse_index(S, c)
    lse = torch.empty(B, Hq, S, device="cuda")
    st = zero_status()
    if mode == "full":
        o = capi.attn_prefill_full(q, k, v, lse=lse, status=st)
        dq, dk, dv = capi.attn_prefill_backward(q, k, v, o, lse, do, status=st)
        mask = None
    else:
        o = capi.attn_prefill_blocksparse(q, k, v, rp, ci, lse=lse, status=st)
        dq, dk, dv = capi.attn_prefill_backward(q, k, v, o, lse, do, rp, ci,
                                                mode=capi.FA_MODE_SPARSE, status=st)
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 128, 512))
    _clean(st)
    keys = np.array([0, 1, 63, 64, 127, 128, 2047, 2048, 4095, 4096, 4607], np.int64)
    for kvh in range(Hkv):
        want_dk, want_dv = oracle.attention_backward_keyrows(
            inputs.bits(q), inputs.bits(k), inputs.bits(v), inputs.bits(do), SCALE, 0, kvh, keys,
            mask)
        kt = torch.from_numpy(keys).cuda()
        assert_close_grad(to_f64(dk[0, kt, kvh]), want_dk, "debug %s dk kvh %d" % (mode, kvh))
        assert_close_grad(to_f64(dv[0, kt, kvh]), want_dv, "debug %s dv kvh %d" % (mode, kvh))
    rows = inputs.sample_rows(B, S, Hq, Hkv, seed=1432, n_random=24, n_groups=1)
    want_dq = oracle.attention_backward_qrows(inputs.bits(q), inputs.bits(k), inputs.bits(v),
                                              inputs.bits(do), SCALE, rows, mask)
    rt = torch.from_numpy(rows).cuda()
    assert_close_grad(to_f64(dq[rt[:, 0], rt[:, 2], rt[:, 1]]), want_dq, "debug %s dq" % mode)
