"""GPU: the give-up path of the kernels' bounded waits.  In the testing mode
of fa_debug_set_wait_limit_ns(0) the kernels issue no TMA loads, so their
waits on loads run out (after 1 ms): the kernel reports FA_DEV_TIMEOUT in the
status word, lets what it has in flight finish, frees its tensor memory and
returns.  The call then ends normally, and the next call with the default
bound on the same stream gives the oracle's result: the device stayed
usable."""
import contextlib
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import assert_close_attention, assert_close_grad, to_f64, zero_status

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)
DEFAULT_NS = 2_000_000_000


@contextlib.contextmanager
def waits_bounded_by(ns):
    torch.cuda.synchronize()
    capi.debug_set_wait_limit_ns(ns)
    try:
        yield
    finally:
        torch.cuda.synchronize()
        capi.debug_set_wait_limit_ns(DEFAULT_NS)


def _gave_up(status):
    return (int(status.item()) & capi.FA_DEV_TIMEOUT) != 0


@pytest.mark.parametrize("Hq,Hkv", [(3, 3), (4, 1)])     # one-tile and two-tile kernels
@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_prefill_gives_up_then_runs_normally(Hq, Hkv, mode):
    S = 1024
    q, k, v = inputs.qkv(1, S, Hq, Hkv, 128, seed=961)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    c = capi.cfg(64, 128, 256)
    rp, ci = capi.blocksparse_index(S, c)

    def run(status):
        if mode == "full":
            return capi.attn_prefill_full(qd, kd, vd, status=status)
        return capi.attn_prefill_blocksparse(qd, kd, vd, rp, ci, status=status)

    st = zero_status()
    with waits_bounded_by(0):
        run(st)
    assert _gave_up(st)
    st = zero_status()
    o = run(st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    mask = (oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 128, 256))
            if mode == "sparse" else None)
    ref, _ = oracle.attention(inputs.bits(q), inputs.bits(k), inputs.bits(v), SCALE, mask)
    assert_close_attention(to_f64(o), ref, "prefill %s after a give-up" % mode)


def test_decode_gives_up_with_nan_heads_then_runs_normally():
    B, Lmax, Hq, Hkv = 2, 4096, 8, 2
    seqlens = np.array([4096, 3000], np.int32)
    q, kc, vc = inputs.decode_inputs(B, Lmax, Hq, Hkv, 128, 971)
    qd, kd, vd = q.cuda(), kc.cuda(), vc.cuda()
    sl = torch.from_numpy(seqlens).cuda()
    c = capi.cfg(64, 128, 1024)
    ref, _ = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), seqlens, SCALE,
                           capi.FA_MODE_FULL, 64, 128, 1024)
    st = zero_status()
    with waits_bounded_by(0):
        o = capi.attn_decode(qd, kd, vd, sl, capi.FA_MODE_FULL, c, status=st)
    assert _gave_up(st)
    got = to_f64(o)
    # A head whose splits all finished is exact; one with a split that gave up is NaN.
    nan_heads = np.isnan(got).all(axis=-1)
    assert nan_heads.any()
    assert not np.isnan(got[~nan_heads]).any()
    if (~nan_heads).any():
        assert np.abs(got[~nan_heads] - ref[~nan_heads]).max() <= 2e-2
    st = zero_status()
    o = capi.attn_decode(qd, kd, vd, sl, capi.FA_MODE_FULL, c, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close_attention(to_f64(o), ref, "decode after a give-up")


def test_backward_gives_up_then_runs_normally():
    B, S, Hq, Hkv = 1, 640, 4, 2
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, 981, device="cuda")
    do = inputs.randn_bf16((B, S, Hq, 128), 982, device="cuda")
    lse = torch.empty(B, Hq, S, device="cuda")
    st = zero_status()
    o = capi.attn_prefill_full(q, k, v, lse=lse, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    with waits_bounded_by(0):
        capi.attn_prefill_backward(q, k, v, o, lse, do, status=st)
    assert _gave_up(st)
    st = zero_status()
    dq, dk, dv = capi.attn_prefill_backward(q, k, v, o, lse, do, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    want = oracle.attention_backward(inputs.bits(q), inputs.bits(k), inputs.bits(v),
                                     inputs.bits(do), SCALE)
    for name, g, w in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        assert_close_grad(to_f64(g), w, "backward after a give-up: %s" % name)
