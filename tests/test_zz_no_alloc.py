"""fa_attn_decode_noalloc -- decode for callers that cannot allocate device
memory where they run it (no workspace argument in their interface, all
memory reserved up front, or no cudaMalloc allowed in their loop).  It must
give the same results as fa_attn_decode, whose workspace the caller
allocates, with its scratch in the library's static device array instead:
the oracle's result within the parity tolerance, and bit for bit the
result of fa_attn_decode (the same kernels with the same split count).

The file sorts last so that a run that stops at the first failure has run
every other test before this one.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import build, capi, inputs
from tests.gpu_util import LSE_ABS_TOL, assert_close_attention, to_f64, zero_status

SCALE = 1 / math.sqrt(128)


def test_noalloc_checks_arguments_like_decode_then_the_scratch_size():
    build.build()
    L = capi.lib()
    cap = L.fa_noalloc_scratch_bytes()
    assert cap == 8 << 20
    p = ctypes.c_void_p(4096)            # aligned, never dereferenced
    c = capi.cfg(64, 128, 2048)
    # Beyond the static scratch: FA_ERR_UNSUPPORTED, nothing launched.
    B, Hq, Hkv, Lmax = 512, 64, 8, 1 << 16
    assert L.fa_decode_workspace_size(B, Hq, Hkv, Lmax, 128) > cap
    assert L.fa_attn_decode_noalloc(p, p, p, p, B, Lmax, Hq, Hkv, 128, 0.1, 0, None, c, p, None,
                                    None, None) == -2
    # The same argument errors as fa_attn_decode, checked before the size.
    for args, want in (((None, p, p, p, B, Lmax, Hq, Hkv, 128), -1),     # null q
                       ((p, p, p, p, 2, 64, 4, 4, 64), -2),              # D != 128
                       ((p, p, p, p, B, Lmax, Hq, 7, 128), -1),          # Hq % Hkv
                       ((p, p, p, p, 2, 64, 32, 2, 128), -2)):           # G = 16
        rc_dec = L.fa_attn_decode(*args, 0.1, 0, None, c, p, None, p, 1 << 30, None, None)
        rc = L.fa_attn_decode_noalloc(*args, 0.1, 0, None, c, p, None, None, None)
        assert rc == rc_dec == want, (args, rc, rc_dec)


def _case(B, Lmax, Hq, Hkv, seqlens, mode, window, seed):
    q, kc, vc = inputs.decode_inputs(B, Lmax, Hq, Hkv, 128, seed)
    sl = np.array(seqlens, np.int32)
    ref, ref_lse = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), sl, SCALE,
                                 mode, 64, 128, window)
    dev = torch.device("cuda")
    return (q.to(dev), kc.to(dev), vc.to(dev), torch.from_numpy(sl).to(dev),
            capi.cfg(64, 128, window), ref, ref_lse)


@pytest.mark.gpu
def test_noalloc_matches_decode_and_the_oracle_on_two_calls_in_a_row():
    build.build()
    calls = [  # (B, Lmax, Hq, Hkv, seqlens, mode, window, seed): the second call is smaller,
               # so partials of the first left in the scratch would show up in its result
        (4, 8192, 32, 8, [8192, 5000, 64, 1], capi.FA_MODE_FULL, 1024, 71),
        (2, 3000, 16, 4, [3000, 1999], capi.FA_MODE_SPARSE, 512, 72),
    ]
    for B, Lmax, Hq, Hkv, seqlens, mode, window, seed in calls:
        q, kc, vc, sl, c, ref, ref_lse = _case(B, Lmax, Hq, Hkv, seqlens, mode, window, seed)
        st_ref, st_new = zero_status(), zero_status()
        lse_ref = torch.empty(B, Hq, device="cuda")
        lse_new = torch.empty(B, Hq, device="cuda")
        got = capi.attn_decode_noalloc(q, kc, vc, sl, mode, c, lse=lse_new, status=st_new)
        want = capi.attn_decode(q, kc, vc, sl, mode, c, lse=lse_ref, status=st_ref)
        torch.cuda.synchronize()
        assert int(st_ref.item()) == 0 and int(st_new.item()) == 0
        assert_close_attention(to_f64(got), ref, "noalloc vs oracle")
        np.testing.assert_allclose(to_f64(lse_new), ref_lse, atol=LSE_ABS_TOL)
        assert torch.equal(got, want)
        assert torch.equal(lse_new, lse_ref)


@pytest.mark.gpu
def test_noalloc_never_returns_an_earlier_calls_result_after_a_give_up():
    """A good call fills the scratch; then a call on other inputs in the
    testing mode of the bounded waits gives up: its heads read NaN or this
    call's own result, never the earlier call's."""
    build.build()
    B, Lmax, Hq, Hkv = 2, 4096, 8, 2
    a = _case(B, Lmax, Hq, Hkv, [4096, 4000], capi.FA_MODE_FULL, 1024, 73)
    b = _case(B, Lmax, Hq, Hkv, [4096, 4000], capi.FA_MODE_FULL, 1024, 74)
    st = zero_status()
    first = capi.attn_decode_noalloc(*a[:4], capi.FA_MODE_FULL, a[4], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    first = to_f64(first)
    torch.cuda.synchronize()
    capi.debug_set_wait_limit_ns(0)
    try:
        got = capi.attn_decode_noalloc(*b[:4], capi.FA_MODE_FULL, b[4], status=st)
        torch.cuda.synchronize()
    finally:
        capi.debug_set_wait_limit_ns(2_000_000_000)
    assert int(st.item()) & capi.FA_DEV_TIMEOUT
    got = to_f64(got)
    nan_heads = np.isnan(got).all(axis=-1)
    assert nan_heads.any() and not np.isnan(got[~nan_heads]).any()
    assert np.abs(got[~nan_heads] - b[5][~nan_heads]).max(initial=0.0) <= 2e-2
    assert not np.any(np.all(np.abs(got - first) < 1e-6, axis=-1))
    # The next call with the default bound is whole again.
    st = zero_status()
    again = capi.attn_decode_noalloc(*b[:4], capi.FA_MODE_FULL, b[4], status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert_close_attention(to_f64(again), b[5], "noalloc after a give-up")
