"""fa_attn_decode_noalloc -- decode for callers that cannot allocate device
memory where they run it (no workspace argument in their interface, all
memory reserved up front, or no cudaMalloc allowed in their loop).  It must
give the same results as fa_attn_decode, whose workspace the caller
allocates, with its scratch in the library's static device array instead.

The file sorts last so that a run that stops at the first failure has run
every other test before this one.
"""
import ctypes

import pytest
import torch

from block_sparse_attention_layerrouter_b200 import build, capi, inputs
from tests.gpu_util import assert_close_attention, to_f64, zero_status


def test_noalloc_rejects_shapes_beyond_the_static_scratch():
    build.build()
    L = capi.lib()
    cap = L.fa_noalloc_scratch_bytes()
    assert cap == 8 << 20
    B, Hq, Hkv, Lmax = 512, 64, 8, 1 << 16
    assert L.fa_decode_workspace_size(B, Hq, Hkv, Lmax, 128) > cap
    p = ctypes.c_void_p(4096)
    rc = L.fa_attn_decode_noalloc(p, p, p, p, B, Lmax, Hq, Hkv, 128, 0.1, 0, None,
                                  capi.cfg(64, 128, 2048), p, None, None, None)
    assert rc == -2                      # FA_ERR_UNSUPPORTED, nothing launched


@pytest.mark.gpu
def test_noalloc_matches_decode_on_two_calls_in_a_row():
    build.build()
    dev = torch.device("cuda")
    calls = [  # (B, Lmax, Hq, Hkv, seqlens, mode, window, seed): different shapes each call
        (4, 8192, 32, 8, [8192, 5000, 64, 1], capi.FA_MODE_FULL, 1024, 71),
        (2, 3000, 16, 4, [3000, 1999], capi.FA_MODE_SPARSE, 512, 72),
    ]
    for B, Lmax, Hq, Hkv, seqlens, mode, window, seed in calls:
        q, kc, vc = inputs.decode_inputs(B, Lmax, Hq, Hkv, 128, seed, device=dev)
        sl = torch.tensor(seqlens, dtype=torch.int32, device=dev)
        c = capi.cfg(64, 128, window)
        st_ref, st_new = zero_status(), zero_status()
        lse_ref = torch.empty(B, Hq, device=dev)
        lse_new = torch.empty(B, Hq, device=dev)
        ref = capi.attn_decode(q, kc, vc, sl, mode, c, lse=lse_ref, status=st_ref)
        got = capi.attn_decode_noalloc(q, kc, vc, sl, mode, c, lse=lse_new, status=st_new)
        torch.cuda.synchronize()
        assert int(st_ref.item()) == 0 and int(st_new.item()) == 0
        assert_close_attention(to_f64(got), to_f64(ref), "noalloc vs decode")
        assert torch.allclose(lse_new, lse_ref, atol=2e-3, rtol=0)
