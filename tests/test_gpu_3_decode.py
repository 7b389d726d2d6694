"""GPU: split-KV decode against the fp64 oracle, both modes, ragged lengths,
GQA groups 1/2/4/8, device-side modes, LSE."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import LSE_ABS_TOL, assert_close_attention, to_f64, zero_status

pytestmark = pytest.mark.gpu


def _decode_case(B, Lmax, Hq, Hkv, seqlens, mode, sink, window, seed, mode_dev=None, spikes=()):
    q, kc, vc = inputs.decode_inputs(B, Lmax, Hq, Hkv, 128, seed)
    G = Hq // Hkv
    for b, lo, hi, g, factor in spikes:   # keys lo..hi-1 of batch b pulled towards query head g
        kc[b, lo:hi, g // G] = (kc[b, lo:hi, g // G].float()
                                + factor * q[b, g].float()).to(torch.bfloat16)
    sl = torch.tensor(seqlens, dtype=torch.int32)
    status = zero_status()
    lse = torch.empty(B, Hq, device="cuda", dtype=torch.float32)
    c = capi.cfg(64, sink, window)
    md = None if mode_dev is None else torch.tensor(mode_dev, dtype=torch.int32, device="cuda")
    o = capi.attn_decode(q.cuda(), kc.cuda(), vc.cuda(), sl.cuda(), mode, c, mode_dev=md, lse=lse,
                         status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    scale = 1.0 / math.sqrt(128)
    qb, kb, vb = inputs.bits(q), inputs.bits(kc), inputs.bits(vc)
    modes = [mode] * B if mode_dev is None else mode_dev
    ref = np.zeros((B, Hq, 128))
    ref_lse = np.zeros((B, Hq))
    for b in range(B):
        o_b, l_b = oracle.decode(qb[b:b + 1], kb[b:b + 1], vb[b:b + 1], sl.numpy()[b:b + 1], scale,
                                 modes[b], 64, sink, window)
        ref[b], ref_lse[b] = o_b[0], l_b[0]
    assert_close_attention(to_f64(o), ref, "decode")
    np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL)


@pytest.mark.parametrize("mode", [capi.FA_MODE_FULL, capi.FA_MODE_SPARSE])
@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (4, 4), (8, 4), (16, 2)])
def test_decode_small(mode, Hq, Hkv):
    _decode_case(3, 1000, Hq, Hkv, [1000, 513, 64], mode, 128, 256, seed=21)


@pytest.mark.parametrize("seqlens", [[1, 2], [63, 65], [129, 4096]])
def test_decode_edge_lengths(seqlens):
    for mode in (capi.FA_MODE_FULL, capi.FA_MODE_SPARSE):
        _decode_case(2, 4096, 8, 2, seqlens, mode, 128, 192, seed=22)


def test_decode_device_modes():
    _decode_case(4, 3000, 32, 8, [3000, 2999, 1500, 200], capi.FA_MODE_FULL, 128, 512, seed=23,
                 mode_dev=[1, 0, 1, 0])


def test_decode_sparse_reads_only_its_blocks():
    """Overwrite V in every KV block outside the sink + window pattern with a
    large value: the sparse result is bit-identical to the clean one, the
    full one (which must read those blocks) moves far away."""
    B, Lmax, Hq, Hkv = 1, 2048, 8, 2
    q, kc, vc = inputs.decode_inputs(B, Lmax, Hq, Hkv, 128, 24)
    q, kc, vc = q.cuda(), kc.cuda(), vc.cuda()
    sl = torch.tensor([Lmax], dtype=torch.int32, device="cuda")
    c = capi.cfg(64, 128, 256)
    clean = capi.attn_decode(q, kc, vc, sl, capi.FA_MODE_SPARSE, c)
    clean_full = capi.attn_decode(q, kc, vc, sl, capi.FA_MODE_FULL, c)
    vp = vc.clone()
    vp[:, 128:Lmax - 256] = 1000.0
    dirty = capi.attn_decode(q, kc, vp, sl, capi.FA_MODE_SPARSE, c)
    full = capi.attn_decode(q, kc, vp, sl, capi.FA_MODE_FULL, c)
    torch.cuda.synchronize()
    assert torch.equal(clean, dirty)
    assert (full.float() - clean_full.float()).abs().max() > 100.0


@pytest.mark.parametrize("mode", [capi.FA_MODE_FULL, capi.FA_MODE_SPARSE])
def test_decode_rising_score_plateaus(mode):
    """Runs of keys pulled towards one query head so that their scores sit
    about 26 and then 45 (log2 units) above the rest, starting in the middle
    of a split and lasting to the end, plus one sink key at about 33: the
    splits meet scores far above what they have seen on later tiles, not only
    the first, and every key after the jump still carries weight; the other
    heads of the group see moderately raised scores.  Against the oracle."""
    L = 3000
    plateaus = [(0, 700, L, 1, 1.6), (0, 2050, L, 1, 1.2),       # 1.6, then 2.8 in all
                (1, 140, L, 6, 1.6), (1, 5, 6, 6, 2.0)]
    _decode_case(2, L, 8, 2, [L, L - 74], mode, 128, 512, seed=24, spikes=plateaus)
