"""GPU: decode over a paged KV cache (bf16 and FP8 E4M3) and the KV append,
against the oracle; paged equals contiguous bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import LSE_ABS_TOL, assert_close_attention, to_f64, zero_status

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)


def _pool(B, max_pages, Hkv, seed, extra_pages=3):
    """A page pool holding B sequences' pages in a seeded random order, plus
    spare pages, and the block table."""
    num_pages = B * max_pages + extra_pages
    rng = np.random.default_rng(seed)
    perm = rng.permutation(num_pages)[:B * max_pages].reshape(B, max_pages).astype(np.int32)
    kp = inputs.randn_bf16((num_pages, 64, Hkv, 128), seed + 100)
    vp = inputs.randn_bf16((num_pages, 64, Hkv, 128), seed + 200)
    return kp, vp, perm


def _fp8_scales(Hkv, seed):
    rng = np.random.default_rng(seed)
    return (rng.uniform(1 / 48, 1 / 24, size=Hkv).astype(np.float32),
            rng.uniform(1 / 48, 1 / 24, size=Hkv).astype(np.float32))


def _quantize_pool(pool_bits, s):
    codes = oracle.kv_quantize(pool_bits, s)          # [num_pages, 64, Hkv, D] uint8
    return torch.from_numpy(codes.copy())


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("fp8", [False, True])
def test_paged_decode_matches_oracle(mode, fp8):
    B, Hq, Hkv, max_pages = 3, 8, 2, 5
    seqlens = np.array([300, 65, 1], np.int32)
    kp, vp, bt = _pool(B, max_pages, Hkv, seed=701)
    q = inputs.randn_bf16((B, Hq, 128), 702)
    c = capi.cfg(64, 64, 128)
    status = zero_status()
    lse = torch.empty(B, Hq, device="cuda")
    if fp8:
        ks, vs = _fp8_scales(Hkv, 703)
        kc, vc = _quantize_pool(inputs.bits(kp), ks), _quantize_pool(inputs.bits(vp), vs)
        kval = oracle.e4m3_decode(kc.numpy()) * ks[None, None, :, None]
        vval = oracle.e4m3_decode(vc.numpy()) * vs[None, None, :, None]
        o = capi.attn_decode_paged(q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(bt).cuda(),
                                   torch.from_numpy(seqlens).cuda(), capi.FA_KV_FP8_E4M3,
                                   torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(),
                                   mode=mode, c=c, lse=lse, status=status)
    else:
        kval = oracle.bf16_bits_to_f64(inputs.bits(kp))
        vval = oracle.bf16_bits_to_f64(inputs.bits(vp))
        o = capi.attn_decode_paged(q.cuda(), kp.cuda(), vp.cuda(), torch.from_numpy(bt).cuda(),
                                   torch.from_numpy(seqlens).cuda(), mode=mode, c=c, lse=lse,
                                   status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kg = oracle.paged_gather(kval, bt, seqlens)
    vg = oracle.paged_gather(vval, bt, seqlens)
    ref, ref_lse = oracle.decode_values(oracle.bf16_bits_to_f64(inputs.bits(q)), kg, vg, seqlens,
                                        SCALE, mode=mode, sink=64, window=128)
    assert_close_attention(to_f64(o), ref, "paged fp8=%s mode=%d" % (fp8, mode))
    np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL)


def test_paged_equals_contiguous_bitwise():
    """A contiguous cache read through the identity block table gives the
    same bits as the contiguous decode."""
    B, Hq, Hkv, L = 2, 8, 2, 640
    q, kc, vc = inputs.decode_inputs(B, L, Hq, Hkv, 128, 711, device="cuda")
    sl = torch.tensor([640, 333], dtype=torch.int32, device="cuda")
    c = capi.cfg(64, 128, 256)
    bt = torch.arange(B * L // 64, dtype=torch.int32, device="cuda").reshape(B, L // 64)
    for mode in (0, 1):
        a = capi.attn_decode(q, kc, vc, sl, mode, c)
        b = capi.attn_decode_paged(q, kc.view(B * L // 64, 64, Hkv, 128),
                                   vc.view(B * L // 64, 64, Hkv, 128), bt, sl, mode=mode, c=c)
        torch.cuda.synchronize()
        assert torch.equal(a, b), "mode %d" % mode


@pytest.mark.parametrize("fp8", [False, True])
def test_kv_append_writes_the_token_and_advances(fp8):
    B, Hkv, max_pages = 3, 2, 3
    kp, vp, bt = _pool(B, max_pages, Hkv, seed=721)
    seqlens = np.array([0, 63, 191], np.int32)   # the last one fills its final slot
    k_new = inputs.randn_bf16((B, Hkv, 128), 722)
    v_new = inputs.randn_bf16((B, Hkv, 128), 723)
    ks, vs = _fp8_scales(Hkv, 724)
    if fp8:
        kpool = _quantize_pool(inputs.bits(kp), ks).cuda()
        vpool = _quantize_pool(inputs.bits(vp), vs).cuda()
    else:
        kpool, vpool = kp.cuda(), vp.cuda()
    before_k, before_v = kpool.clone(), vpool.clone()
    sl = torch.from_numpy(seqlens.copy()).cuda()
    status = zero_status()
    capi.kv_append_paged(k_new.cuda(), v_new.cuda(), kpool, vpool, torch.from_numpy(bt).cuda(), sl,
                         capi.FA_KV_FP8_E4M3 if fp8 else capi.FA_KV_BF16,
                         torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert sl.cpu().tolist() == (seqlens + 1).tolist()
    want_k, want_v = before_k.clone(), before_v.clone()
    for b, pos in enumerate(seqlens):
        page, slot = int(bt[b, pos // 64]), int(pos % 64)
        if fp8:
            want_k[page, slot] = torch.from_numpy(oracle.kv_quantize(inputs.bits(k_new[b]), ks))
            want_v[page, slot] = torch.from_numpy(oracle.kv_quantize(inputs.bits(v_new[b]), vs))
        else:
            want_k[page, slot] = k_new[b].cuda()
            want_v[page, slot] = v_new[b].cuda()
    assert torch.equal(kpool, want_k) and torch.equal(vpool, want_v)
    # The cache is full for sequence 2 now: its next append is refused.
    sl2 = torch.tensor([1, 64, 192], dtype=torch.int32, device="cuda")
    kpool2 = kpool.clone()
    capi.kv_append_paged(k_new.cuda(), v_new.cuda(), kpool2, vpool.clone(),
                         torch.from_numpy(bt).cuda(), sl2,
                         capi.FA_KV_FP8_E4M3 if fp8 else capi.FA_KV_BF16,
                         torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & 2                    # FA_DEV_BAD_INDEX
    assert sl2.cpu().tolist() == [2, 65, 192]


@pytest.mark.parametrize("mode", [0, 1])
def test_fp8_paged_decode_full_size(mode):
    """The decode workload's shape (B8, L 131072, 32/8 heads) with an FP8 paged
    cache, against the oracle on the dequantised values (sampled heads)."""
    wl = inputs.WORKLOADS["decode-b8-l131072-32l"]
    B, L, Hq, Hkv = wl.B, wl.decode_len, wl.Hq, wl.Hkv
    max_pages = L // 64
    num_pages = B * max_pages
    rng = np.random.default_rng(731)
    bt = rng.permutation(num_pages).reshape(B, max_pages).astype(np.int32)
    ks, vs = _fp8_scales(Hkv, 732)
    g = torch.Generator(device="cuda")
    g.manual_seed(733)

    def codes():   # seeded E4M3 codes with exponent field 4..10 (|x| in [1/8, 15])
        shape = (num_pages, 64, Hkv, 128)
        sign = torch.randint(0, 2, shape, generator=g, device="cuda", dtype=torch.int32)
        e = torch.randint(4, 11, shape, generator=g, device="cuda", dtype=torch.int32)
        m = torch.randint(0, 8, shape, generator=g, device="cuda", dtype=torch.int32)
        return ((sign << 7) | (e << 3) | m).to(torch.uint8)

    kc, vc = codes(), codes()
    q = inputs.randn_bf16((B, Hq, 128), 734, device="cuda")
    seqlens = np.array([L - 5 * b * 977 for b in range(B)], np.int32)
    c = capi.cfg(64, wl.sink, wl.window)
    status = zero_status()
    o = capi.attn_decode_paged(q, kc, vc, torch.from_numpy(bt).cuda(),
                               torch.from_numpy(seqlens).cuda(), capi.FA_KV_FP8_E4M3,
                               torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(), mode=mode,
                               c=c, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # Oracle on two sequences and one KV group (all of its query heads).
    kvh = int(rng.integers(0, Hkv))
    G = Hq // Hkv
    kcode, vcode = kc[:, :, kvh].cpu().numpy(), vc[:, :, kvh].cpu().numpy()
    for b in (0, B - 1):
        Lb = int(seqlens[b])
        kb = oracle.paged_gather(kcode[:, :, None], bt[b:b + 1], [Lb])[0, :Lb]
        vb = oracle.paged_gather(vcode[:, :, None], bt[b:b + 1], [Lb])[0, :Lb]
        kval = oracle.e4m3_decode(kb) * ks[kvh]
        vval = oracle.e4m3_decode(vb) * vs[kvh]
        qb = oracle.bf16_bits_to_f64(inputs.bits(q[b, kvh * G:(kvh + 1) * G]))
        ref, _ = oracle.decode_values(qb[None], kval[None], vval[None], [Lb], SCALE, mode=mode,
                                      sink=wl.sink, window=wl.window)
        got = to_f64(o[b, kvh * G:(kvh + 1) * G])
        assert_close_attention(got, ref[0], "fp8 full size b%d mode %d" % (b, mode))


def _fp8_case(B, Hq, Hkv, seqlens, mode, seed, q_scale=None, pull=()):
    """An FP8 paged decode against the oracle on the dequantised cache.
    q_scale [Hq]: per-head factors on the query (bf16 after scaling); pull:
    (b, lo, hi, head, factor) -- keys lo..hi-1 of sequence b get factor x that
    query head added before quantisation (scores far above the rest)."""
    max_pages = (max(seqlens) + 63) // 64
    kp, vp, bt = _pool(B, max_pages, Hkv, seed=seed)
    q = inputs.randn_bf16((B, Hq, 128), seed + 1)
    if q_scale is not None:
        q = (q.float() * torch.tensor(q_scale, dtype=torch.float32)[None, :, None]).to(torch.bfloat16)
    G = Hq // Hkv
    kf = kp.float()
    for b, lo, hi, head, factor in pull:
        t = np.arange(lo, hi)
        pages = torch.from_numpy(bt[b, t // 64].astype(np.int64))
        slots = torch.from_numpy(t % 64)
        kf[pages, slots, head // G] += factor * q[b, head].float()
    kp = kf.to(torch.bfloat16)
    ks, vs = _fp8_scales(Hkv, seed + 2)
    kc, vc = _quantize_pool(inputs.bits(kp), ks), _quantize_pool(inputs.bits(vp), vs)
    c = capi.cfg(64, 64, 256)
    status = zero_status()
    lse = torch.empty(B, Hq, device="cuda")
    sl = np.array(seqlens, np.int32)
    o = capi.attn_decode_paged(q.cuda(), kc.cuda(), vc.cuda(), torch.from_numpy(bt).cuda(),
                               torch.from_numpy(sl).cuda(), capi.FA_KV_FP8_E4M3,
                               torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(),
                               mode=mode, c=c, lse=lse, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    kval = oracle.e4m3_decode(kc.numpy()) * ks[None, None, :, None]
    vval = oracle.e4m3_decode(vc.numpy()) * vs[None, None, :, None]
    kg = oracle.paged_gather(kval, bt, sl)
    vg = oracle.paged_gather(vval, bt, sl)
    ref, ref_lse = oracle.decode_values(oracle.bf16_bits_to_f64(inputs.bits(q)), kg, vg, sl,
                                        SCALE, mode=mode, sink=64, window=256)
    what = "fp8 G=%d mode=%d" % (G, mode)
    assert_close_attention(to_f64(o), ref, what)
    np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL, err_msg=what)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("Hq,Hkv", [(8, 8), (8, 4), (8, 1)])
def test_fp8_decode_group_widths_and_query_ranges(mode, Hq, Hkv):
    """G = 1, 2, 8 with FP8 caches: the f16 products scale each query head by
    a power of two of its own; heads here span 1e-36 .. 300 in magnitude
    (1e-36: the scaling is capped so that it stays finite, and the head's
    scores are ~0 either way) and one is zero (its output is the mean of V)."""
    q_scale = [1e-3, 1e-36, 1.0, 300.0, 0.0, 7.0, 1.0 / 3.0, 40.0]
    _fp8_case(3, Hq, Hkv, [1000, 321, 64], mode, 741, q_scale=q_scale)


@pytest.mark.parametrize("mode", [0, 1])
def test_fp8_decode_rising_score_plateaus(mode):
    """FP8 cache: runs of keys pulled towards one query head so that their
    scores jump about 26 and then 45 (log2) above the rest in the middle of a
    split; every warp that meets them moves its reference and rescales.  The
    pulled values saturate E4M3 in places; both sides read the same codes."""
    L = 3000
    pull = [(0, 700, L, 1, 1.6), (0, 2050, L, 1, 1.2), (1, 140, L - 74, 6, 1.6),
            (1, 5, 6, 6, 2.0)]
    _fp8_case(2, 8, 2, [L, L - 74], mode, 751, pull=pull)
