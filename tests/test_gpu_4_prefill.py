"""GPU: tcgen05 prefill (full and block-sparse) against the fp64 oracle at
sizes the oracle finishes in seconds, across several tiles, ragged tails and
GQA; invariants that hold at any size (all-ones mask == full, masked blocks
never read)."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import LSE_ABS_TOL, assert_close_attention, to_f64, zero_status

pytestmark = pytest.mark.gpu


def _run(q, k, v, mode, window=128, sink=128):
    B, S, Hq, _ = q.shape
    status = zero_status()
    lse = torch.empty(B, Hq, S, device="cuda", dtype=torch.float32)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    if mode == "full":
        o = capi.attn_prefill_full(qd, kd, vd, lse=lse, status=status)
    else:
        rp, ci = capi.blocksparse_index(S, capi.cfg(64, sink, window))
        o = capi.attn_prefill_blocksparse(qd, kd, vd, rp, ci, lse=lse, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return o, lse


def _oracle(q, k, v, mode, window=128, sink=128):
    S = q.shape[1]
    mask = None
    if mode == "sparse":
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, sink, window))
    return oracle.attention(inputs.bits(q), inputs.bits(k), inputs.bits(v), 1 / math.sqrt(128),
                            mask)


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_prefill_mha4_s1024(mode):
    """Single layer, batch 1, 4 MHA heads, S = 1024; window 128, 128 sinks."""
    q, k, v = inputs.qkv(1, 1024, 4, 4, 128, seed=1000)
    o, lse = _run(q, k, v, mode)
    ref, ref_lse = _oracle(q, k, v, mode)
    assert_close_attention(to_f64(o), ref, "prefill %s S=1024" % mode)
    np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL)


@pytest.mark.parametrize("S", [1, 64, 65, 127, 128, 129, 200, 255, 1000])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 1)])
def test_prefill_edge_shapes(S, Hq, Hkv):
    q, k, v = inputs.qkv(2, S, Hq, Hkv, 128, seed=31 + S)
    for mode in ("full", "sparse"):
        o, lse = _run(q, k, v, mode, window=128)
        ref, ref_lse = _oracle(q, k, v, mode, window=128)
        assert_close_attention(to_f64(o), ref, "prefill %s S=%d G=%d" % (mode, S, Hq // Hkv))
        np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL)


@pytest.mark.parametrize("window,sink", [(64, 0), (192, 64), (256, 128), (640, 256)])
def test_prefill_sparse_windows(window, sink):
    q, k, v = inputs.qkv(1, 1536, 4, 2, 128, seed=41 + window)
    o, _ = _run(q, k, v, "sparse", window=window, sink=sink)
    ref, _ = _oracle(q, k, v, "sparse", window=window, sink=sink)
    assert_close_attention(to_f64(o), ref, "sparse w=%d sink=%d" % (window, sink))


def test_all_ones_mask_equals_full_bitwise():
    q, k, v = inputs.qkv(1, 1536, 8, 2, 128, seed=51)
    full, lf = _run(q, k, v, "full")
    ones, lo = _run(q, k, v, "sparse", window=1536, sink=0)
    assert torch.equal(full, ones)
    assert torch.equal(lf, lo)


def test_generic_block_mask_from_random_csr():
    """Any CSR (a random lower-triangular block mask, diagonal kept) is
    honoured exactly, not only the sink + window pattern."""
    S = 1280
    nb = S // 64
    rng = np.random.default_rng(5)
    rows = []
    for i in range(nb):
        keep = [j for j in range(i) if rng.random() < 0.3] + [i]
        rows.append(keep)
    rp, ci = oracle.rows_to_csr(rows)
    q, k, v = inputs.qkv(1, S, 4, 2, 128, seed=52)
    status = zero_status()
    o = capi.attn_prefill_blocksparse(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(rp).cuda(),
                                      torch.from_numpy(ci).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, _ = oracle.attention(inputs.bits(q), inputs.bits(k), inputs.bits(v), 1 / math.sqrt(128),
                              oracle.rows_to_dense_mask(rows))
    assert_close_attention(to_f64(o), ref, "random CSR")


def test_sparse_never_reads_masked_blocks():
    """Overwrite V in blocks 2..25 with a large value: the last query tile
    (blocks 30, 31, window of 4 blocks, 2 sink blocks) loads none of them, so
    its rows are bit-identical; the full path reads them and moves."""
    S = 2048
    q, k, v = inputs.qkv(1, S, 4, 4, 128, seed=53)
    clean, _ = _run(q, k, v, "sparse", window=256)
    clean_full, _ = _run(q, k, v, "full")
    vp = v.clone()
    vp[:, 128:26 * 64] = 1000.0
    dirty, _ = _run(q, k, vp, "sparse", window=256)
    full, _ = _run(q, k, vp, "full")
    tail = slice(S - 128, S)
    assert torch.equal(clean[:, tail], dirty[:, tail])
    assert (full[:, tail].float() - clean_full[:, tail].float()).abs().max() > 100.0


def test_bad_csr_index_is_reported_not_read():
    S = 512
    q, k, v = inputs.qkv(1, S, 2, 2, 128, seed=54)
    rows = [[0]] + [[0, i] for i in range(1, S // 64)]
    rp, ci = oracle.rows_to_csr(rows)
    ci_bad = ci.copy()
    ci_bad[2] = 7            # row 1 lists block 7 (> 1): outside the causal range
    status = zero_status()
    o = capi.attn_prefill_blocksparse(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(rp).cuda(),
                                      torch.from_numpy(ci_bad).cuda(), status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & capi.FA_DEV_BAD_INDEX
    good = capi.attn_prefill_blocksparse(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(rp).cuda(),
                                         torch.from_numpy(ci).cuda())
    torch.cuda.synchronize()
    # rows of block 1 lost block 1 itself; other rows are unchanged
    assert torch.equal(o[:, :64], good[:, :64])
    assert torch.equal(o[:, 128:], good[:, 128:])


def test_deterministic():
    q, k, v = inputs.qkv(1, 2048, 8, 2, 128, seed=55)
    a, _ = _run(q, k, v, "full")
    b, _ = _run(q, k, v, "full")
    assert torch.equal(a, b)


@pytest.mark.parametrize("Hq,Hkv", [(4, 2), (3, 3)])
@pytest.mark.parametrize("mode", ["full", "sparse"])
@pytest.mark.parametrize("start", [256, 320])
def test_prefill_scores_that_grow_across_tiles(Hq, Hkv, mode, start):
    """Keys from token `start` on are scaled by 16 (exact in bf16), so their
    scores lie up to ~60 (log2) above everything the first tiles saw: p =
    2^(s - m) against the running maximum would leave the safe range (a
    row sum far above 2^32), so the kernel must move the reference to the
    tile's own maximum.  start = 256: the growth begins with a 128-key tile;
    start = 320: in the middle of one (the tile's first half still sits near
    the old reference, its second half far above it).  The result must still
    be the oracle's."""
    S = 768
    q, k, v = inputs.qkv(1, S, Hq, Hkv, 128, seed=1201)
    k[:, start:] = (k[:, start:].float() * 16.0).to(torch.bfloat16)
    # The test only means something if the scores really outgrow the first tiles' maximum.
    sc = torch.einsum("bthd,bshd->bhts", q.float()[:, start:, :1], k.float()[:, :, :1]) / 128 ** 0.5
    assert float(sc[..., start:].max() - sc[..., :128].max()) * 1.4427 > 40
    o, lse = _run(q, k, v, mode, window=256)
    ref, ref_lse = _oracle(q, k, v, mode, window=256)
    assert_close_attention(to_f64(o), ref, "growing scores %s" % mode)
    np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL)
