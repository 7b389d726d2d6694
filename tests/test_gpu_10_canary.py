"""GPU: every kernel writes exactly its outputs -- no element before or past
the end of an output, LSE or workspace (sentinel fences around each), and no
output element left unwritten (outputs start as NaN) -- on the shapes whose
row guards matter: ragged S, packed sequences whose last tile reaches past
their end, decode with lengths below Lmax, and the backward's split key tiles
with their fp32 partial sums.  The results are also checked against the
oracle, so a guard that dropped a needed write fails too."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import (LSE_ABS_TOL, Guarded, assert_close_attention, assert_close_grad,
                            to_f64, zero_status)

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)


@pytest.mark.parametrize("S", [65, 127, 129, 255])
@pytest.mark.parametrize("Hq,Hkv", [(3, 3), (4, 1)])     # one-tile kernel (odd G) and two-tile
@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_prefill_writes_only_its_rows(S, Hq, Hkv, mode):
    B = 2
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, seed=901 + S)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = Guarded((B, S, Hq, 128), torch.bfloat16)
    lse = Guarded((B, Hq, S), torch.float32)
    status = zero_status()
    c = capi.cfg(64, 64, 128)
    rp, ci = capi.blocksparse_index(S, c)
    if mode == "full":
        capi.attn_prefill_full(qd, kd, vd, o=o.t, lse=lse.t, status=status)
    else:
        capi.attn_prefill_blocksparse(qd, kd, vd, rp, ci, o=o.t, lse=lse.t, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o.check_all_written("o")
    lse.check_all_written("lse")
    mask = None
    if mode == "sparse":
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 64, 128))
    ref, ref_lse = oracle.attention(inputs.bits(q), inputs.bits(k), inputs.bits(v), SCALE, mask)
    assert_close_attention(to_f64(o.t), ref, "prefill %s S=%d" % (mode, S))
    np.testing.assert_allclose(to_f64(lse.t), ref_lse, atol=LSE_ABS_TOL)


def test_varlen_tiles_past_a_sequence_end_write_nothing_there():
    lengths = [65, 200, 1, 130, 64]
    T = sum(lengths)
    Hq, Hkv = 4, 2
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")
    q = inputs.randn_bf16((T, Hq, 128), 931)
    k = inputs.randn_bf16((T, Hkv, 128), 932)
    v = inputs.randn_bf16((T, Hkv, 128), 933)
    o = Guarded((T, Hq, 128), torch.bfloat16)
    lse = Guarded((Hq, T), torch.float32)
    ws = Guarded((int(capi.lib().fa_varlen_workspace_size(len(lengths), T)),), torch.uint8)
    status = zero_status()
    c = capi.cfg(64, 64, 128)
    rp, ci = capi.blocksparse_index(max(lengths), c)
    modes = torch.tensor([0, 1, 0, 1, 1], dtype=torch.int32, device="cuda")
    capi.attn_prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu, max(lengths), rp, ci,
                             mode_dev=modes, o=o.t, lse=lse.t, workspace=ws.t, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o.check_all_written("o")
    lse.check_all_written("lse")
    ws.check_fences("workspace")
    qb, kb, vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
    t0 = 0
    for L, m in zip(lengths, modes.tolist()):
        mask = (oracle.rows_to_dense_mask(oracle.blocksparse_rows(L, 64, 64, 128)) if m else None)
        ref, ref_lse = oracle.attention(qb[None, t0:t0 + L], kb[None, t0:t0 + L],
                                        vb[None, t0:t0 + L], SCALE, mask)
        assert_close_attention(to_f64(o.t[t0:t0 + L])[None], ref, "varlen L=%d" % L)
        np.testing.assert_allclose(to_f64(lse.t[:, t0:t0 + L])[None], ref_lse, atol=LSE_ABS_TOL)
        t0 += L


@pytest.mark.parametrize("mode", [capi.FA_MODE_FULL, capi.FA_MODE_SPARSE])
def test_decode_writes_only_its_outputs_and_workspace(mode):
    B, Lmax, Hq, Hkv = 3, 5000, 16, 4
    seqlens = [5000, 1234, 1]
    q, kc, vc = inputs.decode_inputs(B, Lmax, Hq, Hkv, 128, 941)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    c = capi.cfg(64, 128, 1024)
    o = Guarded((B, Hq, 128), torch.bfloat16)
    lse = Guarded((B, Hq), torch.float32)
    ws = Guarded((capi.decode_workspace_size(B, Hq, Hkv, Lmax),), torch.uint8)
    status = zero_status()
    capi.attn_decode(q.cuda(), kc.cuda(), vc.cuda(), sl, mode, c, o=o.t, lse=lse.t,
                     workspace=ws.t, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o.check_all_written("o")
    lse.check_all_written("lse")
    ws.check_fences("workspace")
    ref, ref_lse = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc),
                                 np.array(seqlens, np.int32), SCALE, mode, 64, 128, 1024)
    assert_close_attention(to_f64(o.t), ref, "decode")
    np.testing.assert_allclose(to_f64(lse.t), ref_lse, atol=LSE_ABS_TOL)


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_backward_split_tiles_write_only_their_gradients(mode):
    # S = 2560: 40 query blocks, so the first key tiles are cut into chunks
    # whose fp32 partial sums go through the workspace.
    B, S, Hq, Hkv = 1, 2560, 2, 1
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, 951, device="cuda")
    do = inputs.randn_bf16((B, S, Hq, 128), 952, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty(B, Hq, S, device="cuda")
    status = zero_status()
    c = capi.cfg(64, 128, 256)
    rp, ci = capi.blocksparse_index(S, c)
    if mode == "full":
        capi.attn_prefill_full(q, k, v, o=o, lse=lse, status=status)
    else:
        capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o, lse=lse, status=status)
    dq = Guarded((B, S, Hq, 128), torch.bfloat16)
    dk = Guarded((B, S, Hkv, 128), torch.bfloat16)
    dv = Guarded((B, S, Hkv, 128), torch.bfloat16)
    ws = Guarded((capi.attn_backward_workspace_size(B, S, Hq, Hkv),), torch.uint8)
    capi.attn_prefill_backward(q, k, v, o, lse, do, rp, ci, mode=int(mode == "sparse"),
                               dq=dq.t, dk=dk.t, dv=dv.t, workspace=ws.t, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for g, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        g.check_all_written(name)
    ws.check_fences("workspace")
    mask = (oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 128, 256))
            if mode == "sparse" else None)
    want = oracle.attention_backward(inputs.bits(q), inputs.bits(k), inputs.bits(v),
                                     inputs.bits(do), SCALE, mask)
    for name, g, w in zip(("dq", "dk", "dv"), (dq.t, dk.t, dv.t), want):
        assert_close_grad(to_f64(g), w, "%s %s" % (mode, name))


@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_prefill_long_sequence_item_order_covers_every_row(mode):
    """S = 40000 with 4 query heads per KV head: long enough for the
    KV-head-major item order (the whole sequence one band, so each KV
    head's items run one after another; the last tile ragged).  Every output row must be written exactly
    where it belongs: all rows finite inside the fences, sampled rows equal
    to the oracle's."""
    B, S, Hq, Hkv = 2, 40000, 8, 2
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, 991, device="cuda")
    o = Guarded((B, S, Hq, 128), torch.bfloat16)
    lse = Guarded((B, Hq, S), torch.float32)
    status = zero_status()
    c = capi.cfg(64, 128, 1024)
    rp, ci = capi.blocksparse_index(S, c)
    if mode == "full":
        capi.attn_prefill_full(q, k, v, o=o.t, lse=lse.t, status=status)
        mask = None
    else:
        capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o.t, lse=lse.t, status=status)
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 128, 1024))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o.check_all_written("o")
    lse.check_all_written("lse")
    rows = inputs.sample_rows(B, S, Hq, Hkv, seed=991, n_random=48, n_groups=1)
    rng = np.random.default_rng(991)
    rows = rows[np.sort(rng.choice(len(rows), size=min(400, len(rows)), replace=False))]
    ref, ref_lse = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), SCALE,
                                         rows, mask)
    rt = torch.from_numpy(rows).cuda()
    assert_close_attention(to_f64(o.t[rt[:, 0], rt[:, 2], rt[:, 1]]), ref, "S=40000 %s" % mode)
    np.testing.assert_allclose(to_f64(lse.t[rt[:, 0], rt[:, 1], rt[:, 2]]), ref_lse,
                               atol=LSE_ABS_TOL)
