"""GPU: the two-tile prefill kernel at the GQA widths the other tests do not
use -- 6 and 8 query heads per KV head (3 and 4 head pairs sharing each K/V
tile) -- whole tensors at a few tiles, and at lengths long enough for the
KV-head-major item bands (a band is 148 / pairs-per-KV-head query tiles:
49 for G = 6, 37 for G = 8), on sampled rows with fences around the outputs.
Compared with the oracle element by element."""
import math

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi, inputs
from tests.gpu_util import (LSE_ABS_TOL, Guarded, assert_close_attention, to_f64,
                            zero_status)

pytestmark = pytest.mark.gpu
SCALE = 1 / math.sqrt(128)


def _run(q, k, v, mode, sink, window, o=None, lse=None):
    S = q.shape[1]
    status = zero_status()
    if mode == "full":
        out = capi.attn_prefill_full(q, k, v, o=o, lse=lse, status=status)
        mask = None
    else:
        rp, ci = capi.blocksparse_index(S, capi.cfg(64, sink, window))
        out = capi.attn_prefill_blocksparse(q, k, v, rp, ci, o=o, lse=lse, status=status)
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, sink, window))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, mask


@pytest.mark.parametrize("Hq,Hkv", [(6, 1), (8, 1), (16, 2)])
@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_wide_groups_whole_tensor(Hq, Hkv, mode):
    B, S = 1, 1536
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, seed=1300 + Hq + Hkv)
    lse = torch.empty(B, Hq, S, device="cuda", dtype=torch.float32)
    o, mask = _run(q.cuda(), k.cuda(), v.cuda(), mode, 128, 384, lse=lse)
    ref, ref_lse = oracle.attention(inputs.bits(q), inputs.bits(k), inputs.bits(v), SCALE, mask)
    assert_close_attention(to_f64(o), ref, "G=%d %s" % (Hq // Hkv, mode))
    np.testing.assert_allclose(to_f64(lse), ref_lse, atol=LSE_ABS_TOL)


@pytest.mark.parametrize("Hq,S", [(6, 25600), (8, 19200)])
@pytest.mark.parametrize("mode", ["full", "sparse"])
def test_wide_groups_item_bands(Hq, S, mode):
    B, Hkv = 1, 1
    q, k, v = inputs.qkv(B, S, Hq, Hkv, 128, 1310 + Hq, device="cuda")
    o = Guarded((B, S, Hq, 128), torch.bfloat16)
    lse = Guarded((B, Hq, S), torch.float32)
    _, mask = _run(q, k, v, mode, 128, 1024, o=o.t, lse=lse.t)
    o.check_all_written("o")
    lse.check_all_written("lse")
    rows = inputs.sample_rows(B, S, Hq, Hkv, seed=1310 + Hq, n_random=48, n_groups=1)
    rng = np.random.default_rng(1310 + Hq)
    rows = rows[np.sort(rng.choice(len(rows), size=min(300, len(rows)), replace=False))]
    ref, ref_lse = oracle.attention_rows(inputs.bits(q), inputs.bits(k), inputs.bits(v), SCALE,
                                         rows, mask)
    rt = torch.from_numpy(rows).cuda()
    assert_close_attention(to_f64(o.t[rt[:, 0], rt[:, 2], rt[:, 1]]), ref,
                           "G=%d S=%d %s" % (Hq, S, mode))
    np.testing.assert_allclose(to_f64(lse.t[rt[:, 0], rt[:, 1], rt[:, 2]]), ref_lse,
                               atol=LSE_ABS_TOL)
