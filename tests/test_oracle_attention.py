"""Pins of the oracle's block pattern and masked softmax attention.

* Block rule ('Flux Attention' implementation paragraph: 64-token blocks,
  128 sink tokens; window in whole blocks): hand-worked rows and counts.
* Attention ('Self-Attention 이후', section '셀프 어텐션이 비싼 이유': QK^T /
  sqrt(d_k) -> softmax -> V): brute force in pure Python on tiny inputs, an
  explicitly materialised S x S matrix (the three-pass form of the
  FlashAttention newsletter), and special cases with closed forms.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import inputs
from tests import brute


def _bits(x):
    return inputs.bits(torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16))


def _f(bits):
    return oracle.bf16_bits_to_f64(bits)


# ----------------------------------------------------------------- CSR pins
def test_csr_hand_worked_rows(golden_dir):
    with open(os.path.join(golden_dir, "csr_rows.json")) as f:
        g = json.load(f)
    for case in g["cases"]:
        rows = oracle.blocksparse_rows(case["S"], 64, 128, case["window"])
        assert sum(len(r) for r in rows) == case["nnz"]
        for i, want in case.get("rows", {}).items():
            assert rows[int(i)] == want
        if "row_lengths_first" in case:
            n = len(case["row_lengths_first"])
            assert [len(r) for r in rows[:n]] == case["row_lengths_first"]


@pytest.mark.parametrize("S,block,sink,window", [
    (64, 64, 128, 128), (65, 64, 128, 128), (1000, 64, 128, 256),
    (4096, 64, 0, 64), (4096, 64, 256, 64), (777, 16, 32, 48)])
def test_csr_closed_form_count_and_structure(S, block, sink, window):
    rows = oracle.blocksparse_rows(S, block, sink, window)
    sb, wb = sink // block, window // block
    for i, r in enumerate(rows):
        a = min(sb, i + 1)
        lo = max(0, i - wb + 1)
        count = a + (i - lo + 1) - max(0, a - lo)
        assert len(r) == count
        assert r == sorted(set(r)) and all(0 <= j <= i for j in r)
        if wb >= 1:
            assert r[-1] == i                     # own block always kept
    rp, ci = oracle.rows_to_csr(rows)
    assert rp[0] == 0 and rp[-1] == len(ci) and np.all(np.diff(rp) >= 0)


def test_csr_all_ones_when_window_covers_everything():
    rows = oracle.blocksparse_rows(640, 64, 0, 640)
    assert rows == [list(range(i + 1)) for i in range(10)]


# ------------------------------------------------------- attention vs brute
def _tiny_case(seed, B, S, Hq, Hkv, D):
    rng = np.random.default_rng(seed)
    # multiples of 1/8 keep bf16 exact and exp() small
    q = rng.integers(-8, 9, size=(B, S, Hq, D)) / 8.0
    k = rng.integers(-8, 9, size=(B, S, Hkv, D)) / 8.0
    v = rng.integers(-16, 17, size=(B, S, Hkv, D)) / 8.0
    return _bits(q), _bits(k), _bits(v)


@pytest.mark.parametrize("mode", ["full", "sparse"])
@pytest.mark.parametrize("S,Hq,Hkv", [(1, 1, 1), (37, 2, 1), (70, 4, 2)])
def test_attention_matches_brute_force(mode, S, Hq, Hkv):
    B, D, block, sink, window = 2, 8, 16, 16, 32
    qb, kb, vb = _tiny_case(S * 7 + Hq, B, S, Hq, Hkv, D)
    scale = 1.0 / math.sqrt(D)
    mask = None
    if mode == "sparse":
        mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, block, sink, window))
    out, lse = oracle.attention(qb, kb, vb, scale, mask, block)
    qf, kf, vf = _f(qb), _f(kb), _f(vb)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            K = kf[b, :, h // G].tolist()
            V = vf[b, :, h // G].tolist()
            for t in range(S):
                allowed = [brute.key_allowed(t, k, mode, block, sink, window) for k in range(S)]
                o, z = brute.attention_row(qf[b, t, h].tolist(), K, V, scale, allowed)
                np.testing.assert_allclose(out[b, t, h], o, atol=1e-12)
                assert abs(lse[b, h, t] - z) < 1e-12


def test_attention_equals_materialised_matrix():
    """The unfused form: the full S x S score matrix, mask, row softmax, x V."""
    B, S, Hq, Hkv, D = 1, 300, 4, 2, 32
    q, k, v = inputs.qkv(B, S, Hq, Hkv, D, seed=11)
    qb, kb, vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
    scale = 1.0 / math.sqrt(D)
    rows = oracle.blocksparse_rows(S, 64, 128, 128)
    mask = oracle.rows_to_dense_mask(rows)
    for bm in (None, mask):
        out, lse = oracle.attention(qb, kb, vb, scale, bm)
        for h in range(Hq):
            Q, K, V = _f(qb)[0, :, h], _f(kb)[0, :, h // 2], _f(vb)[0, :, h // 2]
            s = Q @ K.T * scale
            allowed = np.tril(np.ones((S, S), bool))
            if bm is not None:
                blk = np.arange(S) // 64
                allowed &= bm[blk[:, None], blk[None, :]].astype(bool)
            s = np.where(allowed, s, -np.inf)
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p /= p.sum(axis=1, keepdims=True)
            np.testing.assert_allclose(out[0, :, h], p @ V, atol=1e-12)


def test_special_cases_row0_and_zero_keys():
    B, S, Hq, Hkv, D = 1, 200, 2, 1, 16
    q, k, v = inputs.qkv(B, S, Hq, Hkv, D, seed=12)
    qb, vb = inputs.bits(q), inputs.bits(v)
    kb = np.zeros_like(inputs.bits(k))            # K == 0: uniform weights
    out, lse = oracle.attention(qb, kb, vb, 0.125)
    V = _f(vb)[0, :, 0]
    cum = np.cumsum(V, axis=0) / np.arange(1, S + 1)[:, None]
    for h in range(Hq):
        np.testing.assert_allclose(out[0, :, h], cum, atol=1e-12)
        np.testing.assert_allclose(lse[0, h], np.log(np.arange(1, S + 1)), atol=1e-12)
    out2, _ = oracle.attention(qb, inputs.bits(k), vb, 0.125)
    np.testing.assert_allclose(out2[0, 0, :], np.broadcast_to(V[0], (Hq, D)), atol=0)


def test_key_shift_invariance():
    """Adding one vector c to every key adds q.c to a whole row of scores:
    the softmax is unchanged (max-subtraction invariance, newsletter)."""
    B, S, Hq, D = 1, 96, 1, 8
    qb, kb, vb = _tiny_case(5, B, S, Hq, 1, D)
    c = np.array([1.0, -2.0, 0.5, 0, 3.0, -1.0, 0.25, 2.0])
    kb2 = _bits(_f(kb) + c)
    assert np.array_equal(_f(kb2), _f(kb) + c)          # exact in bf16
    o1, _ = oracle.attention(qb, kb, vb, 0.5)
    o2, _ = oracle.attention(qb, kb2, vb, 0.5)
    np.testing.assert_allclose(o1, o2, atol=1e-12)


def test_gqa_head_mapping():
    B, S, Hq, Hkv, D = 1, 64, 4, 2, 8
    q, k, v = inputs.qkv(B, S, Hq, Hkv, D, seed=13)
    qb, kb, vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
    out, _ = oracle.attention(qb, kb, vb, 0.3)
    for h in range(Hq):
        single, _ = oracle.attention(qb[:, :, h:h + 1], kb[:, :, h // 2:h // 2 + 1],
                                     vb[:, :, h // 2:h // 2 + 1], 0.3)
        np.testing.assert_allclose(out[:, :, h], single[:, :, 0], atol=0)
    # a transposed mapping (h % Hkv) gives a different answer
    wrong, _ = oracle.attention(qb[:, :, 1:2], kb[:, :, 1:2], vb[:, :, 1:2], 0.3)
    assert np.max(np.abs(wrong[:, :, 0] - out[:, :, 1])) > 1e-3


def test_all_ones_block_mask_equals_full_and_window_cover():
    B, S, Hq, Hkv, D = 1, 320, 2, 2, 16
    q, k, v = inputs.qkv(B, S, Hq, Hkv, D, seed=14)
    qb, kb, vb = inputs.bits(q), inputs.bits(k), inputs.bits(v)
    full, _ = oracle.attention(qb, kb, vb, 0.25)
    ones = np.ones((5, 5), np.uint8)
    a, _ = oracle.attention(qb, kb, vb, 0.25, ones)
    np.testing.assert_array_equal(a, full)
    cover = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 0, 320))
    b_, _ = oracle.attention(qb, kb, vb, 0.25, cover)
    np.testing.assert_array_equal(b_, full)
    sparse = oracle.rows_to_dense_mask(oracle.blocksparse_rows(S, 64, 64, 64))
    c_, _ = oracle.attention(qb, kb, vb, 0.25, sparse)
    assert np.max(np.abs(c_ - full)) > 1e-3        # the mask matters


@pytest.mark.parametrize("mode", [oracle.MODE_FULL, oracle.MODE_SPARSE])
def test_decode_equals_last_prefill_row(mode):
    B, Lmax, Hq, Hkv, D = 2, 400, 4, 2, 16
    q, kc, vc = inputs.decode_inputs(B, Lmax, Hq, Hkv, D, seed=15)
    seqlens = np.array([400, 263], np.int32)
    qb, kb, vb = inputs.bits(q), inputs.bits(kc), inputs.bits(vc)
    out, lse = oracle.decode(qb, kb, vb, seqlens, 0.25, mode, 64, 128, 128)
    for b in range(B):
        L = int(seqlens[b])
        qfull = np.zeros((1, L, Hq, D), np.uint16)
        qfull[0, L - 1] = qb[b]
        mask = None
        if mode == oracle.MODE_SPARSE:
            mask = oracle.rows_to_dense_mask(oracle.blocksparse_rows(L, 64, 128, 128))
        rows = np.array([(0, h, L - 1) for h in range(Hq)], np.int64)
        o, l = oracle.attention_rows(qfull, kb[b:b + 1, :L], vb[b:b + 1, :L], 0.25, rows, mask)
        np.testing.assert_allclose(out[b], o, atol=1e-14)
        np.testing.assert_allclose(lse[b], l, atol=1e-14)


def test_decode_sparse_keys_are_sink_and_window():
    """With V = one-hot of the key index (a distinct marker per key), the
    output support is exactly the attended key set."""
    B, Lmax, Hq, Hkv, D = 1, 1000, 1, 1, 1
    L = 1000
    kc = np.zeros((B, Lmax, Hkv, D))
    q = np.zeros((B, Hq, D))
    # D = 1 cannot encode 1000 keys; use K = 0 so weights are uniform and
    # check the mean of V = key index over the attended set instead.
    vc = np.arange(Lmax, dtype=np.float64).reshape(1, Lmax, 1, 1)
    vc_bits = _bits(vc)
    keys = [k for k in range(L) if brute.key_allowed(L - 1, k, "sparse", 64, 128, 256)]
    out, _ = oracle.decode(_bits(q), _bits(kc), vc_bits, np.array([L], np.int32), 1.0,
                           oracle.MODE_SPARSE, 64, 128, 256)
    expect = np.mean(_f(vc_bits)[0, keys, 0, 0])
    assert abs(out[0, 0, 0] - expect) < 1e-9
    # row block 15 keeps sink blocks 0-1 and window blocks 12..15 (256 tokens)
    assert keys[:128] == list(range(128)) and keys[128] == 12 * 64 and len(keys) == 128 + 232
