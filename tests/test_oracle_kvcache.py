"""Pins of the oracle's FP8 (E4M3) codec, paged gather and fp64 decode."""
import math

import numpy as np

import oracle
from block_sparse_attention_layerrouter_b200 import inputs


def test_e4m3_known_codes():
    # Values fixed by the format: bias 7, 3 mantissa bits, max 448, no inf.
    table = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
             0x38: 1.0, 0x39: 1.125, 0x40: 2.0, 0x7E: 448.0, 0x80: -0.0, 0xB8: -1.0,
             0xFE: -448.0, 0x77: 240.0}
    for code, val in table.items():
        got = oracle.e4m3_decode([code])[0]
        assert got == val and math.copysign(1, got) == math.copysign(1, val), (hex(code), got)
    assert np.isnan(oracle.e4m3_decode([0x7F, 0xFF])).all()


def test_e4m3_round_trip_and_monotone():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    vals = oracle.e4m3_decode(codes)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)
    pos = np.sort(vals[vals > 0])
    assert np.all(np.diff(pos) > 0) and len(pos) == 126


def test_e4m3_rounding_ties_and_saturation():
    # Midpoint between 1.0 (0x38, even) and 1.125 (0x39): goes to the even code.
    assert oracle.e4m3_encode([1.0625])[0] == 0x38
    # Midpoint between 1.125 (0x39) and 1.25 (0x3A, even): up.
    assert oracle.e4m3_encode([1.1875])[0] == 0x3A
    assert oracle.e4m3_encode([1.07])[0] == 0x39
    assert oracle.e4m3_encode([1000.0])[0] == 0x7E
    assert oracle.e4m3_encode([-1e9])[0] == 0xFE
    assert oracle.e4m3_encode([2.0 ** -10])[0] == 0x00     # half the smallest subnormal: even
    assert oracle.e4m3_encode([3 * 2.0 ** -10])[0] == 0x02  # 1.5 subnormal steps: even (2)


def test_kv_quantize_error_bound():
    """|x/s - decode(code)| <= half a step of the code's binade (2^-4 relative)
    inside the normal range."""
    x = inputs.bits(inputs.randn_bf16((64, 2, 16), 77))
    s = np.array([0.02, 0.05], np.float32)
    codes = oracle.kv_quantize(x, s)
    xs = oracle.bf16_bits_to_f64(x) / s[None, :, None]
    err = np.abs(oracle.e4m3_decode(codes) - xs)
    assert np.all(err <= np.maximum(np.abs(xs) * 2.0 ** -4, 2.0 ** -10) + 1e-12)


def test_decode_values_matches_bits_decode():
    B, L, Hq, Hkv, D = 2, 300, 4, 2, 16
    q, kc, vc = inputs.decode_inputs(B, L, Hq, Hkv, D, 78)
    sl = np.array([300, 129], np.int32)
    for mode in (oracle.MODE_FULL, oracle.MODE_SPARSE):
        want, wl = oracle.decode(inputs.bits(q), inputs.bits(kc), inputs.bits(vc), sl, 0.25,
                                 mode=mode, window=128)
        got, gl = oracle.decode_values(q.double().numpy(), kc.double().numpy(),
                                       vc.double().numpy(), sl, 0.25, mode=mode, window=128)
        np.testing.assert_allclose(got, want, atol=1e-12)
        np.testing.assert_allclose(gl, wl, atol=1e-12)


def test_paged_gather_follows_the_block_table():
    pages = np.arange(5 * 4 * 1 * 2).reshape(5, 4, 1, 2)
    bt = np.array([[3, 0, 4], [1, 2, 0]], np.int32)
    out = oracle.paged_gather(pages, bt, [10, 5], page_size=4)
    assert np.array_equal(out[0, 0], pages[3, 0]) and np.array_equal(out[0, 9], pages[4, 1])
    assert np.array_equal(out[1, 4], pages[2, 0]) and np.all(out[1, 5:] == 0)
