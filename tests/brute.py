"""Pure-Python brute force for tiny inputs, independent of ``oracle/``.

Written straight from the textbook definition with Python floats and
``math.exp`` -- no numpy, no C, no max subtraction beyond what keeps exp
finite for the tiny magnitudes used in the tests.  The key rule is spelled
out separately from the oracle's enumeration.
"""
import math


def bits_to_float(b: int) -> float:
    import struct
    return struct.unpack("<f", struct.pack("<I", (int(b) & 0xFFFF) << 16))[0]


def key_allowed(t, k, mode, block, sink, window):
    """Causal, and for the sparse mode: a sink block, or a block within the
    last window/block blocks up to the query's own block."""
    if k > t:
        return False
    if mode == "full":
        return True
    kb, qb = k // block, t // block
    return kb < sink // block or qb - kb < window // block


def attention_row(q, K, V, scale, allowed):
    """q: list of D floats; K, V: lists of rows; allowed: list of bools."""
    scores = {}
    for k, ok in enumerate(allowed):
        if ok:
            scores[k] = scale * sum(a * b for a, b in zip(q, K[k]))
    z = sum(math.exp(s) for s in scores.values())
    out = [0.0] * len(q)
    for k, s in scores.items():
        w = math.exp(s) / z
        for d in range(len(out)):
            out[d] += w * V[k][d]
    return out, math.log(z)
