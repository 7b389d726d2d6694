"""Pins of the pair counting used for FLOP accounting.

'Self-Attention 이후', section '셀프 어텐션이 비싼 이유': N tokens give N^2
score entries (~1M at 1024, ~1B at 32768, ~17B at 131072, 16M at 4K, 16B at
128K).  The causal and block-sparse counts are checked by brute force.
"""
import json
import os

import pytest

import oracle
from tests import brute


def test_entry_counts_match_page(golden_dir):
    with open(os.path.join(golden_dir, "attention_entry_counts.json")) as f:
        g = json.load(f)
    for c in g["counts"]:
        n = c["seq_len"]
        assert abs(n * n - c["approx"]) / c["approx"] < 0.10, c
        # causal keeps S(S+1)/2 of them, a bit over half
        assert oracle.attended_pairs_full(n) * 2 - n == n * n


@pytest.mark.parametrize("S,window", [(64, 128), (200, 128), (1000, 256), (1024, 128)])
def test_sparse_pairs_brute(S, window):
    want = sum(1 for t in range(S) for k in range(S)
               if brute.key_allowed(t, k, "sparse", 64, 128, window))
    assert oracle.attended_pairs_sparse(S, 64, 128, window) == want
    assert oracle.attended_pairs_full(S) == sum(t + 1 for t in range(S))
