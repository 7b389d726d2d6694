"""GPU: the CSR builder is bit-exact against the oracle's brute-force
enumeration ('Flux Attention', implementation paragraph: 64-token blocks,
128 sink tokens; window in whole blocks)."""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_layerrouter_b200 import capi

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("S,sink,window", [
    (1024, 128, 128), (8192, 128, 1024), (32768, 128, 2048), (262144, 128, 4096),
    (1, 128, 128), (64, 128, 128), (65, 128, 128), (127, 0, 64), (1000, 256, 64),
    (4096, 0, 4096), (5000, 640, 192)])
def test_csr_bit_exact(S, sink, window):
    row_ptr, col_idx = capi.blocksparse_index(S, capi.cfg(64, sink, window))
    torch.cuda.synchronize()
    rp, ci = oracle.blocksparse_csr(S, 64, sink, window)
    assert np.array_equal(row_ptr.cpu().numpy(), rp)
    assert np.array_equal(col_idx.cpu().numpy(), ci)
