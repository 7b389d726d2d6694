"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no arithmetic of the method: it only draws random tensors
of the workload shapes and hands out their raw bf16 bits, so that the CUDA
path and the CPU oracle see the very same inputs.

Recipe (the pages give model shapes, not data; their benchmarks --
LongBench-E, RULER, GSM8K, AIME24 -- are stood in for by random tensors of the
same attention shapes):
  * Q, K, V: bf16 drawn from N(0, 1) with torch generators seeded
    ``seed`` (Q), ``seed + 100`` (K) and ``seed + 200`` (V).
  * Router weights: fp32 N(0, 0.02) for W1 and W2 (generator seeded
    ``seed + 300 + layer``), zero biases unless a bias is given.
  * Decode caches: K/V caches bf16 N(0, 1), queries N(0, 1), same seed offsets.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """Shapes of one workload (names follow the model each is shaped like)."""
    name: str
    B: int
    S: int
    Hq: int
    Hkv: int
    D: int = 128
    layers: int = 1
    window: int = 128          # local window, tokens
    sink: int = 128            # sink tokens
    block: int = 64            # sparsity block, tokens
    hidden: int = 64           # router MLP hidden width
    decode_len: int = 0        # >0: decode workload with this cache length
    varlen: bool = False       # packed batch of B requests of seeded lengths <= S
    train: bool = False        # soft-routed training step (forward + backward)
    paged: bool = False        # decode through a paged cache (64-token pages)
    kv_fp8: bool = False       # E4M3 KV cache (paged)
    seed: int = 1000
    notes: str = field(default="", compare=False)


# The five workloads the pages' models suggest (shapes only).
WORKLOADS = {
    "mha4-s1024": Workload("mha4-s1024", B=1, S=1024, Hq=4, Hkv=4, window=128,
                           hidden=64, seed=1000,
                           notes="single layer, 4 MHA heads; both modes"),
    "qwen3-4b-layer-s8192": Workload("qwen3-4b-layer-s8192", B=1, S=8192, Hq=32, Hkv=8,
                                     window=1024, hidden=256, seed=1001,
                                     notes="Qwen3-4B-shaped GQA layer"),
    "llama3.1-8b-32l-s32768": Workload("llama3.1-8b-32l-s32768", B=1, S=32768, Hq=32,
                                       Hkv=8, layers=32, window=2048, hidden=256,
                                       seed=1002, notes="32-layer prefill stack, ~half sparse"),
    "qwen3-8b-layer-s262144": Workload("qwen3-8b-layer-s262144", B=1, S=262144, Hq=32,
                                       Hkv=8, window=4096, hidden=256, seed=1003,
                                       notes="256K prefill, one layer per mode"),
    "decode-b8-l131072-32l": Workload("decode-b8-l131072-32l", B=8, S=1, Hq=32, Hkv=8,
                                      layers=32, window=2048, hidden=256,
                                      decode_len=131072, seed=1004,
                                      notes="decode, 16 full + 16 sparse layers"),
    # Serving batch: 8 requests of seeded lengths in [1024, 32768] packed along
    # the token axis, one Qwen3-4B-shaped layer, each request routed by the
    # layer router on its own prompt.
    "serving-varlen-qwen3-4b": Workload("serving-varlen-qwen3-4b", B=8, S=32768, Hq=32, Hkv=8,
                                        window=1024, hidden=256, varlen=True, seed=1006,
                                        notes="packed variable-length batch, routed per request"),
    # Training step of one soft-routed Qwen3-4B-shaped layer: router, both
    # attention paths with their LSE, then the backward of the mixed output
    # (router weights and Q/K/V gradients through both paths).
    "train-soft-qwen3-4b-layer-s8192": Workload("train-soft-qwen3-4b-layer-s8192", B=1, S=8192,
                                                Hq=32, Hkv=8, window=1024, hidden=256,
                                                train=True, seed=1007,
                                                notes="soft-routed layer, forward + backward"),
    # The decode workload through a paged cache (pages in a seeded random
    # order), bf16 and FP8 E4M3 with per-head scales.
    "decode-paged-b8-l131072-32l": Workload("decode-paged-b8-l131072-32l", B=8, S=1, Hq=32,
                                            Hkv=8, layers=32, window=2048, hidden=256,
                                            decode_len=131072, paged=True, seed=1008,
                                            notes="paged bf16 decode"),
    "decode-fp8-b8-l131072-32l": Workload("decode-fp8-b8-l131072-32l", B=8, S=1, Hq=32, Hkv=8,
                                          layers=32, window=2048, hidden=256, decode_len=131072,
                                          paged=True, kv_fp8=True, seed=1009,
                                          notes="paged FP8 (E4M3) decode"),
    # Profiling shape: the decode workload at a quarter of the context
    # (1 GiB of K/V, still far above the 126 MB L2).
    "decode-b8-l32768": Workload("decode-b8-l32768", B=8, S=1, Hq=32, Hkv=8, layers=2,
                                 window=2048, hidden=256, decode_len=32768, seed=1005,
                                 notes="decode profiling shape"),
}


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, seed: int, device="cpu") -> torch.Tensor:
    """bf16 N(0,1) tensor drawn in fp32 with a seeded generator, then rounded."""
    g = _gen(device, seed)
    return torch.randn(*shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def qkv(B, S, Hq, Hkv, D, seed, device="cpu"):
    """Q [B,S,Hq,D], K and V [B,S,Hkv,D], bf16 N(0,1)."""
    q = randn_bf16((B, S, Hq, D), seed, device)
    k = randn_bf16((B, S, Hkv, D), seed + 100, device)
    v = randn_bf16((B, S, Hkv, D), seed + 200, device)
    return q, k, v


def router_weights(in_features: int, hidden: int, seed: int, layer: int = 0,
                   b2=(0.0, 0.0), std: float = 0.02):
    """W1 [hidden, in], b1 [hidden], W2 [2, hidden], b2 [2]; fp32 CPU tensors."""
    g = _gen("cpu", seed + 300 + layer)
    w1 = torch.randn(hidden, in_features, generator=g) * std
    w2 = torch.randn(2, hidden, generator=g) * std
    b1 = torch.zeros(hidden)
    b2 = torch.tensor(list(b2), dtype=torch.float32)
    return w1.float(), b1.float(), w2.float(), b2.float()


def decode_inputs(B, Lmax, Hq, Hkv, D, seed, device="cpu"):
    """q [B,Hq,D] and K/V caches [B,Lmax,Hkv,D], bf16 N(0,1)."""
    q = randn_bf16((B, Hq, D), seed, device)
    kc = randn_bf16((B, Lmax, Hkv, D), seed + 100, device)
    vc = randn_bf16((B, Lmax, Hkv, D), seed + 200, device)
    return q, kc, vc


def gumbel(B: int, seed: int) -> torch.Tensor:
    """Standard Gumbel samples g = -log(-log(U)), U ~ U(0,1), fp32 [B, 2]
    (the noise of the soft router, drawn here and passed in as an input)."""
    g = _gen("cpu", seed)
    u = torch.rand(B, 2, generator=g, dtype=torch.float64).clamp_(1e-12, 1 - 1e-12)
    return (-torch.log(-torch.log(u))).float()


def varlen_lengths(B: int, max_len: int, seed: int, min_len: int = 1024) -> np.ndarray:
    """Seeded request lengths in [min_len, max_len] (the longest is max_len)."""
    rng = np.random.default_rng(seed)
    L = rng.integers(min_len, max_len + 1, size=B)
    L[int(rng.integers(0, B))] = max_len
    return L.astype(np.int64)


def fp8_codes(shape, seed: int, device="cpu") -> torch.Tensor:
    """Seeded E4M3 codes (uint8) with random sign and mantissa and exponent
    field 4..10 (magnitudes 1/8 .. 15): a stand-in for a quantised cache."""
    g = _gen(device, seed)
    sign = torch.randint(0, 2, shape, generator=g, device=device, dtype=torch.int32)
    e = torch.randint(4, 11, shape, generator=g, device=device, dtype=torch.int32)
    m = torch.randint(0, 8, shape, generator=g, device=device, dtype=torch.int32)
    return ((sign << 7) | (e << 3) | m).to(torch.uint8)


def fp8_scales(H: int, seed: int) -> torch.Tensor:
    """Per-head dequantisation scales, fp32 uniform in [1/48, 1/24]."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.uniform(1 / 48, 1 / 24, size=H).astype(np.float32))


def page_table(B: int, max_pages: int, seed: int, extra: int = 0) -> torch.Tensor:
    """Block table [B, max_pages] int32: a seeded permutation of the pool's
    B * max_pages + extra pages (the first B * max_pages entries)."""
    rng = np.random.default_rng(seed)
    perm = rng.permutation(B * max_pages + extra)[:B * max_pages]
    return torch.from_numpy(perm.reshape(B, max_pages).astype(np.int32))


def bits(t: torch.Tensor) -> np.ndarray:
    """Raw bf16 bit patterns of a tensor as a uint16 numpy array (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def sample_rows(B: int, S: int, Hq: int, Hkv: int, seed: int, block: int = 64,
                n_random: int = 256, n_boundary: int = 8, n_groups: int = 2):
    """Seeded (b, h, t) rows for spot checks at full size: all rows of query
    blocks 0, 1, 2 and the last one, both sides of `n_boundary` random block
    boundaries, and `n_random` random rows; every head of `n_groups` random
    KV groups.  Returns int64 [n, 3]."""
    rng = np.random.default_rng(seed)
    G = Hq // Hkv
    nb = -(-S // block)
    ts = set()
    for qb in sorted({0, 1, 2, nb - 1}):
        if 0 <= qb < nb:
            ts.update(range(qb * block, min(S, (qb + 1) * block)))
    for kb in rng.integers(1, max(2, nb), size=n_boundary):
        ts.update({int(kb) * block - 1, min(S - 1, int(kb) * block)})
    ts.update(int(x) for x in rng.integers(0, S, size=n_random))
    groups = rng.choice(Hkv, size=min(n_groups, Hkv), replace=False)
    heads = [int(g) * G + j for g in groups for j in range(G)]
    bs = range(B) if B <= 2 else sorted({0, B - 1})
    rows = [(b, h, t) for b in bs for h in heads for t in sorted(ts) if 0 <= t < S]
    return np.array(rows, dtype=np.int64)
