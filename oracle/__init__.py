"""CPU fp64 oracle for layer-routed hybrid (full / block-sparse) attention.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` import this package.  It shares no
code with the CUDA library and never imports it; the CUDA library never
imports this package.

Everything here is the plain definition of what the method computes, in fp64,
with no blocking, fusion or reordering beyond what that definition states.
Sources are cited by page title and section:

* [FLUX] "Flux Attention: 효율적인 LLM 추론을 위한 문맥 인식형 하이브리드
  어텐션" -- router paragraphs (pooling of the first and last 100 query
  tokens, MLP context encoder + router head to logits pi_FA / pi_SA, argmax
  hard routing at inference) and the implementation paragraph (64-token
  block sparsity, 128 sink tokens).
* [SOFTMAX] Newsletter "Softmax -> FlashAttention", sections "Softmax, 단순한
  함수가 아니다" (definition and worked example), "수치 안정성이라는 숨은 비용"
  (fp16 overflow near x = 11, max subtraction) and "어려움을 극복하기 위한
  Online Softmax" (running max / sum, rescale by exp(m_old - m_new)).
* [SELFATTN] "Self-Attention 이후: 트랜스포머 다음에 올 것들", section "셀프
  어텐션이 비싼 이유" (scores = Q K^T / sqrt(d_k), softmax, times V).

Readings taken where the pages are silent (the router paragraphs of [FLUX]
state "compress", not the operator, and give no flatten order, tie rule or
window granularity; [SELFATTN] gives the 1/sqrt(d_k) scale):
pooling is the arithmetic mean; the pooled [1 x h x d'] tensor is flattened
head-major (x[h*D + d]); a tie pi_SA == pi_FA routes to FULL; the local window
is counted in whole 64-token blocks including the query's own block; key k is
allowed for query t only when k <= t; query head h reads KV head h // G.

The backward functions are the chain rule through those definitions (the
gradients the router's soft-routing relaxation needs for training).

Parity status: every function below is pinned by tests/test_oracle_*.py
(worked examples, closed forms, invariants, brute force on tiny inputs).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess

import numpy as np

# ---------------------------------------------------------------- constants
# [FLUX] implementation paragraph: 64-token blocks and 128 sink tokens.
BLOCK = 64
SINK_TOKENS = 128
# [FLUX] router paragraph: the first and the last 100 prompt tokens.
N_HEAD_TOKENS = 100
N_TAIL_TOKENS = 100

MODE_FULL = 0
MODE_SPARSE = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attention_ref.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_attention.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C part of the oracle (plain gcc, fp64, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared",
             "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        p = ctypes.c_void_p
        lib.oracle_attention_rows.argtypes = [
            p, p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, p, ctypes.c_int, p, ctypes.c_long, p, p]
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_decode.argtypes = [
            p, p, p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, p, ctypes.c_int, p, p]
        lib.oracle_decode.restype = ctypes.c_int
        for name in ("oracle_attention_backward",):
            fn = getattr(lib, name)
            fn.argtypes = [p, p, p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                           ctypes.c_int, ctypes.c_int, ctypes.c_double, p, ctypes.c_int,
                           p, p, p]
            fn.restype = ctypes.c_int
        lib.oracle_attention_backward_qrows.argtypes = [
            p, p, p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, p, ctypes.c_int, p, ctypes.c_long, p]
        lib.oracle_attention_backward_qrows.restype = ctypes.c_int
        lib.oracle_attention_backward_keyrows.argtypes = [
            p, p, p, p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            p, ctypes.c_long, p, p]
        lib.oracle_attention_backward_keyrows.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the C oracle runs with."""
    return int(_load().oracle_num_threads())


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bit patterns (uint16) exactly to fp64."""
    u32 = bits.astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ softmax
def softmax(x) -> np.ndarray:
    """Row softmax with the row maximum subtracted first ([SOFTMAX], both
    the definition and the max-subtraction section)."""
    x = np.asarray(x, dtype=np.float64)
    m = np.max(x, axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def online_softmax(x, block: int):
    """Blockwise softmax of one row, in the order the [SOFTMAX] online
    section gives: per block, update the running maximum m; multiply the
    running sum (and nothing else is kept) by exp(m_old - m_new); add this
    block's exp(x - m_new).  Returns (probabilities, m, l, rescale factors),
    the factors being the exp(m_old - m_new) applied at each block."""
    x = np.asarray(x, dtype=np.float64)
    m = -math.inf
    l = 0.0
    factors = []
    for start in range(0, x.shape[0], block):
        chunk = x[start:start + block]
        m_new = max(m, float(np.max(chunk)))
        f = math.exp(m - m_new) if m != -math.inf else 0.0
        factors.append(f)
        l = l * f + float(np.sum(np.exp(chunk - m_new)))
        m = m_new
    return np.exp(x - m) / l, m, l, factors


def online_attention_row(scores, values, block: int) -> np.ndarray:
    """The online form applied to one attention row: running max, running
    sum and a running output vector, both rescaled by exp(m_old - m_new)
    whenever a block raises the maximum ([SOFTMAX] online section)."""
    s = np.asarray(scores, dtype=np.float64)
    v = np.asarray(values, dtype=np.float64)
    m, l = -math.inf, 0.0
    acc = np.zeros(v.shape[1])
    for start in range(0, s.shape[0], block):
        cs, cv = s[start:start + block], v[start:start + block]
        m_new = max(m, float(np.max(cs)))
        f = math.exp(m - m_new) if m != -math.inf else 0.0
        p = np.exp(cs - m_new)
        l = l * f + float(np.sum(p))
        acc = acc * f + p @ cv
        m = m_new
    return acc / l


# ------------------------------------------------------------------- router
def router_pool(q_bits: np.ndarray, n_head: int = N_HEAD_TOKENS,
                n_tail: int = N_TAIL_TOKENS) -> np.ndarray:
    """[FLUX] router: take tokens [0, n_head) and [S - n_tail, S) of the query
    tensor xQ [S x h x d'] and compress them to [1 x h x d'] -- here the mean
    over those n_head + n_tail tokens -- flattened head-major to [h * d'].

    q_bits: [B, S, Hq, D] bf16 bits.  Returns fp64 [B, Hq * D].
    Requires S >= n_head + n_tail (the two windows do not overlap)."""
    B, S, Hq, D = q_bits.shape
    if S < n_head + n_tail:
        raise ValueError("S must be >= n_head + n_tail")
    q = bf16_bits_to_f64(q_bits)
    sel = np.concatenate([q[:, :n_head], q[:, S - n_tail:]], axis=1)
    pooled = sel.sum(axis=1) / float(n_head + n_tail)       # [B, Hq, D]
    return pooled.reshape(B, Hq * D)


def router_mlp(x: np.ndarray, w1: np.ndarray, b1: np.ndarray,
               w2: np.ndarray, b2: np.ndarray) -> np.ndarray:
    """[FLUX] context encoder then router head: h = ReLU(W1 x + b1),
    [pi_FA, pi_SA] = W2 h + b2.  Shapes: W1 [H1, Hq*D], b1 [H1], W2 [2, H1],
    b2 [2].  Returns fp64 logits [B, 2] (column 0 = pi_FA, 1 = pi_SA)."""
    w1 = np.asarray(w1, np.float64)
    w2 = np.asarray(w2, np.float64)
    h = x @ w1.T + np.asarray(b1, np.float64)
    h = np.maximum(h, 0.0)
    return h @ w2.T + np.asarray(b2, np.float64)


def router_argmax(logits: np.ndarray) -> np.ndarray:
    """[FLUX] hard routing at inference: argmax over {pi_FA, pi_SA};
    a tie goes to FULL.  Returns int32 modes [B]."""
    return np.where(logits[:, 1] > logits[:, 0], MODE_SPARSE, MODE_FULL).astype(np.int32)


def router_decide(q_bits, w1, b1, w2, b2, n_head=N_HEAD_TOKENS, n_tail=N_TAIL_TOKENS):
    """Pool -> MLP -> argmax.  Returns (logits [B,2], modes [B], pooled x)."""
    x = router_pool(q_bits, n_head, n_tail)
    logits = router_mlp(x, w1, b1, w2, b2)
    return logits, router_argmax(logits), x


def router_soft(logits: np.ndarray, gumbel=None, tau: float = 1.0) -> np.ndarray:
    """[FLUX] training-time relaxation: r_soft = exp((pi_FA + g_FA)/tau) /
    sum_i exp((pi_i + g_i)/tau) over i in {FA, SA}, the Gumbel noise g given
    as an input.  Returns fp64 [B], the weight of the FULL output."""
    z = np.asarray(logits, np.float64)
    if gumbel is not None:
        z = z + np.asarray(gumbel, np.float64)
    return softmax(z / float(tau))[:, 0]


def soft_mix(o_full: np.ndarray, o_sparse: np.ndarray, r: np.ndarray) -> np.ndarray:
    """[FLUX] training-time output: y = r * O_FA + (1 - r) * O_SA, r per
    sequence (leading batch axis)."""
    r = np.asarray(r, np.float64).reshape((-1,) + (1,) * (o_full.ndim - 1))
    return r * o_full + (1.0 - r) * o_sparse


# ---------------------------------------------------------- sparse pattern
def blocksparse_rows(S: int, block: int = BLOCK, sink: int = SINK_TOKENS,
                     window: int = 2 * BLOCK):
    """Brute-force enumeration of the key blocks each query block keeps:
    the sink blocks (the first `sink` tokens) and the local window of
    window/block blocks ending at (and including) the query's own block,
    never a block after the query's own ([FLUX] implementation paragraph
    for the 64-token blocks and 128 sink tokens; the window size is an
    input).  Returns a list of ascending lists."""
    if block <= 0 or sink % block or window % block or S <= 0:
        raise ValueError("sink and window must be multiples of block")
    nb = -(-S // block)
    sink_blocks, win_blocks = sink // block, window // block
    rows = []
    for i in range(nb):
        j = np.arange(i + 1)              # every key block at or before i
        in_sink = j < sink_blocks
        in_window = (i - j) < win_blocks
        rows.append([int(x) for x in j[in_sink | in_window]])
    return rows


def rows_to_csr(rows):
    """Ascending block lists -> (row_ptr int32 [n+1], col_idx int32 [nnz])."""
    row_ptr = np.zeros(len(rows) + 1, dtype=np.int32)
    for i, r in enumerate(rows):
        row_ptr[i + 1] = row_ptr[i] + len(r)
    col_idx = np.array([j for r in rows for j in r], dtype=np.int32)
    return row_ptr, col_idx


def blocksparse_csr(S, block=BLOCK, sink=SINK_TOKENS, window=2 * BLOCK):
    return rows_to_csr(blocksparse_rows(S, block, sink, window))


def rows_to_dense_mask(rows, nkb=None) -> np.ndarray:
    n = len(rows)
    nkb = n if nkb is None else nkb
    m = np.zeros((n, nkb), dtype=np.uint8)
    for i, r in enumerate(rows):
        m[i, r] = 1
    return m


# ---------------------------------------------------------------- attention
def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def attention_rows(q_bits, k_bits, v_bits, scale, rows, block_mask=None,
                   block: int = BLOCK):
    """Masked causal softmax attention for selected rows, fp64 ([SELFATTN]
    definition; [SOFTMAX] max subtraction).  q_bits [B,S,Hq,D], k/v
    [B,S,Hkv,D] as uint16 bf16 bits; rows int64 [n,3] of (b, h, t);
    block_mask None (full causal) or uint8 [nqb, nkb].
    Returns (out fp64 [n, D], lse fp64 [n])."""
    lib = _load()
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    B, S, Hq, D = q_bits.shape
    Hkv = k_bits.shape[2]
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    out = np.zeros((rows.shape[0], D), dtype=np.float64)
    lse = np.zeros(rows.shape[0], dtype=np.float64)
    bm = None if block_mask is None else np.ascontiguousarray(block_mask, dtype=np.uint8)
    rc = lib.oracle_attention_rows(_ptr(q_bits), _ptr(k_bits), _ptr(v_bits), B, S,
                                   Hq, Hkv, D, float(scale), _ptr(bm), int(block),
                                   _ptr(rows), rows.shape[0], _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_attention_rows rejected its arguments")
    return out, lse


def all_rows(B, S, Hq) -> np.ndarray:
    b, t, h = np.meshgrid(np.arange(B), np.arange(S), np.arange(Hq), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), t.ravel()], axis=1).astype(np.int64)


def attention(q_bits, k_bits, v_bits, scale, block_mask=None, block=BLOCK):
    """Every row; returns (out [B,S,Hq,D], lse [B,Hq,S])."""
    B, S, Hq, D = q_bits.shape
    out, lse = attention_rows(q_bits, k_bits, v_bits, scale, all_rows(B, S, Hq),
                              block_mask, block)
    return out.reshape(B, S, Hq, D), lse.reshape(B, S, Hq).transpose(0, 2, 1)


# ----------------------------------------------------------------- backward
# The gradients below are the reverse-mode chain rule through the forward
# definitions above -- what training the router through the soft routing
# relaxation ([FLUX] router paragraphs) differentiates.  The pages print no
# backward; nothing here goes beyond the chain rule.

def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def attention_backward(q_bits, k_bits, v_bits, do_bits, scale, block_mask=None,
                       block: int = BLOCK):
    """dQ, dK, dV (fp64, shapes of q, k, v) of the masked causal attention
    for an upstream gradient dO [B,S,Hq,D] (bf16 bits): dV = P^T dO,
    dS = P * (dO V^T - rowsum(P * dO V^T)), dQ = scale dS K, dK = scale dS^T Q,
    a KV head summing over the G query heads that read it."""
    lib = _load()
    q_bits, k_bits, v_bits, do_bits = map(_u16, (q_bits, k_bits, v_bits, do_bits))
    B, S, Hq, D = q_bits.shape
    Hkv = k_bits.shape[2]
    dq = np.zeros((B, S, Hq, D))
    dk = np.zeros((B, S, Hkv, D))
    dv = np.zeros((B, S, Hkv, D))
    bm = None if block_mask is None else np.ascontiguousarray(block_mask, dtype=np.uint8)
    rc = lib.oracle_attention_backward(_ptr(q_bits), _ptr(k_bits), _ptr(v_bits), _ptr(do_bits),
                                       B, S, Hq, Hkv, D, float(scale), _ptr(bm), int(block),
                                       _ptr(dq), _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError("oracle_attention_backward rejected its arguments")
    return dq, dk, dv


def attention_backward_qrows(q_bits, k_bits, v_bits, do_bits, scale, rows, block_mask=None,
                             block: int = BLOCK) -> np.ndarray:
    """dQ of selected (b, h, t) rows only (each depends on its own row):
    fp64 [n, D]."""
    lib = _load()
    q_bits, k_bits, v_bits, do_bits = map(_u16, (q_bits, k_bits, v_bits, do_bits))
    B, S, Hq, D = q_bits.shape
    Hkv = k_bits.shape[2]
    rows = np.ascontiguousarray(rows, dtype=np.int64).reshape(-1, 3)
    dq = np.zeros((rows.shape[0], D))
    bm = None if block_mask is None else np.ascontiguousarray(block_mask, dtype=np.uint8)
    rc = lib.oracle_attention_backward_qrows(_ptr(q_bits), _ptr(k_bits), _ptr(v_bits),
                                             _ptr(do_bits), B, S, Hq, Hkv, D, float(scale),
                                             _ptr(bm), int(block), _ptr(rows), rows.shape[0],
                                             _ptr(dq))
    if rc != 0:
        raise ValueError("oracle_attention_backward_qrows rejected its arguments")
    return dq


def attention_backward_keyrows(q_bits, k_bits, v_bits, do_bits, scale, b, kvh, keys,
                               block_mask=None, block: int = BLOCK):
    """dK, dV of selected key positions of one (batch, kv head): fp64 [n, D]
    each (every query row of the group is evaluated in full)."""
    lib = _load()
    q_bits, k_bits, v_bits, do_bits = map(_u16, (q_bits, k_bits, v_bits, do_bits))
    B, S, Hq, D = q_bits.shape
    Hkv = k_bits.shape[2]
    keys = np.ascontiguousarray(keys, dtype=np.int64).ravel()
    dk = np.zeros((keys.size, D))
    dv = np.zeros((keys.size, D))
    bm = None if block_mask is None else np.ascontiguousarray(block_mask, dtype=np.uint8)
    rc = lib.oracle_attention_backward_keyrows(_ptr(q_bits), _ptr(k_bits), _ptr(v_bits),
                                               _ptr(do_bits), B, S, Hq, Hkv, D, float(scale),
                                               _ptr(bm), int(block), int(b), int(kvh),
                                               _ptr(keys), keys.size, _ptr(dk), _ptr(dv))
    if rc != 0:
        raise ValueError("oracle_attention_backward_keyrows rejected its arguments")
    return dk, dv


def router_pool_backward(dx: np.ndarray, S: int, Hq: int, D: int,
                         n_head: int = N_HEAD_TOKENS, n_tail: int = N_TAIL_TOKENS) -> np.ndarray:
    """Gradient of router_pool with respect to Q: each of the n_head + n_tail
    selected tokens receives dx / (n_head + n_tail); every other token 0.
    dx [B, Hq*D] -> fp64 [B, S, Hq, D]."""
    B = dx.shape[0]
    g = np.zeros((B, S, Hq, D))
    share = np.asarray(dx, np.float64).reshape(B, Hq, D) / float(n_head + n_tail)
    g[:, :n_head] += share[:, None]
    g[:, S - n_tail:] += share[:, None]
    return g


def soft_routed_backward(x, w1, b1, w2, b2, gumbel, tau, o_full, o_sparse, dy):
    """Chain rule through the soft-routed layer
        a = W1 x + b1, h = ReLU(a), pi = W2 h + b2, z = pi + g,
        r = softmax(z / tau)[FA],  y = r O_FA + (1 - r) O_SA
    for an upstream dy (all fp64; o_full, o_sparse, dy [B, ...]).  ReLU'(0)
    is taken as 0.  Returns a dict with dr [B], dlogits [B,2], dw1, db1, dw2,
    db2, dx [B, in], and the output weights r [B] that scale dy into the
    upstream gradients of the two attention paths (r dy and (1 - r) dy)."""
    x = np.asarray(x, np.float64)
    w1, b1 = np.asarray(w1, np.float64), np.asarray(b1, np.float64)
    w2, b2 = np.asarray(w2, np.float64), np.asarray(b2, np.float64)
    B = x.shape[0]
    a = x @ w1.T + b1
    h = np.maximum(a, 0.0)
    logits = h @ w2.T + b2
    r = router_soft(logits, gumbel, tau)
    diff = (np.asarray(o_full, np.float64) - np.asarray(o_sparse, np.float64)).reshape(B, -1)
    dr = (np.asarray(dy, np.float64).reshape(B, -1) * diff).sum(axis=1)
    # r = 1 / (1 + exp((z_SA - z_FA) / tau)): dr/dz_FA = r (1 - r) / tau = -dr/dz_SA
    dzf = dr * r * (1.0 - r) / float(tau)
    dlogits = np.stack([dzf, -dzf], axis=1)
    dw2 = dlogits.T @ h
    db2 = dlogits.sum(axis=0)
    dh = dlogits @ w2
    da = dh * (a > 0.0)
    dw1 = da.T @ x
    db1 = da.sum(axis=0)
    dx = da @ w1
    return {"r": r, "dr": dr, "dlogits": dlogits, "dw1": dw1, "db1": db1, "dw2": dw2,
            "db2": db2, "dx": dx}


def decode(q_bits, kc_bits, vc_bits, seqlens, scale, mode=MODE_FULL,
           block=BLOCK, sink=SINK_TOKENS, window=2 * BLOCK):
    """One query token per sequence at position L-1 (L = seqlens[b]).  FULL
    attends keys 0..L-1; SPARSE attends the keys the prefill block rule
    keeps for row L-1 ([FLUX]: a sparse layer does not load the KV blocks
    outside its pattern).  Returns (out fp64 [B,Hq,D], lse fp64 [B,Hq])."""
    lib = _load()
    q_bits = np.ascontiguousarray(q_bits, dtype=np.uint16)
    kc_bits = np.ascontiguousarray(kc_bits, dtype=np.uint16)
    vc_bits = np.ascontiguousarray(vc_bits, dtype=np.uint16)
    B, Hq, D = q_bits.shape
    Lmax, Hkv = kc_bits.shape[1], kc_bits.shape[2]
    seqlens = np.ascontiguousarray(seqlens, dtype=np.int32)
    kbo = None
    if mode == MODE_SPARSE:
        nkb = -(-Lmax // block)
        kbo = np.zeros((B, nkb), dtype=np.uint8)
        for b in range(B):
            L = int(seqlens[b])
            rows = blocksparse_rows(L, block, sink, window)
            kbo[b, rows[-1]] = 1
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    rc = lib.oracle_decode(_ptr(q_bits), _ptr(kc_bits), _ptr(vc_bits), _ptr(seqlens),
                           B, Lmax, Hq, Hkv, D, float(scale), _ptr(kbo), int(block),
                           _ptr(out), _ptr(lse))
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return out, lse


# ------------------------------------------------------- FP8 KV cache codec
# OCP 8-bit floating point E4M3 (the "FN" variant): 1 sign bit, 4 exponent
# bits with bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN; the
# largest finite magnitude is 448 (S.1111.110).  The pages note that their
# B200 kernel is BF16-only; an FP8 cache is the adjacent decode variant.

def e4m3_decode(codes) -> np.ndarray:
    """Exact value of each E4M3 code (uint8) as fp64; NaN codes give NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, -6)
    val = np.where(e == 0, sub, normal)
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


_E4M3_CODES = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
_E4M3_VALUES = e4m3_decode(_E4M3_CODES)


def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 code to each finite value (ties to the even code, i.e.
    mantissa bit 0 clear), saturating at +-448; -0 and +0 keep their sign.
    Brute force over the 254 finite codes."""
    x = np.asarray(x, dtype=np.float64)
    flat = x.ravel()
    out = np.empty(flat.size, dtype=np.uint8)
    for i, v in enumerate(flat):
        if not np.isfinite(v):
            raise ValueError("e4m3_encode takes finite values")
        v = min(max(v, -448.0), 448.0)
        d = np.abs(_E4M3_VALUES - v)
        best = np.flatnonzero(d == d.min())
        cands = _E4M3_CODES[best]
        if len(cands) > 1:           # a tie (or +-0): even mantissa, then the sign of v
            even = cands[(cands & 1) == 0]
            cands = even if len(even) else cands
            if len(cands) > 1:
                cands = cands[((cands & 0x80) != 0) == bool(np.signbit(v))]
        out[i] = cands[0]
    return out.reshape(x.shape)


def kv_quantize(x_bits: np.ndarray, scale) -> np.ndarray:
    """E4M3 codes of a bf16 tensor divided by a per-head scale, the quotient
    rounded to fp32 first (IEEE division): code = RN_e4m3(fp32(x / s)).
    x_bits [..., H, D] bf16 bits; scale [H] fp32."""
    x = bf16_bits_to_f64(x_bits).astype(np.float32)
    s = np.asarray(scale, dtype=np.float32)
    q = (x / s[:, None]).astype(np.float32)
    return e4m3_encode(q.astype(np.float64))


def decode_values(q, k, v, seqlens, scale, mode=MODE_FULL, block=BLOCK, sink=SINK_TOKENS,
                  window=2 * BLOCK):
    """decode() on fp64 values instead of bf16 bits (for dequantized FP8
    caches): q [B,Hq,D], k, v [B,Lmax,Hkv,D].  Same key rule, plain numpy."""
    q, k, v = (np.asarray(a, np.float64) for a in (q, k, v))
    B, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        L = int(seqlens[b])
        if mode == MODE_SPARSE:
            keep = np.zeros(L, bool)
            for j in blocksparse_rows(L, block, sink, window)[-1]:
                keep[j * block:min(L, (j + 1) * block)] = True
        else:
            keep = np.ones(L, bool)
        for h in range(Hq):
            s = (k[b, :L, h // G] @ q[b, h]) * scale
            s = np.where(keep, s, -np.inf)
            m = s.max()
            p = np.exp(s - m)
            out[b, h] = (p @ v[b, :L, h // G]) / p.sum()
            lse[b, h] = m + np.log(p.sum())
    return out, lse


def paged_gather(pages: np.ndarray, block_table: np.ndarray, seqlens, page_size: int = BLOCK):
    """The tokens of each sequence, in order, from a paged cache
    pages [num_pages, page_size, H, D] and block_table [B, max_pages]
    (token t of sequence b sits in page block_table[b, t // page_size] at slot
    t % page_size).  Returns [B, Lmax, H, D] (zeros past each length)."""
    B, max_pages = block_table.shape
    Lmax = max_pages * page_size
    out = np.zeros((B, Lmax) + pages.shape[2:], dtype=pages.dtype)
    for b in range(B):
        for t in range(int(seqlens[b])):
            out[b, t] = pages[block_table[b, t // page_size], t % page_size]
    return out


# --------------------------------------------------------------- accounting
def attended_pairs_full(S: int) -> int:
    """Causal (query, key) pairs of one head: S(S+1)/2."""
    return S * (S + 1) // 2


def attended_pairs_sparse(S, block=BLOCK, sink=SINK_TOKENS, window=2 * BLOCK) -> int:
    """Exact causal (query, key) pairs the block rule keeps, one head."""
    total = 0
    for i, r in enumerate(blocksparse_rows(S, block, sink, window)):
        nq = min(S, (i + 1) * block) - i * block
        for j in r:
            nk = min(S, (j + 1) * block) - j * block
            if j < i:
                total += nq * nk
            else:  # diagonal block: key offset <= query offset
                total += nq * (nq + 1) // 2
    return total
