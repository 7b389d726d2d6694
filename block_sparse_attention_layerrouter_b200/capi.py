"""ctypes binding of libfa_hybrid.so, one function per C-ABI entry point.

Argument marshalling only: every function checks dtypes, devices and
contiguity, takes ``data_ptr()`` and the current CUDA stream, calls the C entry
point of the same name and raises :class:`FaError` on a non-zero status.
Every step of the computation runs in the library's CUDA kernels; there is no
fallback.  Outputs and workspaces are allocated with torch when the caller
does not pass them (torch is the memory and stream plumbing only).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa_hybrid.so")

FA_OK = 0
FA_MODE_FULL = 0
FA_MODE_SPARSE = 1
FA_DEV_TIMEOUT = 1
FA_DEV_BAD_INDEX = 2
FA_DEV_DEBUG_BOUNDS = 4


class FaError(RuntimeError):
    def __init__(self, name: str, status: int, text: str):
        super().__init__("%s failed: %s (status %d)" % (name, text, status))
        self.status = status


class SparseCfg(ctypes.Structure):
    """fa_sparse_cfg: block, sink and window in tokens."""
    _fields_ = [("block", ctypes.c_int32), ("sink", ctypes.c_int32), ("window", ctypes.c_int32)]


_lib = None
_VP = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

_SIGNATURES = {
    "fa_status_string": (ctypes.c_char_p, [_I]),
    "fa_version": (_I, []),
    "fa_kernel_launches": (ctypes.c_ulonglong, []),
    "fa_debug_set_wait_limit_ns": (_I, [ctypes.c_ulonglong]),
    "fa_router_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "fa_router_decide": (_I, [_VP, _I, _I, _I, _I, _I, _I, _VP, _VP, _I, _VP, _VP, _VP, _VP,
                              _VP, _SZ, _VP]),
    "fa_blocksparse_index_size": (_I, [_I, SparseCfg, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    "fa_blocksparse_index": (_I, [_I, SparseCfg, _VP, _VP, _VP]),
    "fa_attn_prefill_full": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _VP, _VP]),
    "fa_attn_prefill_blocksparse": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _VP,
                                         _VP, _I, _VP, _VP]),
    "fa_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_attn_decode": (_I, [_VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP, SparseCfg, _VP,
                            _VP, _VP, _SZ, _VP, _VP]),
    "fa_noalloc_scratch_bytes": (_SZ, []),
    "fa_attn_decode_noalloc": (_I, [_VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _I, _VP,
                                    SparseCfg, _VP, _VP, _VP, _VP]),
    "fa_varlen_workspace_size": (_SZ, [_I, _I]),
    "fa_attn_prefill_varlen": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP,
                                    _VP, _VP, _I, _VP, _SZ, _VP, _VP]),
    "fa_hybrid_varlen_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_hybrid_layer_varlen": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _VP,
                                    _VP, _I, _VP, _VP, SparseCfg, _VP, _VP, _VP, _VP, _VP, _SZ,
                                    _VP, _VP]),
    "fa_router_soft": (_I, [_VP, _VP, _I, _F, _VP, _VP]),
    "fa_soft_routed_layer": (_I, [_VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _VP, _VP, _I, _VP,
                                  _VP, _VP, _F, SparseCfg, _VP, _VP, _VP, _VP, _VP, _SZ, _VP,
                                  _VP]),
    "fa_attn_backward_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_attn_prefill_backward": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I,
                                      _I, _F, _VP, _VP, _VP, _I, _VP, _SZ, _VP, _VP]),
    "fa_soft_routed_backward_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "fa_soft_routed_layer_backward": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I,
                                           _I, _F, _VP, _VP, _I, _VP, _VP, _VP, _F, _VP, _VP, _VP,
                                           _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP,
                                           _VP]),
    "fa_kv_append_paged": (_I, [_VP, _VP, _VP, _VP, _I, _VP, _VP, _VP, _I, _I, _VP, _I, _I, _I,
                                _VP, _VP]),
    "fa_decode_paged_workspace_size": (_SZ, [_I, _I, _I, _I, _I]),
    "fa_attn_decode_paged": (_I, [_VP, _VP, _VP, _I, _VP, _VP, _VP, _I, _I, _VP, _I, _I, _I, _I,
                                  _F, _I, _VP, SparseCfg, _VP, _VP, _VP, _SZ, _VP, _VP]),
    "fa_soft_mix": (_I, [_VP, _VP, _VP, _VP, _I, _I, _I, _I, _VP]),
    "fa_hybrid_workspace_size": (_SZ, [_I, _I, _I, _I]),
    "fa_hybrid_layer": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _F, _VP, _VP, _I, _VP,
                             _VP, SparseCfg, _VP, _VP, _VP, _VP, _VP, _SZ, _VP, _VP]),
}
EXPORTED = tuple(_SIGNATURES)


def lib():
    """Load the library (once).  Raises if it was not built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                "libfa_hybrid.so not found at %s: build it with "
                "`python -m block_sparse_attention_layerrouter_b200.build`" % LIB_PATH)
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def use_library(path: str) -> str:
    """Load the library at `path` from now on (e.g. the debug build,
    libfa_hybrid_debug.so, whose kernels bounds-check their output stores);
    returns the path in use before."""
    global _lib, LIB_PATH
    old = LIB_PATH
    LIB_PATH = path
    _lib = None
    return old


def status_string(status: int) -> str:
    return lib().fa_status_string(int(status)).decode()


def kernel_launches() -> int:
    """Kernels this library has enqueued in this process so far (host-side
    count; no GPU access)."""
    return int(lib().fa_kernel_launches())


def debug_set_wait_limit_ns(ns: int):
    """fa_debug_set_wait_limit_ns: the bound of every wait inside the kernels
    on the current device (default 2e9 ns).  A testing aid: a short bound
    makes the kernels give up and report FA_DEV_TIMEOUT."""
    _check("fa_debug_set_wait_limit_ns", lib().fa_debug_set_wait_limit_ns(int(ns)))


def _check(name: str, rc: int):
    if rc != FA_OK:
        raise FaError(name, rc, status_string(rc))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, dim: int):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (no CPU path exists)" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if t.dim() != dim:
        raise ValueError("%s must have %d dims, got %d" % (name, dim, t.dim()))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def cfg(block: int = 64, sink: int = 128, window: int = 128) -> SparseCfg:
    return SparseCfg(block, sink, window)


# ------------------------------------------------------------------ router
def router_workspace_size(B, Hq, D, hidden) -> int:
    return int(lib().fa_router_workspace_size(B, Hq, D, hidden))


def router_decide(q, w1, b1, w2, b2, n_head=100, n_tail=100, logits=None, mode=None,
                  workspace=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """fa_router_decide.  q bf16 [B,S,Hq,D]; fp32 weights on q's device."""
    _need(q, "q", torch.bfloat16, 4)
    B, S, Hq, D = q.shape
    hidden = w1.shape[0]
    for t, n in ((w1, "w1"), (w2, "w2")):
        _need(t, n, torch.float32, 2)
    for t, n in ((b1, "b1"), (b2, "b2")):
        if t is not None:
            _need(t, n, torch.float32, 1)
    dev = q.device
    logits = torch.empty(B, 2, device=dev, dtype=torch.float32) if logits is None else logits
    mode = torch.empty(B, device=dev, dtype=torch.int32) if mode is None else mode
    ws_bytes = router_workspace_size(B, Hq, D, hidden)
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    rc = lib().fa_router_decide(_ptr(q), B, S, Hq, D, n_head, n_tail, _ptr(w1), _ptr(b1), hidden,
                                _ptr(w2), _ptr(b2), _ptr(logits), _ptr(mode), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), _stream(dev))
    _check("fa_router_decide", rc)
    return logits, mode


# ------------------------------------------------------------------- index
def blocksparse_index_size(S: int, c: SparseCfg) -> Tuple[int, int]:
    rows, nnz = ctypes.c_int(0), ctypes.c_int(0)
    _check("fa_blocksparse_index_size",
           lib().fa_blocksparse_index_size(S, c, ctypes.byref(rows), ctypes.byref(nnz)))
    return rows.value, nnz.value


def blocksparse_index(S: int, c: SparseCfg, device="cuda"):
    """fa_blocksparse_index -> (row_ptr int32 [n+1], col_idx int32 [nnz]) on device."""
    rows, nnz = blocksparse_index_size(S, c)
    dev = torch.device(device)
    row_ptr = torch.empty(rows + 1, device=dev, dtype=torch.int32)
    col_idx = torch.empty(max(nnz, 1), device=dev, dtype=torch.int32)
    _check("fa_blocksparse_index",
           lib().fa_blocksparse_index(S, c, _ptr(row_ptr), _ptr(col_idx), _stream(dev)))
    return row_ptr, col_idx[:nnz]


# ----------------------------------------------------------------- prefill
def _prefill_common(q, k, v, o, lse):
    _need(q, "q", torch.bfloat16, 4)
    _need(k, "k", torch.bfloat16, 4)
    _need(v, "v", torch.bfloat16, 4)
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, S, Hkv, D) or v.shape != k.shape:
        raise ValueError("k/v must be [B, S, Hkv, D] matching q")
    o = torch.empty_like(q) if o is None else o
    _need(o, "o", torch.bfloat16, 4)
    if lse is not None:
        _need(lse, "lse", torch.float32, 3)
    return B, S, Hq, Hkv, D, o


def attn_prefill_full(q, k, v, scale=None, o=None, lse=None, status=None) -> torch.Tensor:
    B, S, Hq, Hkv, D, o = _prefill_common(q, k, v, o, lse)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib().fa_attn_prefill_full(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, S, Hq, Hkv,
                                    D, scale, _ptr(status), _stream(q.device))
    _check("fa_attn_prefill_full", rc)
    return o


def attn_prefill_blocksparse(q, k, v, row_ptr, col_idx, block=64, scale=None, o=None, lse=None,
                             status=None) -> torch.Tensor:
    B, S, Hq, Hkv, D, o = _prefill_common(q, k, v, o, lse)
    _need(row_ptr, "row_ptr", torch.int32, 1)
    _need(col_idx, "col_idx", torch.int32, 1)
    if row_ptr.numel() != -(-S // block) + 1:
        raise ValueError("row_ptr must have ceil(S/block)+1 entries")
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    rc = lib().fa_attn_prefill_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, S,
                                           Hq, Hkv, D, scale, _ptr(row_ptr), _ptr(col_idx), block,
                                           _ptr(status), _stream(q.device))
    _check("fa_attn_prefill_blocksparse", rc)
    return o


# ------------------------------------------------------------------ decode
def decode_workspace_size(B, Hq, Hkv, Lmax, D=128) -> int:
    return int(lib().fa_decode_workspace_size(B, Hq, Hkv, Lmax, D))


def attn_decode(q, kcache, vcache, seqlens, mode=FA_MODE_FULL, c: Optional[SparseCfg] = None,
                scale=None, mode_dev=None, o=None, lse=None, workspace=None,
                status=None) -> torch.Tensor:
    _need(q, "q", torch.bfloat16, 3)
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(seqlens, "seqlens", torch.int32, 1)
    B, Hq, D = q.shape
    Lmax, Hkv = kcache.shape[1], kcache.shape[2]
    if vcache.shape != kcache.shape or kcache.shape[0] != B or kcache.shape[3] != D:
        raise ValueError("caches must be [B, Lmax, Hkv, D] matching q")
    c = cfg() if c is None else c
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = torch.empty_like(q) if o is None else o
    ws_bytes = decode_workspace_size(B, Hq, Hkv, Lmax, D)
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), device=q.device, dtype=torch.uint8)
    rc = lib().fa_attn_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), B, Lmax, Hq,
                              Hkv, D, scale, int(mode), _ptr(mode_dev), c, _ptr(o), _ptr(lse),
                              _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _ptr(status), _stream(q.device))
    _check("fa_attn_decode", rc)
    return o


def attn_decode_noalloc(q, kcache, vcache, seqlens, mode=FA_MODE_FULL,
                        c: Optional[SparseCfg] = None, scale=None, mode_dev=None, o=None,
                        lse=None, status=None) -> torch.Tensor:
    """fa_attn_decode_noalloc: decode with the library's static scratch (for
    callers that cannot allocate a workspace).  Raises ValueError when the
    shape needs more scratch than the library holds."""
    _need(q, "q", torch.bfloat16, 3)
    _need(kcache, "kcache", torch.bfloat16, 4)
    _need(vcache, "vcache", torch.bfloat16, 4)
    _need(seqlens, "seqlens", torch.int32, 1)
    B, Hq, D = q.shape
    Lmax, Hkv = kcache.shape[1], kcache.shape[2]
    need = decode_workspace_size(B, Hq, Hkv, Lmax, D)
    cap = int(lib().fa_noalloc_scratch_bytes())
    if need > cap:
        raise ValueError("decode needs %d bytes of scratch; the static scratch holds %d"
                         % (need, cap))
    c = cfg() if c is None else c
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = torch.empty_like(q) if o is None else o
    rc = lib().fa_attn_decode_noalloc(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(seqlens), B,
                                      Lmax, Hq, Hkv, D, scale, int(mode), _ptr(mode_dev), c,
                                      _ptr(o), _ptr(lse), _ptr(status), _stream(q.device))
    _check("fa_attn_decode_noalloc", rc)
    return o


# ------------------------------------------------------------------ hybrid
def hybrid_workspace_size(B, Hq, D, hidden) -> int:
    return int(lib().fa_hybrid_workspace_size(B, Hq, D, hidden))


def hybrid_layer(q, k, v, w1, b1, w2, b2, row_ptr, col_idx, c: SparseCfg, scale=None, o=None,
                 lse=None, logits=None, mode=None, workspace=None, status=None):
    """fa_hybrid_layer -> (o, logits, mode)."""
    B, S, Hq, Hkv, D, o = _prefill_common(q, k, v, o, lse)
    hidden = w1.shape[0]
    dev = q.device
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    logits = torch.empty(B, 2, device=dev, dtype=torch.float32) if logits is None else logits
    mode = torch.empty(B, device=dev, dtype=torch.int32) if mode is None else mode
    ws_bytes = hybrid_workspace_size(B, Hq, D, hidden)
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    rc = lib().fa_hybrid_layer(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, S, Hq, Hkv, D,
                               scale, _ptr(w1), _ptr(b1), hidden, _ptr(w2), _ptr(b2), c,
                               _ptr(row_ptr), _ptr(col_idx), _ptr(logits), _ptr(mode),
                               _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _ptr(status), _stream(dev))
    _check("fa_hybrid_layer", rc)
    return o, logits, mode


# ------------------------------------------------------------ soft routing
def router_soft(logits, gumbel=None, tau=1.0, r=None) -> torch.Tensor:
    """fa_router_soft: weight of the FULL output per sequence."""
    _need(logits, "logits", torch.float32, 2)
    if gumbel is not None:
        _need(gumbel, "gumbel", torch.float32, 2)
    B = logits.shape[0]
    r = torch.empty(B, device=logits.device, dtype=torch.float32) if r is None else r
    _check("fa_router_soft", lib().fa_router_soft(_ptr(logits), _ptr(gumbel), B, float(tau),
                                                  _ptr(r), _stream(logits.device)))
    return r


def soft_routed_layer(q, k, v, w1, b1, w2, b2, row_ptr, col_idx, c: SparseCfg, gumbel=None,
                      tau=1.0, scale=None, o=None, logits=None, r=None, workspace=None,
                      status=None):
    """fa_soft_routed_layer -> (y, logits, r)."""
    B, S, Hq, Hkv, D, o = _prefill_common(q, k, v, o, None)
    hidden = w1.shape[0]
    dev = q.device
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    logits = torch.empty(B, 2, device=dev, dtype=torch.float32) if logits is None else logits
    r = torch.empty(B, device=dev, dtype=torch.float32) if r is None else r
    if gumbel is not None:
        _need(gumbel, "gumbel", torch.float32, 2)
    ws_bytes = hybrid_workspace_size(B, Hq, D, hidden)
    if workspace is None:
        workspace = torch.empty(ws_bytes, device=dev, dtype=torch.uint8)
    rc = lib().fa_soft_routed_layer(_ptr(q), _ptr(k), _ptr(v), _ptr(o), B, S, Hq, Hkv, D, scale,
                                    _ptr(w1), _ptr(b1), hidden, _ptr(w2), _ptr(b2), _ptr(gumbel),
                                    float(tau), c, _ptr(row_ptr), _ptr(col_idx), _ptr(logits),
                                    _ptr(r), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(status),
                                    _stream(dev))
    _check("fa_soft_routed_layer", rc)
    return o, logits, r


# --------------------------------------------------- variable-length batch
def _varlen_common(q, k, v, cu_seqlens, o, lse):
    _need(q, "q", torch.bfloat16, 3)
    _need(k, "k", torch.bfloat16, 3)
    _need(v, "v", torch.bfloat16, 3)
    _need(cu_seqlens, "cu_seqlens", torch.int32, 1)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    if k.shape != (T, Hkv, D) or v.shape != k.shape:
        raise ValueError("k/v must be [total_tokens, Hkv, D] matching q")
    o = torch.empty_like(q) if o is None else o
    _need(o, "o", torch.bfloat16, 3)
    if lse is not None:
        _need(lse, "lse", torch.float32, 2)
    return T, Hq, Hkv, D, cu_seqlens.numel() - 1, o


def attn_prefill_varlen(q, k, v, cu_seqlens, max_seqlen, row_ptr=None, col_idx=None,
                        mode=FA_MODE_FULL, mode_dev=None, scale=None, o=None, lse=None,
                        workspace=None, status=None) -> torch.Tensor:
    """fa_attn_prefill_varlen: packed sequences [total_tokens, H, D]."""
    T, Hq, Hkv, D, B, o = _varlen_common(q, k, v, cu_seqlens, o, lse)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    if workspace is None:
        workspace = torch.empty(int(lib().fa_varlen_workspace_size(B, T)), device=q.device,
                                dtype=torch.uint8)
    rc = lib().fa_attn_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                      _ptr(cu_seqlens), B, T, int(max_seqlen), Hq, Hkv, D, scale,
                                      _ptr(row_ptr), _ptr(col_idx), _ptr(mode_dev), int(mode),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _ptr(status), _stream(q.device))
    _check("fa_attn_prefill_varlen", rc)
    return o


def hybrid_layer_varlen(q, k, v, cu_seqlens, max_seqlen, w1, b1, w2, b2, row_ptr, col_idx,
                        c: SparseCfg, scale=None, o=None, lse=None, logits=None, mode=None,
                        workspace=None, status=None):
    """fa_hybrid_layer_varlen -> (o, logits, mode)."""
    T, Hq, Hkv, D, B, o = _varlen_common(q, k, v, cu_seqlens, o, lse)
    hidden = w1.shape[0]
    dev = q.device
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    logits = torch.empty(B, 2, device=dev, dtype=torch.float32) if logits is None else logits
    mode = torch.empty(B, device=dev, dtype=torch.int32) if mode is None else mode
    if workspace is None:
        workspace = torch.empty(int(lib().fa_hybrid_varlen_workspace_size(B, T, Hq, D, hidden)),
                                device=dev, dtype=torch.uint8)
    rc = lib().fa_hybrid_layer_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse),
                                      _ptr(cu_seqlens), B, T, int(max_seqlen), Hq, Hkv, D, scale,
                                      _ptr(w1), _ptr(b1), hidden, _ptr(w2), _ptr(b2), c,
                                      _ptr(row_ptr), _ptr(col_idx), _ptr(logits), _ptr(mode),
                                      _ptr(workspace), workspace.numel() * workspace.element_size(),
                                      _ptr(status), _stream(dev))
    _check("fa_hybrid_layer_varlen", rc)
    return o, logits, mode


# ------------------------------------------------------------------ backward
def attn_backward_workspace_size(B, S, Hq, Hkv, D=128) -> int:
    return int(lib().fa_attn_backward_workspace_size(B, S, Hq, Hkv, D))


def attn_prefill_backward(q, k, v, o, lse, dout, row_ptr=None, col_idx=None, mode=FA_MODE_FULL,
                          mode_dev=None, scale=None, dq=None, dk=None, dv=None, workspace=None,
                          status=None):
    """fa_attn_prefill_backward -> (dq, dk, dv), bf16 like q, k, v."""
    B, S, Hq, Hkv, D, o = _prefill_common(q, k, v, o, None)
    _need(dout, "dout", torch.bfloat16, 4)
    _need(lse, "lse", torch.float32, 3)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    if workspace is None:
        workspace = torch.empty(attn_backward_workspace_size(B, S, Hq, Hkv, D), device=q.device,
                                dtype=torch.uint8)
    rc = lib().fa_attn_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                        _ptr(dq), _ptr(dk), _ptr(dv), B, S, Hq, Hkv, D, scale,
                                        _ptr(row_ptr), _ptr(col_idx), _ptr(mode_dev), int(mode),
                                        _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _ptr(status), _stream(q.device))
    _check("fa_attn_prefill_backward", rc)
    return dq, dk, dv


def soft_routed_layer_backward(q, k, v, o_full, lse_full, o_sparse, lse_sparse, dy, w1, b1, w2,
                               b2, row_ptr, col_idx, gumbel=None, tau=1.0, scale=None,
                               workspace=None, status=None):
    """fa_soft_routed_layer_backward -> dict of dq, dk, dv (bf16), dw1, db1,
    dw2, db2 (fp32) and r."""
    B, S, Hq, Hkv, D, _ = _prefill_common(q, k, v, o_full, None)
    _need(dy, "dy", torch.bfloat16, 4)
    hidden = w1.shape[0]
    dev = q.device
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = {"dq": torch.empty_like(q), "dk": torch.empty_like(k), "dv": torch.empty_like(v),
           "dw1": torch.empty_like(w1), "db1": torch.empty(hidden, device=dev),
           "dw2": torch.empty_like(w2), "db2": torch.empty(2, device=dev),
           "r": torch.empty(B, device=dev)}
    if workspace is None:
        workspace = torch.empty(int(lib().fa_soft_routed_backward_workspace_size(B, S, Hq, Hkv, D,
                                                                                 hidden)),
                                device=dev, dtype=torch.uint8)
    rc = lib().fa_soft_routed_layer_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o_full), _ptr(lse_full), _ptr(o_sparse), _ptr(lse_sparse),
        _ptr(dy), B, S, Hq, Hkv, D, scale, _ptr(w1), _ptr(b1), hidden, _ptr(w2), _ptr(b2),
        _ptr(gumbel), float(tau), _ptr(row_ptr), _ptr(col_idx), _ptr(out["dq"]), _ptr(out["dk"]),
        _ptr(out["dv"]), _ptr(out["dw1"]), _ptr(out["db1"]), _ptr(out["dw2"]), _ptr(out["db2"]),
        _ptr(out["r"]), _ptr(workspace), workspace.numel() * workspace.element_size(),
        _ptr(status), _stream(dev))
    _check("fa_soft_routed_layer_backward", rc)
    return out


# ----------------------------------------------------- paged / FP8 KV cache
FA_KV_BF16 = 0
FA_KV_FP8_E4M3 = 1


def kv_append_paged(k_new, v_new, k_pages, v_pages, block_table, seqlens, kv_dtype=FA_KV_BF16,
                    k_scale=None, v_scale=None, status=None):
    """fa_kv_append_paged: writes the token at seqlens[b], then seqlens += 1
    (in place, on the device)."""
    _need(k_new, "k_new", torch.bfloat16, 3)
    _need(v_new, "v_new", torch.bfloat16, 3)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seqlens, "seqlens", torch.int32, 1)
    B, Hkv, D = k_new.shape
    num_pages = k_pages.shape[0]
    rc = lib().fa_kv_append_paged(_ptr(k_new), _ptr(v_new), _ptr(k_pages), _ptr(v_pages),
                                  int(kv_dtype), _ptr(k_scale), _ptr(v_scale), _ptr(block_table),
                                  block_table.shape[1], num_pages, _ptr(seqlens), B, Hkv, D,
                                  _ptr(status), _stream(k_new.device))
    _check("fa_kv_append_paged", rc)


def decode_paged_workspace_size(B, Hq, Hkv, max_pages, D=128) -> int:
    return int(lib().fa_decode_paged_workspace_size(B, Hq, Hkv, max_pages, D))


def attn_decode_paged(q, k_pages, v_pages, block_table, seqlens, kv_dtype=FA_KV_BF16,
                      k_scale=None, v_scale=None, mode=FA_MODE_FULL, c: Optional[SparseCfg] = None,
                      mode_dev=None, scale=None, o=None, lse=None, workspace=None, status=None):
    """fa_attn_decode_paged: q bf16 [B,Hq,D]; pools [num_pages,64,Hkv,D]."""
    _need(q, "q", torch.bfloat16, 3)
    _need(block_table, "block_table", torch.int32, 2)
    _need(seqlens, "seqlens", torch.int32, 1)
    B, Hq, D = q.shape
    num_pages, page, Hkv = k_pages.shape[0], k_pages.shape[1], k_pages.shape[2]
    if page != 64:
        raise ValueError("pages hold 64 tokens")
    max_pages = block_table.shape[1]
    c = cfg() if c is None else c
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = torch.empty_like(q) if o is None else o
    if workspace is None:
        workspace = torch.empty(decode_paged_workspace_size(B, Hq, Hkv, max_pages, D),
                                device=q.device, dtype=torch.uint8)
    rc = lib().fa_attn_decode_paged(_ptr(q), _ptr(k_pages), _ptr(v_pages), int(kv_dtype),
                                    _ptr(k_scale), _ptr(v_scale), _ptr(block_table), max_pages,
                                    num_pages, _ptr(seqlens), B, Hq, Hkv, D, scale, int(mode),
                                    _ptr(mode_dev), c, _ptr(o), _ptr(lse), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _ptr(status),
                                    _stream(q.device))
    _check("fa_attn_decode_paged", rc)
    return o


def soft_mix(o_full, o_sparse, r, y=None) -> torch.Tensor:
    """fa_soft_mix: y = r O_FA + (1 - r) O_SA per sequence (bf16)."""
    _need(o_full, "o_full", torch.bfloat16, 4)
    _need(o_sparse, "o_sparse", torch.bfloat16, 4)
    _need(r, "r", torch.float32, 1)
    B, S, Hq, D = o_full.shape
    y = torch.empty_like(o_full) if y is None else y
    _check("fa_soft_mix", lib().fa_soft_mix(_ptr(o_full), _ptr(o_sparse), _ptr(r), _ptr(y), B, S,
                                            Hq, D, _stream(o_full.device)))
    return y
