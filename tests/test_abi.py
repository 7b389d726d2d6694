"""The C-ABI library builds, loads, exports every declared symbol, and rejects
bad arguments on the host (no GPU needed: these calls return before any CUDA
call)."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_layerrouter_b200 import build, capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa_hybrid.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return capi.lib()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FA_API\s+[\w\s\*]*?\b(fa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("fa_router_decide", "fa_blocksparse_index", "fa_attn_prefill_full",
                 "fa_attn_prefill_blocksparse", "fa_attn_decode", "fa_hybrid_layer"):
        assert name in syms
    assert set(syms) == set(capi.EXPORTED)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.fa_version() == 100


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, 7):
        assert capi.status_string(code)
    assert "INVALID" in capi.status_string(-1)


def test_index_size_matches_oracle_counts(lib):
    import oracle
    for S, W in ((1024, 128), (8192, 1024), (32768, 2048), (262144, 4096), (65, 128), (1, 64)):
        rows, nnz = capi.blocksparse_index_size(S, capi.cfg(64, 128, W))
        rp, ci = oracle.blocksparse_csr(S, 64, 128, W)
        assert rows == len(rp) - 1 and nnz == len(ci)


@pytest.mark.parametrize("cfgv,expect", [((64, 128, 32), -1), ((64, 100, 128), -1),
                                         ((32, 128, 128), -2), ((0, 128, 128), -1),
                                         ((64, -64, 128), -1)])
def test_index_size_rejects_bad_cfg(lib, cfgv, expect):
    rows, nnz = ctypes.c_int(0), ctypes.c_int(0)
    rc = lib.fa_blocksparse_index_size(1024, capi.cfg(*cfgv), ctypes.byref(rows), ctypes.byref(nnz))
    assert rc == expect


def test_prefill_rejects_on_host(lib):
    p = ctypes.c_void_p(4096)            # aligned, never dereferenced
    bad = ctypes.c_void_p(4096 + 8)      # misaligned
    f = lib.fa_attn_prefill_full
    assert f(None, p, p, p, None, 1, 128, 4, 4, 128, 0.1, None, None) == -1     # null q
    assert f(bad, p, p, p, None, 1, 128, 4, 4, 128, 0.1, None, None) == -1      # misaligned
    assert f(p, p, p, p, None, 1, 128, 4, 3, 128, 0.1, None, None) == -1        # Hq % Hkv
    assert f(p, p, p, p, None, 1, 128, 4, 4, 64, 0.1, None, None) == -2         # D != 128
    assert f(p, p, p, p, None, 0, 128, 4, 4, 128, 0.1, None, None) == -1        # B = 0
    assert f(p, p, p, p, None, 1, 0, 4, 4, 128, 0.1, None, None) == -1          # S = 0
    assert f(p, p, p, p, None, 1, 128, 4, 4, 128, 0.0, None, None) == -1        # scale
    g = lib.fa_attn_prefill_blocksparse
    assert g(p, p, p, p, None, 1, 128, 4, 4, 128, 0.1, None, p, 64, None, None) == -1
    assert g(p, p, p, p, None, 1, 128, 4, 4, 128, 0.1, p, p, 32, None, None) == -2


def test_decode_and_router_reject_on_host(lib):
    p = ctypes.c_void_p(4096)
    c = capi.cfg(64, 128, 2048)
    d = lib.fa_attn_decode
    ws = lib.fa_decode_workspace_size(8, 32, 8, 131072, 128)
    assert ws > 0
    assert lib.fa_decode_workspace_size(8, 32, 7, 131072, 128) == 0
    assert d(p, p, p, p, 8, 131072, 32, 8, 128, 0.1, 0, None, c, p, None, p, ws - 1, None,
             None) == -3
    assert d(p, p, p, p, 8, 131072, 32, 8, 128, 0.1, 2, None, c, p, None, p, ws, None, None) == -1
    assert d(p, p, p, p, 8, 131072, 48, 3, 128, 0.1, 0, None, c, p, None, p, ws, None, None) == -2
    r = lib.fa_router_decide
    wsr = lib.fa_router_workspace_size(1, 32, 128, 256)
    assert wsr >= 32 * 128 * 4 + 256 * 4
    assert r(p, 1, 199, 32, 128, 100, 100, p, None, 256, p, None, p, p, p, wsr, None) == -2
    assert r(p, 1, 8192, 32, 128, 100, 100, p, None, 256, p, None, p, p, p, wsr - 4, None) == -3
    assert r(p, 1, 8192, 32, 128, 100, 100, None, None, 256, p, None, p, p, p, wsr, None) == -1
    h = lib.fa_hybrid_layer
    assert h(p, p, p, p, None, 1, 8192, 32, 8, 128, 0.1, p, None, 256, p, None, c, None, p, p, p,
             p, wsr, None, None) == -1


def test_product_path_has_no_cpu_fallback(monkeypatch, tmp_path):
    """With the library missing, the binding raises instead of computing."""
    monkeypatch.setattr(capi, "_lib", None)
    monkeypatch.setattr(capi, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not found"):
        capi.lib()


# ---- host-side checks of the backward, paged/FP8 decode and soft-mix entries
_P = ctypes.c_void_p(16)      # an aligned non-null pointer that is never dereferenced
_N = None


def test_backward_entries_reject_on_host(lib):
    b = lib.fa_attn_prefill_backward
    args = [_P] * 9 + [1, 256, 4, 2, 128, 0.088, _N, _N, _N, 0, _P, 1 << 30, _N, _N]
    assert b(*args[:3], _N, *args[4:]) == -1                  # o missing
    bad = list(args); bad[13] = 64                             # D != 128
    assert b(*bad) == -2
    bad = list(args); bad[18] = 1                              # SPARSE without a CSR
    assert b(*bad) == -1
    bad = list(args); bad[20] = 16                             # workspace too small
    assert b(*bad) == -3
    assert lib.fa_attn_backward_workspace_size(1, 256, 4, 2, 128) > 4 * 256 * 4 * 128
    assert lib.fa_attn_backward_workspace_size(1, 256, 4, 3, 128) == 0
    assert lib.fa_soft_routed_backward_workspace_size(1, 256, 4, 2, 128, 64) > \
        lib.fa_attn_backward_workspace_size(1, 256, 4, 2, 128)


def test_paged_decode_entries_reject_on_host(lib):
    c = capi.cfg(64, 128, 256)
    d = lib.fa_attn_decode_paged
    good = [_P, _P, _P, 0, _N, _N, _P, 4, 8, _P, 2, 8, 2, 128, 0.088, 0, _N, c, _P, _N, _P,
            1 << 30, _N, _N]
    bad = list(good); bad[3] = 7                               # unknown cache type
    assert d(*bad) == -1
    bad = list(good); bad[3] = 1                               # FP8 without scales
    assert d(*bad) == -1
    bad = list(good); bad[11] = 7                              # Hq % Hkv != 0
    assert d(*bad) == -1
    bad = list(good); bad[21] = 8                              # workspace too small
    assert d(*bad) == -3
    assert lib.fa_decode_paged_workspace_size(2, 8, 2, 4, 128) == \
        lib.fa_decode_workspace_size(2, 8, 2, 256, 128)
    a = lib.fa_kv_append_paged
    assert a(_P, _P, _P, _P, 0, _N, _N, _P, 4, 8, _P, 2, 2, 64, _N, _N) == -2   # D != 128
    assert a(_P, _P, _P, _P, 1, _N, _N, _P, 4, 8, _P, 2, 2, 128, _N, _N) == -1  # FP8, no scales
    assert a(_P, _P, _P, _P, 0, _N, _N, _N, 4, 8, _P, 2, 2, 128, _N, _N) == -1  # no block table


def test_soft_mix_rejects_on_host(lib):
    assert lib.fa_soft_mix(_P, _P, _P, _N, 1, 8, 2, 128, _N) == -1
    assert lib.fa_soft_mix(_P, _P, _P, _P, 1, 8, 2, 64, _N) == -2


def test_host_rejections_launch_nothing(lib):
    """The launch counter is host-side (readable without a GPU) and calls
    rejected by their host-side checks add nothing to it."""
    before = capi.kernel_launches()
    p = ctypes.c_void_p(4096)
    c = capi.cfg(64, 128, 2048)
    assert lib.fa_attn_prefill_full(None, p, p, p, None, 1, 128, 4, 4, 128, 0.1, None,
                                    None) == -1
    ws = lib.fa_decode_workspace_size(8, 32, 8, 131072, 128)
    assert lib.fa_attn_decode(p, p, p, p, 8, 131072, 32, 8, 128, 0.1, 0, None, c, p, None, p,
                              ws - 1, None, None) == -3
    assert capi.kernel_launches() == before
