"""The C-ABI library loads and exports every entry point its header declares;
host-side argument checks reject bad calls before touching the GPU (no GPU
needed: these paths return before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dsa.h")


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_02_b200 import build
    build.build()
    from long_context_sparse_02_b200 import _lib
    return _lib


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:dsa_status|size_t|const char \*|int32_t)\s*(dsa_\w+)\s*\(", src, re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("dsa_indexer_scores", "dsa_topk", "dsa_sparse_attn", "dsa_layer_forward", "dsa_swa_decode",
                 "dsa_layer_workspace_bytes", "dsa_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib.lib, name), name
    assert set(declared_functions()) <= set(lib.EXPORTS) | {"dsa_abi_version"}


def test_status_strings_and_version(lib):
    assert lib.lib.dsa_abi_version() == 2
    assert lib.lib.dsa_status_string(0) == b"ok"
    assert lib.lib.dsa_status_string(3).startswith(b"workspace")


def _paged(num_seqs=1, page_size=64, num_pages=4):
    P = ctypes.c_void_p
    return lib_paged(P(16), P(32), num_seqs, 4, page_size, num_pages)


def lib_paged(*a):
    from long_context_sparse_02_b200._lib import Paged
    return Paged(*a)


def test_host_side_argument_errors(lib):
    L = lib.lib
    P = ctypes.c_void_p
    ok_pg = lib_paged(P(256), P(512), 2, 4, 64, 8)
    bad_pg = lib_paged(P(256), P(512), 2, 4, 32, 8)   # page size must be 64
    # indexer: unsupported head count, bad page size, q_seq without q_pos, ld < max_len
    assert L.dsa_indexer_scores(P(16), P(16), P(16), ctypes.byref(ok_pg), None, None, 2, 12, 128, 10, P(16), 16,
                                None) == 2
    assert L.dsa_indexer_scores(P(16), P(16), P(16), ctypes.byref(bad_pg), None, None, 2, 16, 128, 10, P(16), 16,
                                None) == 1
    assert L.dsa_indexer_scores(P(16), P(16), P(16), ctypes.byref(ok_pg), P(16), None, 2, 16, 128, 10, P(16), 16,
                                None) == 1
    assert L.dsa_indexer_scores(P(16), P(16), P(16), ctypes.byref(ok_pg), None, None, 2, 16, 128, 10, P(16), 8,
                                None) == 1
    # decode convention needs T <= num_seqs
    assert L.dsa_indexer_scores(P(16), P(16), P(16), ctypes.byref(ok_pg), None, None, 3, 16, 128, 10, P(16), 16,
                                None) == 1
    # top-K: K too large, ld < max_row_len
    assert L.dsa_topk(P(16), 100, P(16), 4, 5000, 100, P(16), None, 0, None) == 2
    assert L.dsa_topk(P(16), 50, P(16), 4, 8, 100, P(16), None, 0, None) == 1
    # attention: K not a multiple of 64, unsupported dims, too many heads, misaligned q
    assert L.dsa_sparse_attn(P(16), P(16), ctypes.byref(ok_pg), None, P(16), 100, P(16), 1.0, 2, 8, 64, 64, P(16),
                             None, None, 0, None) == 2
    assert L.dsa_sparse_attn(P(16), P(16), ctypes.byref(ok_pg), None, P(16), 128, P(16), 1.0, 2, 8, 128, 128, P(16),
                             None, None, 0, None) == 2
    assert L.dsa_sparse_attn(P(16), P(16), ctypes.byref(ok_pg), None, P(16), 128, P(16), 1.0, 2, 256, 64, 64, P(16),
                             None, None, 0, None) == 2
    assert L.dsa_sparse_attn(P(18), P(16), ctypes.byref(ok_pg), None, P(16), 128, P(16), 1.0, 2, 8, 64, 64, P(16),
                             None, None, 0, None) == 1
    # SWA: unsupported head dim / window
    assert L.dsa_swa_decode(P(16), P(16), P(16), P(16), 2, 8, 64, 128, 1.0, P(16), None) == 2
    assert L.dsa_swa_decode(P(16), P(16), P(16), P(16), 2, 8, 128, 64, 1.0, P(16), None) == 2
    # layer: bad mode, decode with T != num_seqs
    from long_context_sparse_02_b200._lib import LayerArgs
    a = LayerArgs()
    a.mode = 7
    assert L.dsa_layer_forward(ctypes.byref(a), None, 0, None) == 1
    a.mode = 1
    a.pg = ok_pg
    a.T, a.HI, a.DI, a.K, a.H, a.Dqk, a.Dv, a.max_len, a.sm_scale = 3, 16, 128, 128, 8, 64, 64, 100, 0.1
    assert L.dsa_layer_forward(ctypes.byref(a), None, 0, None) == 1
    # append: unsupported key width, non-finite scale, bad page size, misaligned keys, missing latent cache
    assert L.dsa_append_kv(P(16), 1.0, None, P(16), P(16), ctypes.byref(ok_pg), 2, 96, 0, P(16), None, None) == 2
    assert L.dsa_append_kv(P(16), float("nan"), None, P(16), P(16), ctypes.byref(ok_pg), 2, 128, 0, P(16), None,
                           None) == 1
    assert L.dsa_append_kv(P(16), 1.0, None, P(16), P(16), ctypes.byref(bad_pg), 2, 128, 0, P(16), None, None) == 1
    assert L.dsa_append_kv(P(18), 1.0, None, P(16), P(16), ctypes.byref(ok_pg), 2, 128, 0, P(16), None, None) == 1
    assert L.dsa_append_kv(P(16), 1.0, P(16), P(16), P(16), ctypes.byref(ok_pg), 2, 128, 576, P(16), None,
                           None) == 1
    assert L.dsa_append_kv(P(16), 1.0, P(16), P(16), P(16), ctypes.byref(ok_pg), 2, 128, 570, P(16), P(16),
                           None) == 2
    # zero-sized calls are no-ops
    assert L.dsa_append_kv(None, 1.0, None, None, None, ctypes.byref(ok_pg), 0, 128, 0, None, None, None) == 0
    assert L.dsa_topk(P(16), 10, P(16), 0, 8, 10, P(16), None, 0, None) == 0
    # histogram-fed top-K: bad K, ld below the row length, misaligned scores, no histogram, no workspace
    assert L.dsa_topk_hist(P(16), 100, P(16), 4, 5000, 100, P(16), P(16), None, 0, None) == 2
    assert L.dsa_topk_hist(P(16), 50, P(16), 4, 8, 100, P(16), P(16), None, 0, None) == 1
    assert L.dsa_topk_hist(P(20), 100, P(16), 4, 8, 100, P(16), P(16), None, 0, None) == 1
    assert L.dsa_topk_hist(P(16), 100, P(16), 4, 8, 100, None, P(16), None, 0, None) == 1
    assert L.dsa_topk_hist(P(16), 100, P(16), 4, 8, 100, P(16), P(16), None, 0, None) == 3
    assert L.dsa_topk_hist(P(16), 10, P(16), 0, 8, 10, P(16), P(16), None, 0, None) == 0


def test_layer_workspace_follows_the_documented_layout(lib):
    """dsa_layer_workspace_bytes (host only) adds up the regions dsa.h lists:
    the per-query score histogram (2048 bins of 4 bytes, in decode and for
    T <= 64), the fp32 score rows (ld = max_len rounded up to 4), the idx rows
    when idx_out is NULL, then the top-K scratch (the histogram-fed top-K's
    whenever the histogram is there) and the attention scratch; each of the
    first three regions 256-byte aligned.  runtime.LayerOnDevice.scores reads
    the score rows behind that histogram region."""
    from long_context_sparse_02_b200._lib import LayerArgs
    L = lib.lib

    def ws(mode, T, max_len, idx_out=None, K=2048, H=128, Dv=512):
        a = LayerArgs()
        a.mode, a.T, a.max_len, a.K, a.H, a.Dv, a.HI, a.DI, a.Dqk = mode, T, max_len, K, H, Dv, 32, 128, 576
        a.idx_out = idx_out
        return L.dsa_layer_workspace_bytes(ctypes.byref(a))

    def up(n):
        return (n + 255) // 256 * 256

    for T in (1, 8, 64, 65, 300):
        for mode in (0, 1):
            for max_len in (1, 1000, 131072):
                base = ws(mode, T, max_len, idx_out=ctypes.c_void_p(16))
                assert ws(mode, T, max_len) - base == up(T * 2048 * 4)
                hist = up(T * 2048 * 4) if (mode == 1 or T <= 64) else 0
                rows = up(T * ((max_len + 3) // 4 * 4) * 4)
                topk = L.dsa_topk_hist_workspace_bytes(T, max_len) if hist else \
                    L.dsa_topk_workspace_bytes(T, 2048, max_len)
                scratch = topk + L.dsa_sparse_attn_workspace_bytes(T, 128, 2048, 512)
                assert base == hist + rows + scratch, (T, mode, max_len)
    assert ws(1, 65, 1000) - ws(0, 65, 1000) == up(65 * 2048 * 4) + L.dsa_topk_hist_workspace_bytes(65, 1000) - \
        L.dsa_topk_workspace_bytes(65, 2048, 1000)
    assert ws(0, 0, 10) == 0 and ws(0, 4, 0) == 0 and ws(0, 4, 10, K=0) == 0
