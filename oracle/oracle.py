"""CPU oracle for the Gated DSA layer -- TEST INFRASTRUCTURE ONLY.

Thin ctypes front end over ``oracle.c`` (plain C, fp64).  Only the test
suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this module; the product path never does.  Nothing here shares code
with the CUDA library.

Arrays are numpy; 8-bit float and bfloat16 tensors travel as their raw bit
patterns (``uint8`` / ``uint16``), which the C side decodes from the format
definitions.  See ``oracle.c`` for the passages each function follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    L = ctypes.c_int64
    D = ctypes.c_double
    lib.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
    lib.orc_e4m3_to_f64.restype = D
    lib.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.orc_bf16_to_f64.restype = D
    lib.orc_e4m3_from_f64.argtypes = [D]
    lib.orc_e4m3_from_f64.restype = ctypes.c_uint8
    lib.orc_append_kv.argtypes = [P, ctypes.c_float, P, P, P, I, P, P, I, I, I, I, I, I, P, P]
    lib.orc_append_kv.restype = I
    lib.orc_indexer_scores.argtypes = [P, P, P, P, P, I, I, I, I, P, P, I, I, I, P, L]
    lib.orc_e8m0_to_f64.argtypes = [ctypes.c_uint8]
    lib.orc_e8m0_to_f64.restype = D
    lib.orc_mx_encode.argtypes = [P, L, P, P]
    lib.orc_mx_encode.restype = I
    lib.orc_append_kv_mx.argtypes = [P, P, P, P, I, P, P, I, I, I, I, I, I, P, P, P]
    lib.orc_append_kv_mx.restype = I
    lib.orc_indexer_scores_mx.argtypes = [P, P, P, P, P, P, P, I, I, I, I, P, P, I, I, I, P, L]
    lib.orc_indexer_scores_mx.restype = I
    lib.orc_topk.argtypes = [P, L, P, I, I, P]
    lib.orc_sparse_attn.argtypes = [P, P, P, P, I, I, I, I, P, P, I, P, D, I, I, I, I, P, P]
    lib.orc_swa_decode.argtypes = [P, P, P, P, I, I, I, I, D, P]
    lib.orc_layer_forward.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, P, P,
                                      I, I, I, I, I, I, I, D, P, L, P, P]
    for f in ("orc_indexer_scores", "orc_topk", "orc_sparse_attn", "orc_swa_decode",
              "orc_layer_forward"):
        getattr(lib, f).restype = I
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB)
    return _lib


class use_library:
    """Temporarily route every call through another build of the oracle
    (used by the tests that plant mistakes in a copy of oracle.c)."""

    def __init__(self, path: str):
        self.path = path

    def __enter__(self):
        global _lib
        _load()
        self._saved = _lib
        _lib = _bind(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._saved
        return False


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: bad input (code {rc})")


def e4m3_to_f64(code: int) -> float:
    return _load().orc_e4m3_to_f64(int(code))


def bf16_to_f64(code: int) -> float:
    return _load().orc_bf16_to_f64(int(code))


def e4m3_from_f64(x: float) -> int:
    return int(_load().orc_e4m3_from_f64(float(x)))


class Paged:
    """Paged-cache geometry: seq_lens [B], block_table [B, max_blocks]."""

    def __init__(self, seq_lens, block_table, page_size: int, num_pages: int):
        self.seq_lens = _c(seq_lens, np.int32)
        self.block_table = _c(block_table, np.int32)
        assert self.block_table.ndim == 2
        self.num_seqs = int(self.seq_lens.shape[0])
        self.max_blocks = int(self.block_table.shape[1])
        self.page_size = int(page_size)
        self.num_pages = int(num_pages)

    def args(self):
        return (_p(self.seq_lens), _p(self.block_table), self.num_seqs, self.max_blocks,
                self.page_size, self.num_pages)


def indexer_scores(q_idx, w, k_cache, pg: Paged, q_seq, q_pos, ld=None, fill=-np.inf):
    """Scores [T, ld] fp32; entries past each query's position hold ``fill``."""
    q_idx = _c(q_idx, np.uint8)
    T, HI, DI = q_idx.shape
    w = _c(w, np.float32).reshape(T, HI)
    k_cache = _c(k_cache, np.uint8)
    q_seq = _c(q_seq, np.int32)
    q_pos = _c(q_pos, np.int32)
    if ld is None:
        ld = int(q_pos.max()) + 1 if T else 1
    scores = np.full((T, ld), fill, dtype=np.float32)
    rc = _load().orc_indexer_scores(_p(q_idx), _p(w), _p(k_cache), *pg.args(), _p(q_seq),
                                    _p(q_pos), T, HI, DI, _p(scores), ld)
    _check(rc, "indexer_scores")
    return scores


def topk(scores, row_len, K: int):
    scores = _c(scores, np.float32)
    R, ld = scores.shape
    row_len = _c(row_len, np.int32)
    idx = np.empty((R, K), dtype=np.int32)
    rc = _load().orc_topk(_p(scores), ld, _p(row_len), R, K, _p(idx))
    _check(rc, "topk")
    return idx


def sparse_attn(q, kv_cache, pg: Paged, q_seq, idx, gate, sm_scale: float, Dv: int,
                return_lse: bool = False):
    q = _c(q, np.uint16)
    T, H, Dqk = q.shape
    kv_cache = _c(kv_cache, np.uint16)
    q_seq = _c(q_seq, np.int32)
    idx = _c(idx, np.int32)
    K = idx.shape[1]
    gate = _c(gate, np.uint16).reshape(T, H)
    out = np.empty((T, H, Dv), dtype=np.float64)
    lse = np.empty((T, H), dtype=np.float64)
    rc = _load().orc_sparse_attn(_p(q), _p(kv_cache), *pg.args(), _p(q_seq), _p(idx), K,
                                 _p(gate), float(sm_scale), T, H, Dqk, Dv, _p(out), _p(lse))
    _check(rc, "sparse_attn")
    return (out, lse) if return_lse else out


def swa_decode(q, k_ring, v_ring, seq_lens, window: int, sm_scale: float):
    q = _c(q, np.uint16)
    B, H, D = q.shape
    k_ring = _c(k_ring, np.uint16)
    v_ring = _c(v_ring, np.uint16)
    assert k_ring.shape == (B, window, H, D) and v_ring.shape == k_ring.shape
    seq_lens = _c(seq_lens, np.int32)
    out = np.empty((B, H, D), dtype=np.float64)
    rc = _load().orc_swa_decode(_p(q), _p(k_ring), _p(v_ring), _p(seq_lens), B, H, D, window,
                                float(sm_scale), _p(out))
    _check(rc, "swa_decode")
    return out


def layer_forward(q_idx, w, k_cache, q, kv_cache, gate, pg: Paged, q_seq, q_pos, K: int,
                  Dv: int, sm_scale: float):
    """Returns (scores, idx, out)."""
    q_idx = _c(q_idx, np.uint8)
    T, HI, DI = q_idx.shape
    q = _c(q, np.uint16)
    _, H, Dqk = q.shape
    w = _c(w, np.float32).reshape(T, HI)
    q_seq = _c(q_seq, np.int32)
    q_pos = _c(q_pos, np.int32)
    ld = int(q_pos.max()) + 1 if T else 1
    scores = np.full((T, ld), -np.inf, dtype=np.float32)
    idx = np.empty((T, K), dtype=np.int32)
    out = np.empty((T, H, Dv), dtype=np.float64)
    rc = _load().orc_layer_forward(_p(q_idx), _p(w), _p(_c(k_cache, np.uint8)), _p(q),
                                   _p(_c(kv_cache, np.uint16)), _p(_c(gate, np.uint16)),
                                   *pg.args(), _p(q_seq), _p(q_pos), T, HI, DI, K, H, Dqk, Dv,
                                   float(sm_scale), _p(scores), ld, _p(idx), _p(out))
    _check(rc, "layer_forward")
    return scores, idx, out


def append_kv(k_new, k_scale: float, latent_new, tok_seq, tok_pos, pg: Paged, k_cache, kv_cache):
    """Returns copies of (k_cache, kv_cache) with the new tokens written in."""
    k_new = _c(k_new, np.uint16)
    n, DI = k_new.shape
    k_cache = _c(k_cache, np.uint8).copy()
    kv_cache = _c(kv_cache, np.uint16).copy()
    Dqk = kv_cache.shape[-1]
    lat = None if latent_new is None else _c(latent_new, np.uint16)
    rc = _load().orc_append_kv(_p(k_new), float(k_scale), None if lat is None else _p(lat),
                               _p(_c(tok_seq, np.int32)), _p(_c(tok_pos, np.int32)), n, *pg.args(), DI, Dqk,
                               _p(k_cache), _p(kv_cache))
    _check(rc, "append_kv")
    return k_cache, kv_cache


# ---------------------------------------------------------------- MXFP8 (blocks of 32, E8M0 scales)

MX_BLOCK = 32


def e8m0_to_f64(code: int) -> float:
    return _load().orc_e8m0_to_f64(int(code))


def mx_encode(x):
    """x float64 [..., n], n a multiple of 32: (E4M3 codes [..., n], E8M0 scales [..., n/32])."""
    x = _c(x, np.float64)
    n = x.shape[-1]
    if n % MX_BLOCK:
        raise ValueError("last dimension must be a multiple of 32")
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty(x.shape[:-1] + (n // MX_BLOCK,), dtype=np.uint8)
    rc = _load().orc_mx_encode(_p(x), x.size // MX_BLOCK, _p(codes), _p(scales))
    _check(rc, "mx_encode")
    return codes, scales


def mx_decode(codes, scales):
    """Values of MXFP8 blocks (float64), from the oracle's own decoders."""
    codes = np.asarray(codes, dtype=np.uint8)
    scales = np.asarray(scales, dtype=np.uint8)
    lib = _load()
    ev = np.array([lib.orc_e4m3_to_f64(c) for c in range(256)])
    sv = np.array([lib.orc_e8m0_to_f64(c) for c in range(256)])
    return ev[codes] * np.repeat(sv[scales], MX_BLOCK, axis=-1)


def append_kv_mx(k_new, latent_new, tok_seq, tok_pos, pg: Paged, k_cache, k_scales, kv_cache):
    """Returns copies of (k_cache, k_scales, kv_cache) with the new tokens written in."""
    k_new = _c(k_new, np.uint16)
    n, DI = k_new.shape
    k_cache = _c(k_cache, np.uint8).copy()
    k_scales = _c(k_scales, np.uint8).copy()
    kv_cache = _c(kv_cache, np.uint16).copy()
    Dqk = kv_cache.shape[-1]
    lat = None if latent_new is None else _c(latent_new, np.uint16)
    rc = _load().orc_append_kv_mx(_p(k_new), None if lat is None else _p(lat), _p(_c(tok_seq, np.int32)),
                                  _p(_c(tok_pos, np.int32)), n, *pg.args(), DI, Dqk, _p(k_cache),
                                  _p(k_scales), _p(kv_cache))
    _check(rc, "append_kv_mx")
    return k_cache, k_scales, kv_cache


def indexer_scores_mx(q_idx, q_scales, w, k_cache, k_scales, pg: Paged, q_seq, q_pos, ld=None, fill=-np.inf):
    """MXFP8 indexer scores [T, ld] fp32; q_scales [T, HI, DI/32], k_scales [pages, page_size, DI/32]."""
    q_idx = _c(q_idx, np.uint8)
    T, HI, DI = q_idx.shape
    q_scales = _c(q_scales, np.uint8).reshape(T, HI, DI // MX_BLOCK)
    w = _c(w, np.float32).reshape(T, HI)
    k_cache = _c(k_cache, np.uint8)
    k_scales = _c(k_scales, np.uint8)
    if k_scales.size * MX_BLOCK != k_cache.size:
        raise ValueError("k_scales must hold one scale per 32 key elements")
    q_seq = _c(q_seq, np.int32)
    q_pos = _c(q_pos, np.int32)
    if ld is None:
        ld = int(q_pos.max()) + 1 if T else 1
    scores = np.full((T, ld), fill, dtype=np.float32)
    rc = _load().orc_indexer_scores_mx(_p(q_idx), _p(q_scales), _p(w), _p(k_cache), _p(k_scales), *pg.args(),
                                       _p(q_seq), _p(q_pos), T, HI, DI, _p(scores), ld)
    _check(rc, "indexer_scores_mx")
    return scores
