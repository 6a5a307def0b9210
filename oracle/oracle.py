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


# ---------------------------------------------------------------- context-parallel decode (one long sequence, G ranks)

def rank_ranges(seq_len: int, page_size: int, G: int):
    """Rank r's contiguous range [lo, hi) of a sequence's positions: the
    sequence's pages dealt out in G runs of ceil(pages / G) whole pages (the
    last runs may be short or empty)."""
    pages = -(-int(seq_len) // page_size)
    per = -(-pages // G) if pages else 0
    out = []
    for r in range(G):
        lo = min(r * per * page_size, seq_len)
        hi = min((r + 1) * per * page_size, seq_len)
        out.append((lo, hi))
    return out


def layer_forward_context_parallel(q_idx, w, k_cache, q, kv_cache, gate, pg: Paged, K: int, Dv: int,
                                   sm_scale: float, G: int):
    """The decode layer (query b at the last position of sequence b) with
    every sequence's history split over G ranks by rank_ranges.  Per rank:
    the indexer scores of its own positions and their top-K (candidate
    (score, position) pairs).  The union of the G lists, under the top-K's
    order (score descending, position ascending, -0 equal to +0), cut to K
    and sorted by position, is the selection -- the same as one device's,
    because a position among the K best of the whole history is among the K
    best of its own range.  Per rank: attention over the selected rows it
    holds, giving (out_r, lse_r); the output is sum_r exp(lse_r - L) out_r
    with L = logsumexp_r lse_r (the gate, one factor per (token, head), is
    common to every rank's term).  Returns (idx [B, K], out [B, H, Dv])."""
    q_idx = _c(q_idx, np.uint8)
    B = q_idx.shape[0]
    P = pg.page_size
    seq_lens = pg.seq_lens
    assert B == pg.num_seqs
    cand_s = [[] for _ in range(B)]
    cand_p = [[] for _ in range(B)]
    ranges = [rank_ranges(int(seq_lens[b]), P, G) for b in range(B)]
    locals_ = []
    for r in range(G):
        lo = np.array([ranges[b][r][0] for b in range(B)], np.int64)
        hi = np.array([ranges[b][r][1] for b in range(B)], np.int64)
        n = (hi - lo).astype(np.int32)
        # the rank's own block table: the sequences' pages from lo on (lo is page-aligned)
        bt = np.full(pg.block_table.shape, -1, np.int32)
        for b in range(B):
            nb = -(-int(n[b]) // P)
            bt[b, :nb] = pg.block_table[b, lo[b] // P: lo[b] // P + nb]
        pr = Paged(n, bt, P, pg.num_pages)
        locals_.append((lo, hi, pr))
        live = np.nonzero(n > 0)[0]
        if len(live) == 0:
            continue
        ld = int(n.max())
        sc = indexer_scores(q_idx[live], _c(w, np.float32)[live], k_cache, pr, live.astype(np.int32),
                            (n[live] - 1).astype(np.int32), ld=ld)
        kept = topk(sc, n[live], K)
        for i, b in enumerate(live):
            sel = kept[i][kept[i] >= 0]
            cand_s[b].append(sc[i, sel])
            cand_p[b].append(sel.astype(np.int64) + lo[b])
    idx = np.full((B, K), -1, np.int32)
    for b in range(B):
        s = np.concatenate(cand_s[b]) if cand_s[b] else np.zeros(0, np.float32)
        p = np.concatenate(cand_p[b]) if cand_p[b] else np.zeros(0, np.int64)
        order = np.lexsort((p, -s.astype(np.float64)))[:K]  # score descending, then position ascending
        keep = np.sort(p[order])
        idx[b, :len(keep)] = keep
    H = _c(q, np.uint16).shape[1]
    outs, lses = [], []
    for lo, hi, pr in locals_:
        li = np.where((idx >= lo[:, None]) & (idx < hi[:, None]), idx - lo[:, None], -1).astype(np.int32)
        o, l = sparse_attn(q, kv_cache, pr, np.arange(B, dtype=np.int32), li, gate, sm_scale, Dv, return_lse=True)
        outs.append(o)
        lses.append(l)
    lse = np.stack(lses)                                    # [G, B, H]
    m = lse.max(axis=0)
    wgt = np.where(np.isneginf(lse), 0.0, np.exp(lse - np.where(np.isneginf(m), 0.0, m)))
    out = (wgt[..., None] * np.stack(outs)).sum(axis=0) / np.maximum(wgt.sum(axis=0), 1e-300)[..., None]
    return idx, out
