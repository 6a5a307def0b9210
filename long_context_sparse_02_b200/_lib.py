"""ctypes binding of libdsa.so.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Functions take torch CUDA tensors, check dtype, device and layout,
pass raw pointers and the current CUDA stream, and raise DsaError on a
non-zero status.  Importing this module without the built library raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

DSA_OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace missing or too small",
          4: "CUDA error", 5: "device wait timed out"}
DEVERR_POSITION, DEVERR_PAGE, DEVERR_TIMEOUT, DEVERR_SHAPE = 1, 2, 4, 8
MODE_PREFILL, MODE_DECODE = 0, 1


class DsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {STATUS.get(status, status)} (status {status})")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"libdsa.so is not built ({LIB_PATH}); run long_context_sparse_02_b200/build.py")

lib = ctypes.CDLL(LIB_PATH)

P = ctypes.c_void_p
I32 = ctypes.c_int32
I64 = ctypes.c_int64
SZ = ctypes.c_size_t
F32 = ctypes.c_float


class Paged(ctypes.Structure):
    _fields_ = [("seq_lens", P), ("block_table", P), ("num_seqs", I32), ("max_blocks_per_seq", I32),
                ("page_size", I32), ("num_pages", I32)]


class LayerArgs(ctypes.Structure):
    _fields_ = [("mode", I32), ("q_idx", P), ("w", P), ("k_idx_cache", P), ("q", P), ("kv_cache", P),
                ("gate", P), ("pg", Paged), ("q_seq", P), ("q_pos", P), ("T", I32), ("HI", I32), ("DI", I32),
                ("K", I32), ("H", I32), ("Dqk", I32), ("Dv", I32), ("max_len", I32), ("sm_scale", F32),
                ("out", P), ("idx_out", P), ("lse", P), ("q_idx_scales", P), ("k_idx_scales", P)]


lib.dsa_abi_version.restype = I32
lib.dsa_abi_version.argtypes = []
lib.dsa_status_string.restype = ctypes.c_char_p
lib.dsa_status_string.argtypes = [ctypes.c_int]
lib.dsa_device_error.restype = ctypes.c_int
lib.dsa_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), I32]
lib.dsa_indexer_scores.restype = ctypes.c_int
lib.dsa_indexer_scores.argtypes = [P, P, P, ctypes.POINTER(Paged), P, P, I32, I32, I32, I32, P, I64, P]
lib.dsa_indexer_scores_mx.restype = ctypes.c_int
lib.dsa_indexer_scores_mx.argtypes = [P, P, P, P, P, ctypes.POINTER(Paged), P, P, I32, I32, I32, I32, P, I64, P]
lib.dsa_append_kv_mx.restype = ctypes.c_int
lib.dsa_append_kv_mx.argtypes = [P, P, P, P, ctypes.POINTER(Paged), I32, I32, I32, P, P, P, P]
lib.dsa_topk_workspace_bytes.restype = SZ
lib.dsa_topk_workspace_bytes.argtypes = [I32, I32, I32]
lib.dsa_topk.restype = ctypes.c_int
lib.dsa_topk.argtypes = [P, I64, P, I32, I32, I32, P, P, SZ, P]
lib.dsa_topk_hist_workspace_bytes.restype = SZ
lib.dsa_topk_hist_workspace_bytes.argtypes = [I32, I32]
lib.dsa_topk_hist.restype = ctypes.c_int
lib.dsa_topk_hist.argtypes = [P, I64, P, I32, I32, I32, P, P, P, SZ, P]
lib.dsa_topk_static.restype = ctypes.c_int
lib.dsa_topk_static.argtypes = [P, I64, P, I32, I32, I32, P, P]
lib.dsa_sparse_attn_workspace_bytes.restype = SZ
lib.dsa_sparse_attn_workspace_bytes.argtypes = [I32, I32, I32, I32]
lib.dsa_sparse_attn.restype = ctypes.c_int
lib.dsa_sparse_attn.argtypes = [P, P, ctypes.POINTER(Paged), P, P, I32, P, F32, I32, I32, I32, I32, P, P, P,
                                SZ, P]
lib.dsa_layer_workspace_bytes.restype = SZ
lib.dsa_layer_workspace_bytes.argtypes = [ctypes.POINTER(LayerArgs)]
lib.dsa_layer_forward.restype = ctypes.c_int
lib.dsa_layer_forward.argtypes = [ctypes.POINTER(LayerArgs), P, SZ, P]
lib.dsa_layer_forward_profiled.restype = ctypes.c_int
lib.dsa_layer_forward_profiled.argtypes = [ctypes.POINTER(LayerArgs), P, SZ, ctypes.POINTER(P), P]
lib.dsa_layer_kernel_launches.restype = I32
lib.dsa_append_kv.restype = ctypes.c_int
lib.dsa_append_kv.argtypes = [P, F32, P, P, P, ctypes.POINTER(Paged), I32, I32, I32, P, P, P]
lib.dsa_layer_kernel_launches.argtypes = [ctypes.POINTER(LayerArgs)]
lib.dsa_cp_candidates.restype = ctypes.c_int
lib.dsa_cp_candidates.argtypes = [P, I64, P, I32, I32, P, P, P, P]
lib.dsa_cp_select_workspace_bytes.restype = SZ
lib.dsa_cp_select_workspace_bytes.argtypes = [I32, I32, I32]
lib.dsa_cp_select.restype = ctypes.c_int
lib.dsa_cp_select.argtypes = [P, P, I32, I32, I32, P, P, P, P, P, SZ, P]
lib.dsa_cp_lse_merge.restype = ctypes.c_int
lib.dsa_cp_lse_merge.argtypes = [P, P, I32, I32, I32, I32, P, P]
lib.dsa_test_skip_indexer_tile.restype = ctypes.c_int
lib.dsa_test_skip_indexer_tile.argtypes = [I64]
lib.dsa_swa_decode.restype = ctypes.c_int
lib.dsa_swa_decode.argtypes = [P, P, P, P, I32, I32, I32, I32, F32, P, P]

EXPORTS = ["dsa_abi_version", "dsa_status_string", "dsa_device_error", "dsa_indexer_scores", "dsa_indexer_scores_mx",
           "dsa_append_kv_mx",
           "dsa_topk_workspace_bytes", "dsa_topk", "dsa_topk_hist_workspace_bytes", "dsa_topk_hist", "dsa_topk_static", "dsa_sparse_attn_workspace_bytes",
           "dsa_sparse_attn",
           "dsa_layer_workspace_bytes", "dsa_layer_forward", "dsa_layer_forward_profiled",
           "dsa_layer_kernel_launches", "dsa_swa_decode", "dsa_append_kv", "dsa_cp_candidates",
           "dsa_cp_select_workspace_bytes", "dsa_cp_select", "dsa_cp_lse_merge",
           "dsa_test_skip_indexer_tile"]


def _check(fn: str, status: int):
    if status != DSA_OK:
        raise DsaError(fn, status)


def _ptr(t, dtype, name, nullable=False):
    if t is None:
        if nullable:
            return None
        raise ValueError(f"{name} is required")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def paged(seq_lens: torch.Tensor, block_table: torch.Tensor, num_pages: int, page_size: int = 64) -> Paged:
    """The C struct holds raw pointers, so it also keeps the two tensors alive."""
    pg = Paged(_ptr(seq_lens, torch.int32, "seq_lens"), _ptr(block_table, torch.int32, "block_table"),
               int(seq_lens.shape[0]), int(block_table.shape[1]), int(page_size), int(num_pages))
    pg._tensors = (seq_lens, block_table)
    return pg


def device_error(reset: bool = True) -> int:
    code = ctypes.c_uint32(0)
    _check("dsa_device_error", lib.dsa_device_error(ctypes.byref(code), 1 if reset else 0))
    return int(code.value)


def indexer_scores(q_idx, w, k_cache, pg: Paged, q_seq, q_pos, max_len: int, scores):
    """q_idx uint8 [T,HI,DI]; w fp32 [T,HI]; k_cache uint8 [pages,64,DI];
    q_seq/q_pos int32 [T] or None (decode); scores fp32 [T, ld]."""
    T, HI, DI = q_idx.shape
    _check("dsa_indexer_scores", lib.dsa_indexer_scores(
        _ptr(q_idx, torch.uint8, "q_idx"), _ptr(w, torch.float32, "w"), _ptr(k_cache, torch.uint8, "k_cache"),
        ctypes.byref(pg), _ptr(q_seq, torch.int32, "q_seq", True), _ptr(q_pos, torch.int32, "q_pos", True),
        T, HI, DI, int(max_len), _ptr(scores, torch.float32, "scores"), int(scores.shape[1]), _stream()))
    return scores


def topk_workspace_bytes(R: int, K: int, max_row_len: int) -> int:
    return int(lib.dsa_topk_workspace_bytes(R, K, max_row_len))


def topk(scores, row_len, K: int, max_row_len: int, idx=None, ws=None):
    R, ld = scores.shape
    if idx is None:
        idx = torch.empty((R, K), dtype=torch.int32, device=scores.device)
    need = topk_workspace_bytes(R, K, max_row_len)
    if ws is None and need:
        ws = torch.empty(need, dtype=torch.uint8, device=scores.device)
    _check("dsa_topk", lib.dsa_topk(
        _ptr(scores, torch.float32, "scores"), ld, _ptr(row_len, torch.int32, "row_len"), R, K, int(max_row_len),
        _ptr(idx, torch.int32, "idx"), _ptr(ws, torch.uint8, "ws", True), need if ws is None else ws.numel(),
        _stream()))
    return idx


def topk_hist(scores, row_len, hist, K: int, max_row_len: int, idx=None, ws=None):
    """hist uint32 (as torch.int32) [R, 2048]: counts of key(score) >> 21 per row; zeroed by the call."""
    R, ld = scores.shape
    if idx is None:
        idx = torch.empty((R, K), dtype=torch.int32, device=scores.device)
    need = int(lib.dsa_topk_hist_workspace_bytes(R, int(max_row_len)))
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=scores.device)
    _check("dsa_topk_hist", lib.dsa_topk_hist(
        _ptr(scores, torch.float32, "scores"), ld, _ptr(row_len, torch.int32, "row_len"), R, K, int(max_row_len),
        _ptr(hist, torch.int32, "hist"), _ptr(idx, torch.int32, "idx"), _ptr(ws, torch.uint8, "ws"), ws.numel(),
        _stream()))
    return idx


def sparse_attn_workspace_bytes(T: int, H: int, K: int, Dv: int) -> int:
    return int(lib.dsa_sparse_attn_workspace_bytes(T, H, K, Dv))


def sparse_attn(q, kv_cache, pg: Paged, q_seq, idx, gate, sm_scale: float, Dv: int, out=None, lse=None, ws=None):
    """q bf16 [T,H,Dqk]; kv_cache bf16 [pages,64,Dqk]; idx int32 [T,K]; gate bf16 [T,H]."""
    T, H, Dqk = q.shape
    K = idx.shape[1]
    if out is None:
        out = torch.empty((T, H, Dv), dtype=torch.bfloat16, device=q.device)
    need = sparse_attn_workspace_bytes(T, H, K, Dv)
    if ws is None and need:
        ws = torch.empty(need, dtype=torch.uint8, device=q.device)
    _check("dsa_sparse_attn", lib.dsa_sparse_attn(
        _ptr(q, torch.bfloat16, "q"), _ptr(kv_cache, torch.bfloat16, "kv_cache"), ctypes.byref(pg),
        _ptr(q_seq, torch.int32, "q_seq", True), _ptr(idx, torch.int32, "idx"), K,
        _ptr(gate, torch.bfloat16, "gate"), float(sm_scale), T, H, Dqk, Dv, _ptr(out, torch.bfloat16, "out"),
        _ptr(lse, torch.float32, "lse", True), _ptr(ws, torch.uint8, "ws", True),
        need if ws is None else ws.numel(), _stream()))
    return out


def layer_args(mode, q_idx, w, k_cache, q, kv_cache, gate, pg: Paged, q_seq, q_pos, K: int, Dv: int,
               sm_scale: float, max_len: int, out, idx_out=None, lse=None, q_scales=None,
               k_scales=None) -> LayerArgs:
    T, HI, DI = q_idx.shape
    _, H, Dqk = q.shape
    a = LayerArgs(int(mode), _ptr(q_idx, torch.uint8, "q_idx"), _ptr(w, torch.float32, "w"),
                     _ptr(k_cache, torch.uint8, "k_cache"), _ptr(q, torch.bfloat16, "q"),
                     _ptr(kv_cache, torch.bfloat16, "kv_cache"), _ptr(gate, torch.bfloat16, "gate"), pg,
                     _ptr(q_seq, torch.int32, "q_seq", True), _ptr(q_pos, torch.int32, "q_pos", True),
                     T, HI, DI, int(K), H, Dqk, int(Dv), int(max_len), float(sm_scale),
                     _ptr(out, torch.bfloat16, "out"), _ptr(idx_out, torch.int32, "idx_out", True),
                     _ptr(lse, torch.float32, "lse", True), _ptr(q_scales, torch.uint8, "q_scales", True),
                     _ptr(k_scales, torch.uint8, "k_scales", True))
    a._tensors = (q_idx, w, k_cache, q, kv_cache, gate, getattr(pg, "_tensors", None), q_seq, q_pos, out, idx_out,
                  lse, q_scales, k_scales)
    return a


def layer_workspace_bytes(args: LayerArgs) -> int:
    return int(lib.dsa_layer_workspace_bytes(ctypes.byref(args)))


def layer_kernel_launches(args: LayerArgs) -> int:
    return int(lib.dsa_layer_kernel_launches(ctypes.byref(args)))


def layer_forward(args: LayerArgs, ws: torch.Tensor):
    _check("dsa_layer_forward", lib.dsa_layer_forward(ctypes.byref(args), _ptr(ws, torch.uint8, "ws"),
                                                      ws.numel(), _stream()))


def layer_forward_profiled(args: LayerArgs, ws: torch.Tensor, events):
    """events: four recorded-once torch.cuda.Event objects (or None)."""
    arr = (P * 4)(*[P(e.cuda_event) if e is not None else P(0) for e in events])
    _check("dsa_layer_forward_profiled", lib.dsa_layer_forward_profiled(
        ctypes.byref(args), _ptr(ws, torch.uint8, "ws"), ws.numel(), arr, _stream()))


def swa_decode(q, k_ring, v_ring, seq_lens, window: int, sm_scale: float, out=None):
    B, H, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    _check("dsa_swa_decode", lib.dsa_swa_decode(
        _ptr(q, torch.bfloat16, "q"), _ptr(k_ring, torch.bfloat16, "k_ring"), _ptr(v_ring, torch.bfloat16, "v_ring"),
        _ptr(seq_lens, torch.int32, "seq_lens"), B, H, D, int(window), float(sm_scale),
        _ptr(out, torch.bfloat16, "out"), _stream()))
    return out


def append_kv(k_new, k_scale: float, latent_new, tok_seq, tok_pos, pg: Paged, k_cache, kv_cache):
    """k_new bf16 [n, DI]; latent_new bf16 [n, Dqk] or None; tok_seq/tok_pos int32 [n];
    k_cache uint8 (e4m3) [pages, 64, DI] and kv_cache bf16 [pages, 64, Dqk], written in place."""
    n, DI = k_new.shape
    Dqk = int(kv_cache.shape[-1]) if kv_cache is not None else 0
    _check("dsa_append_kv", lib.dsa_append_kv(
        _ptr(k_new, torch.bfloat16, "k_new"), float(k_scale), _ptr(latent_new, torch.bfloat16, "latent_new", True),
        _ptr(tok_seq, torch.int32, "tok_seq"), _ptr(tok_pos, torch.int32, "tok_pos"), ctypes.byref(pg), n, DI, Dqk,
        _ptr(k_cache, torch.uint8, "k_cache"), _ptr(kv_cache, torch.bfloat16, "kv_cache", True), _stream()))


def cp_candidates(scores, idx_local, lo, cand_score=None, cand_pos=None):
    """(score, global position) of each locally kept index; scores fp32 [B, ld], idx_local int32 [B, K]."""
    B, K = idx_local.shape
    if cand_score is None:
        cand_score = torch.empty((B, K), dtype=torch.float32, device=scores.device)
    if cand_pos is None:
        cand_pos = torch.empty((B, K), dtype=torch.int32, device=scores.device)
    _check("dsa_cp_candidates", lib.dsa_cp_candidates(
        _ptr(scores, torch.float32, "scores"), int(scores.shape[1]), _ptr(idx_local, torch.int32, "idx_local"), B, K,
        _ptr(lo, torch.int32, "lo"), _ptr(cand_score, torch.float32, "cand_score"),
        _ptr(cand_pos, torch.int32, "cand_pos"), _stream()))
    return cand_score, cand_pos


def cp_select(cand_score, cand_pos, lo, hi, idx_global=None, idx_local=None, ws=None):
    """cand_score fp32 / cand_pos int32 [G, B, K] (every rank's candidates) -> (idx_global, idx_local) [B, K]."""
    G, B, K = cand_score.shape
    dev = cand_score.device
    if idx_global is None:
        idx_global = torch.empty((B, K), dtype=torch.int32, device=dev)
    if idx_local is None:
        idx_local = torch.empty((B, K), dtype=torch.int32, device=dev)
    need = int(lib.dsa_cp_select_workspace_bytes(G, B, K))
    if ws is None:
        ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check("dsa_cp_select", lib.dsa_cp_select(
        _ptr(cand_score, torch.float32, "cand_score"), _ptr(cand_pos, torch.int32, "cand_pos"), G, B, K,
        _ptr(lo, torch.int32, "lo"), _ptr(hi, torch.int32, "hi"), _ptr(idx_global, torch.int32, "idx_global"),
        _ptr(idx_local, torch.int32, "idx_local"), _ptr(ws, torch.uint8, "ws"), ws.numel(), _stream()))
    return idx_global, idx_local


def cp_lse_merge(o, lse, out=None):
    """o bf16 [G, B, H, Dv], lse fp32 [G, B, H] -> out bf16 [B, H, Dv]."""
    G, B, H, Dv = o.shape
    if out is None:
        out = torch.empty((B, H, Dv), dtype=torch.bfloat16, device=o.device)
    _check("dsa_cp_lse_merge", lib.dsa_cp_lse_merge(
        _ptr(o, torch.bfloat16, "o"), _ptr(lse, torch.float32, "lse"), G, B, H, Dv, _ptr(out, torch.bfloat16, "out"),
        _stream()))
    return out


def indexer_scores_mx(q_idx, q_scales, w, k_cache, k_scales, pg: Paged, q_seq, q_pos, max_len: int, scores):
    """MXFP8 indexer: q_idx uint8 [T,HI,DI] and q_scales uint8 [T,HI,DI/32]; k_cache uint8 [pages,64,DI] and
    k_scales uint8 [pages,64,DI/32]; w fp32 [T,HI]; scores fp32 [T, ld]."""
    T, HI, DI = q_idx.shape
    _check("dsa_indexer_scores_mx", lib.dsa_indexer_scores_mx(
        _ptr(q_idx, torch.uint8, "q_idx"), _ptr(q_scales, torch.uint8, "q_scales"), _ptr(w, torch.float32, "w"),
        _ptr(k_cache, torch.uint8, "k_cache"), _ptr(k_scales, torch.uint8, "k_scales"), ctypes.byref(pg),
        _ptr(q_seq, torch.int32, "q_seq", True), _ptr(q_pos, torch.int32, "q_pos", True), T, HI, DI, int(max_len),
        _ptr(scores, torch.float32, "scores"), int(scores.shape[1]), _stream()))
    return scores


def append_kv_mx(k_new, latent_new, tok_seq, tok_pos, pg: Paged, k_cache, k_scales, kv_cache):
    """MXFP8 append: k_new bf16 [n, DI]; latent_new bf16 [n, Dqk] or None; k_cache uint8 [pages, 64, DI],
    k_scales uint8 [pages, 64, DI/32] and kv_cache bf16 [pages, 64, Dqk], written in place."""
    n, DI = k_new.shape
    Dqk = int(kv_cache.shape[-1]) if kv_cache is not None else 0
    _check("dsa_append_kv_mx", lib.dsa_append_kv_mx(
        _ptr(k_new, torch.bfloat16, "k_new"), _ptr(latent_new, torch.bfloat16, "latent_new", True),
        _ptr(tok_seq, torch.int32, "tok_seq"), _ptr(tok_pos, torch.int32, "tok_pos"), ctypes.byref(pg), n, DI, Dqk,
        _ptr(k_cache, torch.uint8, "k_cache"), _ptr(k_scales, torch.uint8, "k_scales"),
        _ptr(kv_cache, torch.bfloat16, "kv_cache", True), _stream()))
