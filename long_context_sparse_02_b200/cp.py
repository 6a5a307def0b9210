"""Context-parallel decode: one long sequence's history over G GPUs.

Host-side orchestration of the C-ABI calls (include/dsa.h, "context-parallel
decode"); every step that computes runs in libdsa.so.  Rank r holds a
contiguous run of whole pages of every sequence.  A decode step is

  local indexer + top-K  ->  candidates  ->  all-gather  ->  select
  ->  attention over the kept rows this rank holds  ->  all-gather  ->  merge

with the selection identical to one GPU's ("Open-Source LLM Architecture
Evolution", Architecture Breakdown §2, "Top-K selection": a position among
the K best of the whole history is among the K best of its own range) and
the outputs merged by their log-sum-exp weights.  The two exchanges go
through a caller-given `all_gather(tensor) -> [G, *tensor.shape]`
(torch.distributed with NCCL across GPUs; a list stack when G ranks are
emulated one after another on one GPU).
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib


def rank_ranges(seq_len: int, page_size: int, G: int):
    """[lo, hi) of each rank: the sequence's pages dealt out in G runs of
    ceil(pages / G) whole pages (the last runs may be short or empty)."""
    pages = -(-int(seq_len) // page_size)
    per = -(-pages // G) if pages else 0
    return [(min(r * per * page_size, seq_len), min((r + 1) * per * page_size, seq_len)) for r in range(G)]


def local_view(seq_lens, block_table, page_size: int, G: int, r: int):
    """Rank r's share of every sequence: lo, hi [B] and its paged view (local
    lengths hi - lo and the block table from page lo / page_size on)."""
    seq_lens = np.asarray(seq_lens, np.int64)
    block_table = np.asarray(block_table, np.int32)
    B = len(seq_lens)
    lo = np.zeros(B, np.int32)
    hi = np.zeros(B, np.int32)
    bt = np.full(block_table.shape, -1, np.int32)
    for b in range(B):
        lo[b], hi[b] = rank_ranges(int(seq_lens[b]), page_size, G)[r]
        nb = -(-int(hi[b] - lo[b]) // page_size)
        bt[b, :nb] = block_table[b, lo[b] // page_size: lo[b] // page_size + nb]
    return lo, hi, (hi - lo).astype(np.int32), bt


class CpRank:
    """Rank r of G for a decode batch whose caches this GPU holds in full or in
    part (only the pages of its runs are read).  Device tensors: the caches
    (paged, global page ids), and per step the queries of every sequence."""

    def __init__(self, r: int, G: int, seq_lens, block_table, num_pages: int, k_cache, kv_cache, K: int, Dv: int,
                 sm_scale: float, page_size: int = 64, device="cuda"):
        self.r, self.G, self.K, self.Dv, self.sm_scale = r, G, int(K), int(Dv), float(sm_scale)
        lo, hi, n, bt = local_view(seq_lens, block_table, page_size, G, r)
        self.B = len(n)
        self.lo, self.hi = torch.from_numpy(lo).to(device), torch.from_numpy(hi).to(device)
        self.n = torch.from_numpy(n).to(device)
        self.bt = torch.from_numpy(bt).to(device)
        self.pg = _lib.paged(self.n, self.bt, num_pages, page_size)
        self.k_cache, self.kv_cache = k_cache, kv_cache
        self.max_len = max(1, int(n.max()))
        self.scores = torch.empty((self.B, (self.max_len + 3) // 4 * 4), dtype=torch.float32, device=device)

    def candidates(self, q_idx, w):
        """Local scores and top-K -> (score, global position) [B, K]."""
        _lib.indexer_scores(q_idx, w, self.k_cache, self.pg, None, None, self.max_len, self.scores)
        idx = _lib.topk(self.scores, self.n, self.K, self.max_len)
        return _lib.cp_candidates(self.scores, idx, self.lo)

    def attend(self, all_score, all_pos, q, gate):
        """The global selection from every rank's candidates [G, B, K]; this
        rank's gated partial output and log-sum-exp over the rows it holds."""
        idx_g, idx_l = _lib.cp_select(all_score, all_pos, self.lo, self.hi)
        H = q.shape[1]
        lse = torch.empty((self.B, H), dtype=torch.float32, device=q.device)
        o = _lib.sparse_attn(q, self.kv_cache, self.pg, None, idx_l, gate, self.sm_scale, self.Dv, lse=lse)
        return o, lse, idx_g


def decode_step(rank, q_idx, w, q, gate, all_gather, merge=None):
    """One context-parallel decode step on one rank; returns (out [B, H, Dv]
    bf16, idx [B, K] global positions).  Every rank takes the same two
    exchanges in the same order."""
    cs, cpos = rank.candidates(q_idx, w)
    all_s, all_p = all_gather(cs), all_gather(cpos)
    o, lse, idx = rank.attend(all_s, all_p, q, gate)
    all_o, all_l = all_gather(o), all_gather(lse)
    return (merge or _lib.cp_lse_merge)(all_o, all_l), idx


def emulate(ranks, q_idx, w, q, gate):
    """The G ranks one after another on this GPU (the exchanges become stacks
    of the ranks' tensors): the same calls, in the same order, as G GPUs make."""
    cands = [rk.candidates(q_idx, w) for rk in ranks]
    all_s = torch.stack([c[0] for c in cands])
    all_p = torch.stack([c[1] for c in cands])
    parts = [rk.attend(all_s, all_p, q, gate) for rk in ranks]
    out = _lib.cp_lse_merge(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]))
    return out, parts[0][2]


def torch_all_gather(group=None):
    """all_gather over torch.distributed (NCCL between GPUs): [G, *shape]."""
    import torch.distributed as dist

    def ag(t):
        G = dist.get_world_size(group)
        out = torch.empty((G,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return out
    return ag
