"""Seeded synthetic inputs for the Gated DSA layer.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic.  Both the CUDA path's tests and the CPU oracle take
their inputs from here, so the two sides see identical bytes.

Workloads follow the shapes the pages describe: a 1,048,576-token context,
32x128 and 16x128 no-RoPE FP8 indexers, top-K = 2048, a 5:1 layout of
sliding-window (128) and DSA layers; the latent KV row is 576 wide
(512 + 64) and paged 64 tokens per page.  No dataset is involved: every
value is drawn here from ``numpy.random.default_rng(seed)``.

Indexer operands are "dyadic": small integers times 2^-4 (exact in e4m3),
and weights on a 2^-6 grid.  Under that scheme every partial sum of the
indexer score is exact in fp32, whatever the summation order, so the GPU's
scores and selected indices can be compared bit for bit with the oracle.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

PAGE_SIZE = 64


# ---- format conversions (storage only: library casts, no method math) ----

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f32_to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


# ---- building blocks -------------------------------------------------------

def dyadic_e4m3(rng: np.random.Generator, shape, lo: int = -4, hi: int = 4) -> np.ndarray:
    """e4m3 codes of n * 2^-4 with n uniform in [lo, hi]."""
    n = rng.integers(lo, hi + 1, size=shape, dtype=np.int64)
    return f32_to_e4m3_bits(n.astype(np.float32) / 16.0)


def mx_dyadic(rng: np.random.Generator, shape, lo_code: int = 117, hi_code: int = 132):
    """MXFP8 operands whose decoded values are the dyadic indexer values
    n * 2^-4, n in [-4, 4]: each 32-element block along the last axis draws a
    scale code c in [lo_code, hi_code] and stores the elements as E4M3 codes
    of n * 2^-4 / 2^(c - 127) (exact in E4M3 for codes 117..132).  Returns
    (element codes uint8 [..., n], scale codes uint8 [..., n/32])."""
    shape = tuple(shape)
    n = rng.integers(-4, 5, size=shape).astype(np.float32)
    codes = rng.integers(lo_code, hi_code + 1, size=shape[:-1] + (shape[-1] // 32,)).astype(np.uint8)
    s = np.repeat(codes.astype(np.int32) - 127, 32, axis=-1)
    return f32_to_e4m3_bits(np.ldexp(n * np.float32(2.0 ** -4), -s).astype(np.float32)), codes


def dyadic_weights(rng: np.random.Generator, shape, signed: bool = False) -> np.ndarray:
    """fp32 weights n * 2^-6, n uniform in [0, 64] (or [-64, 64] when signed)."""
    lo = -64 if signed else 0
    n = rng.integers(lo, 65, size=shape, dtype=np.int64)
    return (n.astype(np.float32) / 64.0)


def normal_bf16(rng: np.random.Generator, shape, chunk: int = 1 << 26) -> np.ndarray:
    """bf16 bit patterns of N(0,1) draws (generated in chunks to bound memory)."""
    total = int(np.prod(shape))
    out = np.empty(total, dtype=np.uint16)
    for s in range(0, total, chunk):
        e = min(total, s + chunk)
        out[s:e] = f32_to_bf16_bits(rng.standard_normal(e - s, dtype=np.float32))
    return out.reshape(shape)


def paged_layout(rng: np.random.Generator, seq_lens, page_size: int = PAGE_SIZE,
                 spare_pages: int = 0):
    """A block table that scatters every sequence over randomly permuted physical
    pages. Returns (block_table [B, max_blocks] int32, num_pages). Unused table
    entries are -1."""
    seq_lens = np.asarray(seq_lens, dtype=np.int64)
    blocks = [int(math.ceil(int(L) / page_size)) for L in seq_lens]
    max_blocks = max(1, max(blocks) if blocks else 1)
    num_pages = int(sum(blocks)) + int(spare_pages)
    perm = rng.permutation(num_pages).astype(np.int32)
    bt = np.full((len(seq_lens), max_blocks), -1, dtype=np.int32)
    off = 0
    for b, nb in enumerate(blocks):
        bt[b, :nb] = perm[off:off + nb]
        off += nb
    return bt, num_pages


# ---- a whole layer's inputs ------------------------------------------------

@dataclasses.dataclass
class LayerCase:
    name: str
    q_idx: np.ndarray       # uint8 e4m3 [T, HI, DI]
    w: np.ndarray           # fp32 [T, HI]
    k_cache: np.ndarray     # uint8 e4m3 [num_pages, page, DI]
    q: np.ndarray           # uint16 bf16 [T, H, Dqk]
    kv_cache: np.ndarray    # uint16 bf16 [num_pages, page, Dqk]
    gate: np.ndarray        # uint16 bf16 [T, H]
    seq_lens: np.ndarray    # int32 [B]
    block_table: np.ndarray  # int32 [B, max_blocks]
    q_seq: np.ndarray       # int32 [T]
    q_pos: np.ndarray       # int32 [T]
    K: int
    Dv: int
    sm_scale: float
    page_size: int
    num_pages: int

    @property
    def T(self):
        return int(self.q_idx.shape[0])

    @property
    def HI(self):
        return int(self.q_idx.shape[1])

    @property
    def DI(self):
        return int(self.q_idx.shape[2])

    @property
    def H(self):
        return int(self.q.shape[1])

    @property
    def Dqk(self):
        return int(self.q.shape[2])

    @property
    def max_len(self):
        return int(self.seq_lens.max())


def layer_case(name: str, seed: int, seq_lens, q_seq, q_pos, HI: int, DI: int, K: int, H: int,
               Dqk: int, Dv: int, w_signed: bool = False, page_size: int = PAGE_SIZE,
               spare_pages: int = 0, sm_scale: Optional[float] = None,
               latent: bool = True) -> LayerCase:
    """Inputs for one layer call. One sub-stream of the seeded generator per
    tensor, so a tensor's values do not depend on the others' shapes."""
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    q_seq = np.asarray(q_seq, dtype=np.int32)
    q_pos = np.asarray(q_pos, dtype=np.int32)
    T = int(q_seq.shape[0])
    ss = np.random.SeedSequence(seed)
    r_pages, r_qi, r_w, r_ki, r_q, r_kv, r_g = [np.random.default_rng(s) for s in ss.spawn(7)]
    bt, num_pages = paged_layout(r_pages, seq_lens, page_size, spare_pages)
    q_idx = dyadic_e4m3(r_qi, (T, HI, DI))
    w = dyadic_weights(r_w, (T, HI), signed=w_signed)
    k_cache = dyadic_e4m3(r_ki, (num_pages, page_size, DI))
    q = normal_bf16(r_q, (T, H, Dqk))
    kv_cache = normal_bf16(r_kv, (num_pages, page_size, Dqk)) if latent else \
        np.zeros((num_pages, page_size, Dqk), dtype=np.uint16)
    gate = normal_bf16(r_g, (T, H))
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(Dqk)
    return LayerCase(name, q_idx, w, k_cache, q, kv_cache, gate, seq_lens, bt, q_seq, q_pos,
                     K, Dv, float(sm_scale), page_size, num_pages)


# ---- the workloads -----------------------------------------------------------

def tiny_prefill(seed: int = 0, T: int = 1024) -> LayerCase:
    """One sequence, T=1024 causal queries; indexer 4 heads x 64; K=128;
    8 query heads over a 64-wide latent (key = value = the row)."""
    return layer_case("tiny_prefill_T1024", seed, [T], np.zeros(T, np.int32),
                      np.arange(T, dtype=np.int32), HI=4, DI=64, K=128, H=8, Dqk=64, Dv=64)


def decode_case(seed: int, seq_lens, HI: int = 32, DI: int = 128, K: int = 2048, H: int = 128,
                Dqk: int = 576, Dv: int = 512, name: str = "decode", **kw) -> LayerCase:
    """One query per sequence at position seq_len - 1."""
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = len(seq_lens)
    return layer_case(name, seed, seq_lens, np.arange(B, dtype=np.int32), seq_lens - 1,
                      HI=HI, DI=DI, K=K, H=H, Dqk=Dqk, Dv=Dv, **kw)


def decode_128k(seed: int = 0, B: int = 8, L: int = 131072) -> LayerCase:
    """Batch 8 x 131072-token contexts, 32x128 indexer, K=2048, 128 heads
    over the 576-wide latent (512 value dims)."""
    return decode_case(seed, [L] * B, HI=32, name=f"decode_B{B}_L{L}")


def decode_1m(seed: int = 0) -> LayerCase:
    return decode_case(seed, [1 << 20], HI=32, name="decode_B1_L1048576")


def mtp_decode(seed: int = 0, B: int = 8, L: int = 131072, n: int = 4, HI: int = 32) -> LayerCase:
    """Several query tokens per sequence at its last n positions (draft tokens
    of speculative decoding), as explicit (sequence, position) queries."""
    seq_lens = np.full(B, L, np.int32) if np.isscalar(L) else np.asarray(L, np.int32)
    q_seq = np.repeat(np.arange(B, dtype=np.int32), n)
    q_pos = (seq_lens[q_seq] - n + np.tile(np.arange(n, dtype=np.int32), B)).astype(np.int32)
    return layer_case(f"mtp_B{B}x{n}_L{int(seq_lens.max())}", seed, seq_lens, q_seq, q_pos, HI=HI, DI=128, K=2048,
                      H=128, Dqk=576, Dv=512)


def with_queries(case: LayerCase, seed: int, q_seq, q_pos, name: str) -> LayerCase:
    """The same caches with other (sequence, position) queries: new query-side
    tensors (indexer queries and weights, attention queries, gate logits) of
    the case's shapes, one seeded sub-stream each."""
    q_seq = np.asarray(q_seq, dtype=np.int32)
    q_pos = np.asarray(q_pos, dtype=np.int32)
    T = int(q_seq.shape[0])
    r_qi, r_w, r_q, r_g = [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(4)]
    return dataclasses.replace(case, name=name, q_idx=dyadic_e4m3(r_qi, (T, case.HI, case.DI)),
                               w=dyadic_weights(r_w, (T, case.HI)), q=normal_bf16(r_q, (T, case.H, case.Dqk)),
                               gate=normal_bf16(r_g, (T, case.H)), q_seq=q_seq, q_pos=q_pos)


def prefill_case(seed: int, T: int, HI: int = 16, DI: int = 128, K: int = 2048, H: int = 128,
                 Dqk: int = 576, Dv: int = 512, **kw) -> LayerCase:
    """One sequence of T tokens, every token a causal query."""
    return layer_case(f"prefill_T{T}", seed, [T], np.zeros(T, np.int32),
                      np.arange(T, dtype=np.int32), HI=HI, DI=DI, K=K, H=H, Dqk=Dqk, Dv=Dv, **kw)


def hybrid_seq_lens(seed: int = 0, B: int = 64, lo: int = 4096, hi: int = 65536) -> np.ndarray:
    """Ragged continuous-batch lengths, uniform in [lo, hi]."""
    return np.random.default_rng(seed).integers(lo, hi + 1, size=B).astype(np.int32)


def hybrid_dsa(seed: int = 0) -> LayerCase:
    return decode_case(seed, hybrid_seq_lens(seed), HI=16, name="hybrid_dsa_B64")


@dataclasses.dataclass
class SwaCase:
    q: np.ndarray        # uint16 bf16 [B, H, D]
    k_ring: np.ndarray   # uint16 bf16 [B, W, H, D]
    v_ring: np.ndarray   # uint16 bf16 [B, W, H, D]
    seq_lens: np.ndarray  # int32 [B]
    window: int
    sm_scale: float


def swa_case(seed: int, seq_lens, H: int = 64, D: int = 128, window: int = 128) -> SwaCase:
    seq_lens = np.asarray(seq_lens, dtype=np.int32)
    B = len(seq_lens)
    r_q, r_k, r_v = [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(3)]
    return SwaCase(normal_bf16(r_q, (B, H, D)), normal_bf16(r_k, (B, window, H, D)),
                   normal_bf16(r_v, (B, window, H, D)), seq_lens, window, 1.0 / math.sqrt(D))


def score_rows(seed: int, R: int, n: int, kind: str = "normal") -> np.ndarray:
    """Synthetic score rows for exercising top-K alone.
    kind: 'normal' (N(0,1) fp32), 'ties' (few distinct values), 'zeros'
    (+0/-0 mix), 'const' (all equal), 'dyadic' (multiples of 2^-14),
    'outlier' (N(0,1) and one score of 1e30 per row), 'narrow'
    (1 + N(0,1) 2^-20), 'near' / 'cluster' (N(0,1) with an eighth of the
    row drawn tightly around 1.53: hundreds / thousands of keys per fine bin)."""
    rng = np.random.default_rng(seed)
    if kind == "normal":
        return rng.standard_normal((R, n), dtype=np.float32)
    if kind == "ties":
        return rng.integers(-3, 4, size=(R, n)).astype(np.float32) * 0.25
    if kind == "zeros":
        v = rng.integers(-1, 2, size=(R, n)).astype(np.float32)
        z = rng.random((R, n)) < 0.5
        v[(v == 0) & z] = -0.0
        return v
    if kind == "const":
        return np.full((R, n), 1.5, dtype=np.float32)
    if kind == "dyadic":
        return rng.integers(-(1 << 16), 1 << 16, size=(R, n)).astype(np.float32) * (2.0 ** -14)
    if kind == "narrow":  # 1 + N(0,1) 2^-20: thousands of keys share one fine bin
        return (1.0 + rng.standard_normal((R, n)) * 2.0 ** -20).astype(np.float32)
    if kind in ("near", "cluster"):  # N(0,1), an eighth of it moved to 1.53 + N(0,1) 2^-12 (2^-16)
        v = rng.standard_normal((R, n), dtype=np.float32)
        m = rng.random((R, n)) < 0.125
        sd = 2.0 ** -12 if kind == "near" else 2.0 ** -16
        v[m] = (1.53 + rng.standard_normal(int(m.sum())) * sd).astype(np.float32)
        return v
    if kind == "outlier":  # N(0,1) with one huge score per row
        v = rng.standard_normal((R, n), dtype=np.float32)
        v[np.arange(R), rng.integers(0, n, size=R)] = 1e30
        return v
    raise ValueError(kind)
