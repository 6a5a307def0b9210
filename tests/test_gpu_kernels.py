"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Sizes span several tiles plus ragged tails.  Indexer scores on dyadic inputs
and every top-K index must match bit for bit; attention outputs must agree
within rtol 2e-2 / atol 1e-2 (bf16 output), plus a relative Frobenius error
of at most 1e-2.
"""
import math

import numpy as np
import pytest
import torch

from long_context_sparse_02_b200 import synth

pytestmark = pytest.mark.gpu

RTOL, ATOL, FRO = 2e-2, 1e-2, 1e-2


@pytest.fixture(scope="module")
def L():
    from long_context_sparse_02_b200 import build
    build.build()
    from long_context_sparse_02_b200 import _lib
    _lib.device_error(reset=True)
    return _lib


def dev(a):
    from long_context_sparse_02_b200.runtime import to_dev
    return to_dev(a)


def bf16_to_np(t):
    return t.float().cpu().numpy().astype(np.float64)


def assert_attn_close(got, ref):
    np.testing.assert_allclose(got, ref, rtol=RTOL, atol=ATOL)
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert fro <= FRO, fro


def no_device_error(L):
    torch.cuda.synchronize()
    assert L.device_error(reset=True) == 0


# ------------------------------------------------------------------ indexer

INDEXER_CASES = [
    # name, HI, DI, seq_lens, queries (None = decode), signed w
    ("prefill_h4_d64", 4, 64, [1000], "prefill", False),
    ("prefill_h16_d128", 16, 128, [700], "prefill", True),
    ("prefill_h32_d128_two_seqs", 32, 128, [333, 517], "prefill2", False),
    ("prefill_h64_d64", 64, 64, [260], "prefill", True),
    ("prefill_h8_d128", 8, 128, [390], "prefill", False),
    ("decode_h32_d128", 32, 128, [1, 63, 64, 65, 128, 129, 4999], "decode", True),
    ("decode_h16_d128", 16, 128, [3000, 257], "decode", False),
    ("decode_h64_d64", 64, 64, [70, 2050], "decode", True),
    ("decode_h4_d64", 4, 64, [1500], "decode", False),
    # few explicit queries, several per sequence: grouped key streams (runs of 5 -> 4 + 1, singletons, a return)
    ("drafts_h32_d128", 32, 128, [3000, 257, 5000], "drafts", True),
    ("drafts_h16_d128", 16, 128, [4999, 130, 2050], "drafts", False),
]


def _indexer_case(HI, DI, seq_lens, kind, signed, seed=7):
    if kind == "decode":
        return synth.decode_case(seed, seq_lens, HI=HI, DI=DI, K=64, H=1, Dqk=64, Dv=64, w_signed=signed)
    if kind == "prefill":
        T = seq_lens[0]
        return synth.layer_case("p", seed, seq_lens, np.zeros(T, np.int32), np.arange(T, dtype=np.int32), HI=HI,
                                DI=DI, K=64, H=1, Dqk=64, Dv=64, w_signed=signed)
    if kind == "drafts":
        q_seq = np.array([0, 0, 0, 0, 0, 1, 2, 2, 2, 0, 1], np.int32)
        last = np.asarray(seq_lens, np.int32)[q_seq] - 1
        back = np.array([4, 3, 2, 1, 0, 0, 2, 1, 0, 0, 77], np.int32)  # distinct positions, the last ones first
        return synth.layer_case("d", seed, seq_lens, q_seq, np.maximum(last - back, 0), HI=HI, DI=DI, K=64, H=1,
                                Dqk=64, Dv=64, w_signed=signed)
    # two sequences, every token of each a query, concatenated
    q_seq = np.concatenate([np.full(n, b, np.int32) for b, n in enumerate(seq_lens)])
    q_pos = np.concatenate([np.arange(n, dtype=np.int32) for n in seq_lens])
    return synth.layer_case("p2", seed, seq_lens, q_seq, q_pos, HI=HI, DI=DI, K=64, H=1, Dqk=64, Dv=64,
                            w_signed=signed)


@pytest.mark.parametrize("name,HI,DI,seq_lens,kind,signed", INDEXER_CASES, ids=[c[0] for c in INDEXER_CASES])
def test_indexer_scores_bit_exact(L, orc, name, HI, DI, seq_lens, kind, signed):
    c = _indexer_case(HI, DI, seq_lens, kind, signed)
    decode = kind == "decode"
    q_pos = (c.seq_lens - 1) if decode else c.q_pos
    q_seq = np.arange(len(c.seq_lens), dtype=np.int32) if decode else c.q_seq
    max_len = int(q_pos.max()) + 1
    ld = (max_len + 3) // 4 * 4
    pg = L.paged(dev(c.seq_lens), dev(c.block_table), c.num_pages)
    scores = torch.full((c.T, ld), float("nan"), device="cuda")
    L.indexer_scores(dev(c.q_idx), dev(c.w), dev(c.k_cache), pg, None if decode else dev(c.q_seq),
                     None if decode else dev(c.q_pos), max_len, scores)
    got = scores.cpu().numpy()
    ref = orc.indexer_scores(c.q_idx, c.w, c.k_cache, orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages),
                             q_seq, q_pos, ld=ld)
    for t in range(c.T):
        n = q_pos[t] + 1
        assert np.array_equal(got[t, :n], ref[t, :n]), (t, np.flatnonzero(got[t, :n] != ref[t, :n])[:8])
        assert np.all(np.isnan(got[t, n:])), t   # nothing written past the query's position
    no_device_error(L)


def test_indexer_non_dyadic_within_fp32_rounding(L, orc):
    """Arbitrary e4m3 operands: the fp32 accumulation order differs from the
    oracle's fp64 sum, so agreement is to fp32 rounding only."""
    rng = np.random.default_rng(3)
    c = synth.decode_case(9, [3000, 777], HI=32, DI=128, K=64, H=1, Dqk=64, Dv=64)
    c.q_idx = synth.f32_to_e4m3_bits(rng.standard_normal(c.q_idx.shape).astype(np.float32))
    c.k_cache = synth.f32_to_e4m3_bits(rng.standard_normal(c.k_cache.shape).astype(np.float32) * 2)
    c.w = rng.random(c.w.shape).astype(np.float32)
    pg = L.paged(dev(c.seq_lens), dev(c.block_table), c.num_pages)
    scores = torch.zeros((2, 3000), device="cuda")
    L.indexer_scores(dev(c.q_idx), dev(c.w), dev(c.k_cache), pg, None, None, 3000, scores)
    ref = orc.indexer_scores(c.q_idx, c.w, c.k_cache, orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages),
                             [0, 1], c.seq_lens - 1, ld=3000)
    got = scores.cpu().numpy()
    for t, n in enumerate(c.seq_lens):
        np.testing.assert_allclose(got[t, :n], ref[t, :n], rtol=2e-6, atol=1e-5)


# ------------------------------------------------------------------ top-K

TOPK_CASES = [
    # rows, n (ld), K, kinds, path
    (37, 3001, 128, "normal"), (16, 4100, 2048, "ties"), (8, 2500, 64, "zeros"), (5, 1000, 100, "const"),
    (9, 5000, 1, "dyadic"), (3, 49152, 2048, "ties"),
    (3, 70000, 2048, "normal"), (2, 131072, 2048, "dyadic"), (2, 90001, 2048, "ties"), (2, 60000, 17, "const"),
    (1, 300000, 2048, "zeros"),
    (8, 131072, 2048, "normal"), (4, 4000, 2048, "outlier"), (2, 131072, 2048, "outlier"),
    (80, 70000, 2048, "normal"), (76, 120000, 2048, "dyadic"),
    # many rows of at most 32768 (prefill): one CTA per row, list in shared memory
    (300, 32768, 2048, "normal"), (310, 20000, 2048, "ties"), (296, 9000, 512, "dyadic"),
    (300, 32768, 2048, "narrow"), (300, 32768, 2048, "near"), (300, 32768, 2048, "cluster"), (300, 32768, 2048, "outlier"),
    (300, 3000, 2048, "zeros"), (300, 9001, 64, "normal"),
    # the per-row kernel's edges: every score equal and +-0 ties (the list overflows: radix fallback), rows on both
    # sides of the 4096-entry list, K as large as the list, K = 1
    (300, 20000, 2048, "const"), (300, 20000, 2048, "zeros"), (300, 4097, 2048, "normal"),
    (300, 32768, 4096, "normal"), (300, 32768, 1, "dyadic"),
]


@pytest.mark.parametrize("R,n,K,kind", TOPK_CASES, ids=[f"{c[0]}x{c[1]}_K{c[2]}_{c[3]}" for c in TOPK_CASES])
def test_topk_bit_exact(L, orc, R, n, K, kind):
    sc = synth.score_rows(11, R, n, kind)
    rng = np.random.default_rng(12)
    rl = rng.integers(0, n + 1, size=R).astype(np.int32)
    rl[0] = n
    if R > 2:
        rl[1], rl[2] = min(K, n), min(K + 1, n)
    idx = L.topk(dev(sc), dev(rl), K, n)
    ref = orc.topk(sc, rl, K)
    got = idx.cpu().numpy()
    for r in range(R):
        assert np.array_equal(got[r], ref[r]), (r, rl[r])
    no_device_error(L)


def coarse_hist(sc, rl):
    """Counts of each row's order-preserving score keys by their top 11 bits
    (the caller-side input of dsa_topk_hist; -0.0 counts as +0.0)."""
    u = sc.astype(np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0
    key = np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)
    h = np.zeros((sc.shape[0], 2048), np.int64)
    for r in range(sc.shape[0]):
        h[r] = np.bincount(key[r, :rl[r]] >> 21, minlength=2048)
    return h.astype(np.uint32).view(np.int32)


@pytest.mark.parametrize("R,n,K,kind", TOPK_CASES, ids=[f"{c[0]}x{c[1]}_K{c[2]}_{c[3]}" for c in TOPK_CASES])
def test_topk_hist_bit_exact(L, orc, R, n, K, kind):
    """The histogram-fed top-K (one launch, last-CTA select) on the same rows,
    twice on one workspace; a garbage histogram takes the whole-row select."""
    sc = synth.score_rows(11, R, n, kind)
    ld = (n + 3) // 4 * 4
    scp = np.zeros((R, ld), np.float32)
    scp[:, :n] = sc
    rng = np.random.default_rng(12)
    rl = rng.integers(0, n + 1, size=R).astype(np.int32)
    rl[0] = n
    if R > 2:
        rl[1], rl[2] = min(K, n), min(K + 1, n)
    ref = orc.topk(sc, rl, K)
    hist = dev(coarse_hist(sc, rl))
    ws = torch.full((L.lib.dsa_topk_hist_workspace_bytes(R, n),), 0x5A, dtype=torch.uint8, device="cuda")
    for rep in range(3):
        if rep == 2:  # counts that do not describe the rows
            hist = torch.randint(0, 64, (R, 2048), dtype=torch.int32, device="cuda")
        elif rep == 1:
            assert int(hist.abs().sum()) == 0  # the first call cleared the counts
            hist = dev(coarse_hist(sc, rl))
        idx = L.topk_hist(dev(scp), dev(rl), hist, K, n, ws=ws)
        got = idx.cpu().numpy()
        for r in range(R):
            assert np.array_equal(got[r], ref[r]), (rep, r, rl[r])
    no_device_error(L)


# ------------------------------------------------------------------ attention

@pytest.mark.parametrize("Dqk,Dv,H,K,seq_lens,T,pad", [
    (64, 64, 8, 128, [900], 5, False),
    (64, 64, 3, 64, [50, 700], 7, True),
    (576, 512, 128, 2048, [5000], 3, False),
    (576, 512, 128, 2048, [300, 9000], 4, True),
    (576, 512, 40, 256, [2000], 16, True),
    (576, 512, 128, 512, [600, 3000], 64, True),
    (576, 512, 128, 960, [5000], 2, False),
    (576, 512, 128, 2560, [3000, 9000], 3, True),
], ids=["tiny", "tiny_pad", "full_T3", "full_decode_split", "heads40", "prefill_T64", "ragged_K960",
        "K2560_two_kernel"])
def test_sparse_attn_within_tolerance(L, orc, Dqk, Dv, H, K, seq_lens, T, pad):
    rng = np.random.default_rng(5)
    B = len(seq_lens)
    q_seq = rng.integers(0, B, size=T).astype(np.int32)
    c = synth.layer_case("a", 21, seq_lens, q_seq, np.zeros(T, np.int32), HI=4, DI=64, K=K, H=H, Dqk=Dqk, Dv=Dv)
    idx = np.full((T, K), -1, np.int32)
    for t in range(T):
        n = int(c.seq_lens[q_seq[t]])
        take = min(K, n) if not pad else int(rng.integers(0, min(K, n) + 1))
        sel = np.sort(rng.choice(n, size=take, replace=False)).astype(np.int32)
        idx[t, :take] = sel
        if pad and take and t % 2:   # scatter padding inside the list too
            idx[t] = rng.permutation(idx[t])
    pg = L.paged(dev(c.seq_lens), dev(c.block_table), c.num_pages)
    lse = torch.empty((T, H), dtype=torch.float32, device="cuda")
    out = L.sparse_attn(dev(c.q), dev(c.kv_cache), pg, dev(q_seq), dev(idx), dev(c.gate), c.sm_scale, Dv, lse=lse)
    ref, ref_lse = orc.sparse_attn(c.q, c.kv_cache, orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages), q_seq,
                                   idx, c.gate, c.sm_scale, Dv, return_lse=True)
    assert_attn_close(bf16_to_np(out), ref)
    got_lse = lse.cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got_lse), fin)
    np.testing.assert_allclose(got_lse[fin], ref_lse[fin], rtol=1e-3, atol=2e-3)
    no_device_error(L)


def test_sparse_attn_decode_splits_and_empty_rows(L, orc):
    """Decode convention (q_seq NULL) with split-K partials and a query whose
    selection is empty (all padding)."""
    c = synth.decode_case(4, [4096, 17, 2048], K=2048)
    idx = np.full((3, 2048), -1, np.int32)
    idx[0] = np.arange(0, 4096, 2)
    idx[2, :1000] = np.arange(1000) * 2
    pg = L.paged(dev(c.seq_lens), dev(c.block_table), c.num_pages)
    out = L.sparse_attn(dev(c.q), dev(c.kv_cache), pg, None, dev(idx), dev(c.gate), c.sm_scale, 512)
    ref = orc.sparse_attn(c.q, c.kv_cache, orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages), [0, 1, 2], idx,
                          c.gate, c.sm_scale, 512)
    got = bf16_to_np(out)
    assert np.all(got[1] == 0)
    assert_attn_close(got, ref)
    no_device_error(L)


def test_device_errors_are_reported_not_faulted(L, orc):
    """A selected position past its sequence and a bad block-table entry are
    skipped (treated as padding) and flagged in the device error word."""
    c = synth.decode_case(6, [300], K=128, H=8, Dqk=64, Dv=64)
    idx = np.full((1, 128), -1, np.int32)
    idx[0, :3] = [5, 299, 300]          # 300 is past the sequence
    pg = L.paged(dev(c.seq_lens), dev(c.block_table), c.num_pages)
    L.device_error(reset=True)
    out = L.sparse_attn(dev(c.q), dev(c.kv_cache), pg, None, dev(idx), dev(c.gate), c.sm_scale, 64)
    torch.cuda.synchronize()
    assert L.device_error(reset=True) & L.DEVERR_POSITION
    idx2 = idx.copy()
    idx2[0, 2] = -1
    ref = orc.sparse_attn(c.q, c.kv_cache, orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages), [0], idx2, c.gate,
                          c.sm_scale, 64)
    assert_attn_close(bf16_to_np(out), ref)
    bt = c.block_table.copy()
    bt[0, 1] = c.num_pages + 5          # page id out of range (positions 64..127)
    idx3 = idx2.copy()
    idx3[0, 2] = 100
    pg2 = L.paged(dev(c.seq_lens), dev(bt), c.num_pages)
    L.sparse_attn(dev(c.q), dev(c.kv_cache), pg2, None, dev(idx3), dev(c.gate), c.sm_scale, 64)
    torch.cuda.synchronize()
    assert L.device_error(reset=True) & L.DEVERR_PAGE


# ------------------------------------------------------------------ SWA

def test_swa_decode_within_tolerance(L, orc):
    case = synth.swa_case(8, [1, 50, 128, 129, 5000, 64], H=16)
    out = L.swa_decode(dev(case.q), dev(case.k_ring), dev(case.v_ring), dev(case.seq_lens), case.window,
                       case.sm_scale)
    ref = orc.swa_decode(case.q, case.k_ring, case.v_ring, case.seq_lens, case.window, case.sm_scale)
    assert_attn_close(bf16_to_np(out), ref)
    no_device_error(L)


# ------------------------------------------------------------------ the layer

LAYER_CASES = [
    ("tiny_prefill_T1024", lambda: synth.tiny_prefill(0), False),
    ("decode_ragged", lambda: synth.decode_case(3, [1, 65, 2048, 2049, 7000], K=2048, HI=32), True),
    ("decode_h16", lambda: synth.decode_case(4, [5000, 12345], K=2048, HI=16), True),
    ("prefill_T300_K128", lambda: synth.prefill_case(5, 300, K=128), False),
    ("mtp_ragged_3_drafts", lambda: synth.mtp_decode(8, B=4, L=[2050, 9000, 130, 4097], n=3), False),
    ("prefill_two_seqs", lambda: synth.layer_case(
        "two", 6, [200, 300], np.r_[np.zeros(200, np.int32), np.ones(300, np.int32)],
        np.r_[np.arange(200), np.arange(300)].astype(np.int32), HI=16, DI=128, K=128, H=16, Dqk=576, Dv=512), False),
]


@pytest.mark.parametrize("name,make,decode", LAYER_CASES, ids=[c[0] for c in LAYER_CASES])
def test_layer_forward_matches_oracle(L, orc, name, make, decode):
    from long_context_sparse_02_b200.runtime import LayerOnDevice
    c = make()
    lay = LayerOnDevice(c, decode=decode)
    lay.forward()
    torch.cuda.synchronize()
    q_seq = np.arange(c.T, dtype=np.int32) if decode else c.q_seq
    q_pos = (c.seq_lens - 1).astype(np.int32) if decode else c.q_pos
    pg = orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages)
    _, idx, out = orc.layer_forward(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg, q_seq, q_pos, c.K, c.Dv,
                                    c.sm_scale)
    assert np.array_equal(lay.idx.cpu().numpy(), idx)
    assert_attn_close(bf16_to_np(lay.out), out)
    no_device_error(L)


def test_layer_decode_topk_fallbacks(L, orc):
    """Decode through dsa_layer_forward where the top-K cannot use the
    indexer's score histogram: (1) the workspace starts as garbage, so the
    counts do not add up to the row length and the first call takes the full
    path (clearing the histogram); the second call takes the histogram path;
    (2) sequence 0's key rows are reordered so its scores rise with position,
    which crowds every kept position into the last warps' lists (more than a
    warp's list holds) and sends the top-K to the full path after its sweep."""
    from long_context_sparse_02_b200.runtime import LayerOnDevice
    c = synth.decode_case(7, [100000, 9000], K=2048, HI=32)
    pg = orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages)
    q_seq = np.arange(c.T, dtype=np.int32)
    q_pos = (c.seq_lens - 1).astype(np.int32)
    sc = orc.indexer_scores(c.q_idx, c.w, c.k_cache, pg, q_seq, q_pos)
    n0 = int(c.seq_lens[0])
    order = np.argsort(sc[0, :n0], kind="stable")
    pages = c.block_table[0, np.arange(n0) // 64]
    slots = np.arange(n0) % 64
    kc = c.k_cache.copy()
    kc[pages, slots] = c.k_cache[pages[order], slots[order]]
    c.k_cache = kc
    _, idx, out = orc.layer_forward(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg, q_seq, q_pos, c.K, c.Dv,
                                    c.sm_scale)
    assert np.array_equal(idx[0], np.arange(n0 - c.K, n0))  # the rise put every kept key at the end
    lay = LayerOnDevice(c, decode=True)
    lay.ws.fill_(0xA5)
    for call in range(2):
        lay.forward()
        torch.cuda.synchronize()
        assert np.array_equal(lay.idx.cpu().numpy(), idx), call
        assert_attn_close(bf16_to_np(lay.out), out)
    no_device_error(L)


# ------------------------------------------------------------------ the append step

@pytest.mark.parametrize("DI,Dqk,n,scale", [(128, 576, 300, 1.0), (128, 576, 8, 0.0625), (64, 64, 1000, 3.0),
                                            (128, 0, 77, 0.5)], ids=["decode_576_n300", "scaled_n8", "tiny_n1000",
                                                                     "keys_only"])
def test_append_kv_bit_exact(L, orc, DI, Dqk, n, scale):
    """New tokens' keys quantised to e4m3 and latent rows copied into the
    paged caches: every byte equal to the oracle's, other rows untouched."""
    rng = np.random.default_rng(n)
    seq_lens = np.array([3000, 1700, 900], np.int32)
    bt, npg = synth.paged_layout(rng, seq_lens)
    # positions: distinct, spread over the sequences
    tok_seq = rng.integers(0, 3, n).astype(np.int32)
    tok_pos = np.empty(n, np.int32)
    for b in range(3):
        m = tok_seq == b
        tok_pos[m] = rng.choice(seq_lens[b], m.sum(), replace=False)
    # keys: a wide dynamic range, exact e4m3 midpoints, saturation, signed zeros and subnormals
    kf = (rng.standard_normal((n, DI)) * np.exp2(rng.integers(-14, 10, (n, DI)))).astype(np.float32)
    kf.ravel()[: 6 * DI] = np.resize(np.array([0.0, -0.0, 448.0, 464.0, 1e6, -1e6, 2.0 ** -10, 3 * 2.0 ** -11,
                                               0.96875, -0.96875, 17.0, 18.0], np.float32), 6 * DI)
    k_new = synth.f32_to_bf16_bits(kf)
    k_cache = rng.integers(0, 256, (npg, 64, DI)).astype(np.uint8)
    Dc = Dqk if Dqk else 8
    kv_cache = rng.integers(0, 65536, (npg, 64, Dc)).astype(np.uint16)
    lat = rng.integers(0, 65536, (n, Dc)).astype(np.uint16) if Dqk else None
    pg = orc.Paged(seq_lens, bt, 64, npg)
    ref_k, ref_v = orc.append_kv(k_new, scale, lat, tok_seq, tok_pos, pg, k_cache, kv_cache)
    dk, dv = dev(k_cache), dev(kv_cache)
    dpg = L.paged(dev(seq_lens), dev(bt), npg)
    L.append_kv(dev(k_new), scale, None if lat is None else dev(lat), dev(tok_seq), dev(tok_pos), dpg, dk,
                dv if Dqk else None)
    no_device_error(L)
    assert np.array_equal(dk.cpu().numpy(), ref_k)
    assert np.array_equal(dv.view(torch.int16).cpu().numpy().view(np.uint16), ref_v)


def test_append_kv_reports_bad_positions_without_fault(L, orc):
    seq_lens = np.array([100], np.int32)
    bt = np.array([[0, 1]], np.int32)
    pg = L.paged(dev(seq_lens), dev(bt), 2)
    k_cache = torch.zeros((2, 64, 128), dtype=torch.uint8, device="cuda")
    k_new = dev(synth.f32_to_bf16_bits(np.ones((2, 128), np.float32)))
    L.device_error(reset=True)
    L.append_kv(k_new, 1.0, None, dev(np.array([0, 0], np.int32)), dev(np.array([100, 5], np.int32)), pg,
                k_cache, None)
    torch.cuda.synchronize()
    assert L.device_error(reset=True) == 1  # DSA_DEVERR_POSITION: position 100 is past the sequence
    assert (k_cache[0, 5] == 0x38).all() and int(k_cache.sum()) == 0x38 * 128  # only the valid token landed


# ------------------------------------------------------------------ bounded waits

def test_timed_out_wait_abandons_the_launch_and_the_next_call_is_exact(L, orc):
    """A decode-indexer tile that is never filled (dsa_test_skip_indexer_tile):
    the MMA's wait on it runs out after its limit, the error word reports
    DSA_DEVERR_TIMEOUT, the launch returns (its CTAs free their tensor memory)
    and the context stays usable -- the next call, with the tile filled
    again, is bit-exact."""
    import time
    from long_context_sparse_02_b200.runtime import LayerOnDevice
    c = synth.decode_case(21, [3000, 1200], HI=32, K=256, H=16, Dqk=64, Dv=64)
    pg = orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages)
    _, idx, out = orc.layer_forward(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg,
                                    np.arange(2, dtype=np.int32), (c.seq_lens - 1).astype(np.int32), c.K, c.Dv,
                                    c.sm_scale)
    lay = LayerOnDevice(c, decode=True)
    L.device_error(reset=True)
    try:
        assert L.lib.dsa_test_skip_indexer_tile(0) == 0
        t0 = time.perf_counter()
        lay.forward()
        torch.cuda.synchronize()
        dt = time.perf_counter() - t0
    finally:
        assert L.lib.dsa_test_skip_indexer_tile(-1) == 0
    err = L.device_error(reset=True)
    assert err & L.DEVERR_TIMEOUT, hex(err)
    assert dt < 10.0, dt  # the waits are bounded: about a second each
    for _ in range(2):
        lay.forward()
        torch.cuda.synchronize()
        assert L.device_error(reset=True) == 0
        assert np.array_equal(lay.idx.cpu().numpy(), idx)
        assert_attn_close(lay.out.float().cpu().numpy().astype(np.float64), out)
    assert L.lib.dsa_test_skip_indexer_tile(-2) == 1  # out of range: rejected
