"""Pins for the CPU oracle (no GPU).

Each test ties the oracle to something other than itself: a library routine
it must reduce to in a special case (torch's FP8/bf16 casts, a numpy matmul,
torch's scaled_dot_product_attention, scipy's logsumexp), a brute-force sort,
a value worked out by hand, or an invariant the definition implies.  The
cases are chosen so that a dropped ReLU, a transposed operand, a wrong head,
page or sequence index, a wrong tie rule or a missing gate fails one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from long_context_sparse_02_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def e4m3(vals):
    return synth.f32_to_e4m3_bits(np.asarray(vals, dtype=np.float32))


def bf16(vals):
    return synth.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


def dec_e4m3_torch(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def dec_bf16_torch(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def one_seq_pages(n_rows, page_size=4, rng=None, spare=0):
    """Block table for one sequence of n_rows positions over shuffled pages."""
    nb = (n_rows + page_size - 1) // page_size
    num_pages = nb + spare
    perm = np.arange(num_pages, dtype=np.int32) if rng is None else rng.permutation(num_pages).astype(np.int32)
    return perm[:nb].reshape(1, nb), num_pages


def scatter_rows(rows, bt, page_size, num_pages, fill=0):
    """Place logical rows (one sequence) into a paged cache."""
    rows = np.asarray(rows)
    cache = np.full((num_pages, page_size) + rows.shape[1:], fill, dtype=rows.dtype)
    for s in range(rows.shape[0]):
        cache[bt[0, s // page_size], s % page_size] = rows[s]
    return cache


# ---------------------------------------------------------------- formats

def test_e4m3_decoder_matches_torch_on_all_codes(orc):
    codes = np.arange(256, dtype=np.uint8)
    ref = dec_e4m3_torch(codes)
    got = np.array([orc.e4m3_to_f64(c) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])
    assert orc.e4m3_to_f64(0x7E) == 448.0 and orc.e4m3_to_f64(0x01) == 2.0 ** -9


def test_bf16_decoder_matches_torch_on_all_codes(orc):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = dec_bf16_torch(codes)
    got = np.array([orc.bf16_to_f64(int(c)) for c in codes])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ---------------------------------------------------------------- indexer

def test_indexer_hand_worked_example(orc):
    """T=4 queries of one sequence, 2 heads of dim 2, K=2.
    kI rows: k0=[1,0] k1=[0,1] k2=[1,1] k3=[0,2].
    t=0: q=[[1,0],[0,1]] w=[1,1]:   s0: 1*relu(1)+1*relu(0) = 1
    t=1: q=[[1,1],[-1,0]] w=[1,.5]: s0: 1*1+.5*relu(-1)=1   s1: 1*1+.5*0 = 1
    t=2: q=[[2,0],[0,2]] w=[.5,.5]: s0: .5*2=1  s1: .5*2=1  s2: .5*2+.5*2 = 2
    t=3: q=[[1,-1],[.5,.5]] w=[1,2]: s0: 1*1+2*.5=2  s1: relu(-1)+2*.5=1
                                    s2: relu(0)+2*1=2  s3: relu(-2)+2*1=2
    Top-2 (ties to the lower position): t0 -> [0,-1], t1 -> [0,1],
    t2 -> {s2 (2), then s0 over s1 at 1} = [0,2], t3 -> {s0,s2 over s3} = [0,2].
    """
    k = np.array([[1, 0], [0, 1], [1, 1], [0, 2]], np.float32)
    q = np.array([[[1, 0], [0, 1]], [[1, 1], [-1, 0]], [[2, 0], [0, 2]], [[1, -1], [.5, .5]]], np.float32)
    w = np.array([[1, 1], [1, .5], [.5, .5], [1, 2]], np.float32)
    bt, npg = one_seq_pages(4, page_size=2, rng=np.random.default_rng(3), spare=1)
    kc = scatter_rows(e4m3(k), bt, 2, npg)
    pg = orc.Paged([4], bt, 2, npg)
    sc = orc.indexer_scores(e4m3(q), w, kc, pg, np.zeros(4, np.int32), np.arange(4, dtype=np.int32))
    exp = np.array([[1, -np.inf, -np.inf, -np.inf], [1, 1, -np.inf, -np.inf],
                    [1, 1, 2, -np.inf], [2, 1, 2, 2]], np.float32)
    assert np.array_equal(sc, exp)
    idx = orc.topk(sc, np.arange(1, 5, dtype=np.int32), 2)
    assert idx.tolist() == [[0, -1], [0, 1], [0, 2], [0, 2]]


def _rand_indexer(rng, T, HI, DI, L, page_size=8):
    q = rng.integers(-4, 5, size=(T, HI, DI)).astype(np.float32) / 16
    k = rng.integers(-4, 5, size=(L, DI)).astype(np.float32) / 16
    bt, npg = one_seq_pages(L, page_size, rng, spare=2)
    kc = scatter_rows(e4m3(k), bt, page_size, npg)
    return q, k, bt, npg, kc


def test_indexer_single_head_is_relu_matmul(orc):
    """H_I=1, w=1: I = max(0, Q K^T) -- a numpy matmul of the decoded operands."""
    rng = np.random.default_rng(11)
    T, DI, L = 24, 32, 40
    q, k, bt, npg, kc = _rand_indexer(rng, T, 1, DI, L)
    qpos = rng.integers(0, L, size=T).astype(np.int32)
    pg = orc.Paged([L], bt, 8, npg)
    sc = orc.indexer_scores(e4m3(q), np.ones((T, 1), np.float32), kc, pg, np.zeros(T, np.int32), qpos, ld=L)
    ref = np.maximum(dec_e4m3_torch(e4m3(q[:, 0, :])) @ dec_e4m3_torch(e4m3(k)).T, 0.0)
    for t in range(T):
        assert np.array_equal(sc[t, :qpos[t] + 1].astype(np.float64), ref[t, :qpos[t] + 1])
        assert np.all(np.isneginf(sc[t, qpos[t] + 1:]))


def test_indexer_one_hot_weight_selects_that_head(orc):
    rng = np.random.default_rng(12)
    T, HI, DI, L = 8, 4, 16, 30
    q, k, bt, npg, kc = _rand_indexer(rng, T, HI, DI, L)
    pg = orc.Paged([L], bt, 8, npg)
    qpos = np.full(T, L - 1, np.int32)
    kd = dec_e4m3_torch(e4m3(k))
    for h in range(HI):
        w = np.zeros((T, HI), np.float32)
        w[:, h] = 0.75
        sc = orc.indexer_scores(e4m3(q), w, kc, pg, np.zeros(T, np.int32), qpos)
        ref = 0.75 * np.maximum(dec_e4m3_torch(e4m3(q[:, h, :])) @ kd.T, 0.0)
        assert np.array_equal(sc.astype(np.float64), ref)


def test_indexer_linear_in_w_and_signed_w(orc):
    rng = np.random.default_rng(13)
    T, HI, DI, L = 6, 8, 32, 20
    q, k, bt, npg, kc = _rand_indexer(rng, T, HI, DI, L)
    pg = orc.Paged([L], bt, 8, npg)
    qpos = np.full(T, L - 1, np.int32)
    w1 = synth.dyadic_weights(rng, (T, HI), signed=True)
    w2 = synth.dyadic_weights(rng, (T, HI), signed=True)
    a = orc.indexer_scores(e4m3(q), w1, kc, pg, np.zeros(T, np.int32), qpos)
    b = orc.indexer_scores(e4m3(q), w2, kc, pg, np.zeros(T, np.int32), qpos)
    c = orc.indexer_scores(e4m3(q), w1 + w2, kc, pg, np.zeros(T, np.int32), qpos)
    assert np.array_equal(a + b, c)
    # negating every weight negates every score (ReLU sits before w)
    d = orc.indexer_scores(e4m3(q), -w1, kc, pg, np.zeros(T, np.int32), qpos)
    assert np.array_equal(d, -a)


def test_indexer_page_permutation_and_causality(orc):
    rng = np.random.default_rng(14)
    T, HI, DI, L, P = 10, 2, 16, 37, 8
    q = rng.integers(-4, 5, size=(T, HI, DI)).astype(np.float32) / 16
    k = rng.integers(-4, 5, size=(L, DI)).astype(np.float32) / 16
    w = synth.dyadic_weights(rng, (T, HI))
    qpos = rng.integers(0, L, size=T).astype(np.int32)
    outs = []
    for seed in (1, 2):
        bt, npg = one_seq_pages(L, P, np.random.default_rng(seed), spare=3)
        kc = scatter_rows(e4m3(k), bt, P, npg)
        outs.append(orc.indexer_scores(e4m3(q), w, kc, orc.Paged([L], bt, P, npg),
                                       np.zeros(T, np.int32), qpos, ld=L))
    assert np.array_equal(outs[0], outs[1])
    # rows after a query's position never influence it
    k2 = k.copy()
    k2[L // 2:] = 0.25
    bt, npg = one_seq_pages(L, P, np.random.default_rng(1), spare=3)
    kc = scatter_rows(e4m3(k2), bt, P, npg)
    sc = orc.indexer_scores(e4m3(q), w, kc, orc.Paged([L], bt, P, npg), np.zeros(T, np.int32), qpos, ld=L)
    for t in range(T):
        if qpos[t] < L // 2:
            assert np.array_equal(sc[t], outs[0][t])


def test_indexer_sequences_are_isolated(orc):
    """Two sequences in one cache: each query sees only its own sequence."""
    rng = np.random.default_rng(15)
    HI, DI, P = 2, 16, 4
    lens = [9, 14]
    ks = [rng.integers(-4, 5, size=(L, DI)).astype(np.float32) / 16 for L in lens]
    bt, npg = synth.paged_layout(rng, lens, P, spare_pages=2)
    kc = np.zeros((npg, P, DI), np.uint8)
    for b, L in enumerate(lens):
        for s in range(L):
            kc[bt[b, s // P], s % P] = e4m3(ks[b][s])
    q = rng.integers(-4, 5, size=(2, HI, DI)).astype(np.float32) / 16
    w = np.ones((2, HI), np.float32)
    both = orc.indexer_scores(e4m3(q), w, kc, orc.Paged(lens, bt, P, npg), np.array([1, 0], np.int32),
                              np.array([13, 8], np.int32), ld=14)
    for t, b in ((0, 1), (1, 0)):
        L = lens[b]
        ref = sum(np.maximum(dec_e4m3_torch(e4m3(q[t, h])) @ dec_e4m3_torch(e4m3(ks[b])).T, 0) for h in range(HI))
        assert np.array_equal(both[t, :L].astype(np.float64), ref)


def test_indexer_rejects_position_past_sequence(orc):
    bt, npg = one_seq_pages(4, 4)
    pg = orc.Paged([4], bt, 4, npg)
    with pytest.raises(ValueError):
        orc.indexer_scores(np.zeros((1, 1, 16), np.uint8), np.ones((1, 1), np.float32),
                           np.zeros((npg, 4, 16), np.uint8), pg, [0], [4], ld=8)


def test_dyadic_scheme_is_exact_in_fp32():
    """Bound from the input scheme: |q*k| <= (4/16)^2 per term, 128 terms, so
    |dot| <= 8 on a 2^-8 grid; w <= 1 on a 2^-6 grid; 32 heads -> |I| <= 256
    on a 2^-14 grid, i.e. at most 2^22 grid units < 2^24 (fp32's significand),
    so every partial sum in any order is exact."""
    units = 32 * 1 * (128 * 16) * (2 ** 6)   # heads * max(w)/2^-6 * max|dot|/2^-8 ... in 2^-14 units
    assert units <= 2 ** 22 < 2 ** 24


# ---------------------------------------------------------------- top-K

def brute_topk(row, n, K):
    order = sorted(range(n), key=lambda s: (-float(row[s]), s))
    sel = sorted(order[:K])
    return sel + [-1] * (K - len(sel))


@pytest.mark.parametrize("kind", ["normal", "ties", "zeros", "const", "dyadic"])
def test_topk_matches_brute_force_sort(orc, kind):
    R, n, K = 12, 97, 16
    sc = synth.score_rows(5, R, n, kind)
    rl = np.random.default_rng(6).integers(0, n + 1, size=R).astype(np.int32)
    rl[0], rl[1], rl[2] = n, K, K + 1
    idx = orc.topk(sc, rl, K)
    for r in range(R):
        assert idx[r].tolist() == brute_topk(sc[r], rl[r], K)


def test_topk_invariants_and_tie_rule(orc):
    sc = synth.score_rows(8, 20, 300, "ties")
    rl = np.full(20, 300, np.int32)
    K = 37
    idx = orc.topk(sc, rl, K)
    for r in range(20):
        sel = idx[r]
        assert len(sel) == K and np.all(np.diff(sel) > 0) and sel.max() < 300
        mask = np.zeros(300, bool)
        mask[sel] = True
        thr = sc[r][mask].min()
        assert thr >= sc[r][~mask].max()
        tied = np.flatnonzero(sc[r] == thr)
        took = np.flatnonzero(mask & (sc[r] == thr))
        assert np.array_equal(took, tied[:len(took)])


def test_topk_short_rows_keep_everything_and_signed_zero(orc):
    idx = orc.topk(np.array([[0.0, -0.0, 0.0, 5.0]], np.float32), [4], 2)
    assert idx.tolist() == [[0, 3]]
    idx = orc.topk(np.array([[0.0, -0.0, 0.0, -1.0]], np.float32), [4], 2)
    assert idx.tolist() == [[0, 1]]   # -0 ties with +0: lower positions win
    idx = orc.topk(np.zeros((2, 5), np.float32), [3, 0], 4)
    assert idx.tolist() == [[0, 1, 2, -1], [-1, -1, -1, -1]]


def test_topk_rejects_nan(orc):
    with pytest.raises(ValueError):
        orc.topk(np.array([[1.0, np.nan, 0.0]], np.float32), [3], 2)


# ---------------------------------------------------------------- attention

def _attn_case(rng, L, H, D, Dv, P=4):
    c = rng.standard_normal((L, D)).astype(np.float32)
    cb = bf16(c)
    bt, npg = one_seq_pages(L, P, rng, spare=1)
    kv = scatter_rows(cb, bt, P, npg)
    return cb, bt, npg, kv


def sdpa_gated(q_bits, c_bits, gate_bits, sm_scale, Dv, causal_T):
    """Dense causal MQA attention through torch's SDPA in fp64, times sigmoid(g)."""
    q = torch.from_numpy(dec_bf16_torch(q_bits))            # [T,H,D]
    c = torch.from_numpy(dec_bf16_torch(c_bits))            # [L,D]
    T, H, D = q.shape
    k = c[None, None].expand(1, H, -1, -1)
    v = c[None, None, :, :Dv].expand(1, H, -1, -1)
    qq = q.permute(1, 0, 2)[None]
    L = c.shape[0]
    mask = torch.ones(T, L, dtype=torch.bool).tril(L - T)
    o = torch.nn.functional.scaled_dot_product_attention(qq, k, v, attn_mask=mask, scale=sm_scale)
    o = o[0].permute(1, 0, 2)
    g = torch.sigmoid(torch.from_numpy(dec_bf16_torch(gate_bits)))
    return (o * g[..., None]).numpy()


def test_attention_with_all_positions_is_dense_causal_sdpa(orc):
    rng = np.random.default_rng(21)
    T, H, D, Dv = 19, 3, 16, 12
    cb, bt, npg, kv = _attn_case(rng, T, H, D, Dv)
    q = bf16(rng.standard_normal((T, H, D)))
    g = bf16(rng.standard_normal((T, H)))
    idx = np.array([list(range(t + 1)) + [-1] * (T - t - 1) for t in range(T)], np.int32)
    pg = orc.Paged([T], bt, 4, npg)
    out = orc.sparse_attn(q, kv, pg, np.zeros(T, np.int32), idx, g, 0.3, Dv)
    ref = sdpa_gated(q, cb, g, 0.3, Dv, T)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_attention_one_row_permutation_padding_gate(orc):
    rng = np.random.default_rng(22)
    L, H, D, Dv = 23, 4, 8, 8
    cb, bt, npg, kv = _attn_case(rng, L, H, D, Dv)
    pg = orc.Paged([L], bt, 4, npg)
    q = bf16(rng.standard_normal((1, H, D)))
    g0 = bf16(np.zeros((1, H)))
    cd = dec_bf16_torch(cb)
    # a single selected row: softmax weight 1, output = row * sigmoid(0) = row / 2
    out = orc.sparse_attn(q, kv, pg, [0], np.array([[-1, 7, -1]], np.int32), g0, 1.0, Dv)
    assert np.array_equal(out[0], np.broadcast_to(cd[7] / 2, (H, Dv)))
    sel = np.array([[3, 9, 14, 20, 2]], np.int32)
    a = orc.sparse_attn(q, kv, pg, [0], sel, g0, 0.5, Dv)
    b = orc.sparse_attn(q, kv, pg, [0], sel[:, ::-1].copy(), g0, 0.5, Dv)
    np.testing.assert_allclose(a, b, rtol=1e-14, atol=1e-15)
    c = orc.sparse_attn(q, kv, pg, [0], np.array([[3, -1, 9, 14, -1, 20, 2]], np.int32), g0, 0.5, Dv)
    np.testing.assert_allclose(a, c, rtol=1e-14, atol=1e-15)
    # inside the per-dim hull of the selected rows (times the gate 1/2)
    lo, hi = cd[sel[0]].min(0) / 2, cd[sel[0]].max(0) / 2
    assert np.all(a[0] >= lo - 1e-12) and np.all(a[0] <= hi + 1e-12)
    # a large gate logit passes the output through; g=0 halves it exactly
    big = orc.sparse_attn(q, kv, pg, [0], sel, bf16(np.full((1, H), 40.0)), 0.5, Dv)
    np.testing.assert_allclose(big, 2 * a, rtol=1e-15, atol=0)


def test_attention_lse_and_empty_selection(orc):
    from scipy.special import logsumexp
    rng = np.random.default_rng(23)
    L, H, D = 10, 2, 8
    cb, bt, npg, kv = _attn_case(rng, L, H, D, D)
    pg = orc.Paged([L], bt, 4, npg)
    q = bf16(rng.standard_normal((2, H, D)))
    idx = np.array([[1, 4, 6], [-1, -1, -1]], np.int32)
    out, lse = orc.sparse_attn(q, kv, pg, [0, 0], idx, bf16(np.zeros((2, H))), 0.25, D, return_lse=True)
    qd, cd = dec_bf16_torch(q), dec_bf16_torch(cb)
    for h in range(H):
        assert abs(lse[0, h] - logsumexp(0.25 * cd[[1, 4, 6]] @ qd[0, h])) < 1e-12
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))


# ---------------------------------------------------------------- SWA

def test_swa_matches_sdpa_over_the_window(orc):
    rng = np.random.default_rng(31)
    B, H, D, W = 3, 2, 8, 16
    case = synth.swa_case(31, [5, 16, 40], H=H, D=D, window=W)
    out = orc.swa_decode(case.q, case.k_ring, case.v_ring, case.seq_lens, W, case.sm_scale)
    for b, L in enumerate(case.seq_lens):
        pos = np.arange(max(0, L - W), L)
        slots = pos % W
        k = torch.from_numpy(dec_bf16_torch(case.k_ring[b, slots]))  # [n,H,D]
        v = torch.from_numpy(dec_bf16_torch(case.v_ring[b, slots]))
        q = torch.from_numpy(dec_bf16_torch(case.q[b]))               # [H,D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[:, None, :], k.permute(1, 0, 2), v.permute(1, 0, 2), scale=case.sm_scale)[:, 0]
        np.testing.assert_allclose(out[b], ref.numpy(), rtol=1e-12, atol=1e-12)
    assert rng is not None


# ---------------------------------------------------------------- layer

def test_layer_with_k_at_least_T_is_dense_causal_attention(orc):
    c = synth.layer_case("k_ge_t", 41, [24], np.zeros(24, np.int32), np.arange(24, dtype=np.int32),
                         HI=2, DI=16, K=32, H=3, Dqk=16, Dv=8, page_size=8, spare_pages=1)
    pg = orc.Paged(c.seq_lens, c.block_table, c.page_size, c.num_pages)
    _, idx, out = orc.layer_forward(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg, c.q_seq,
                                    c.q_pos, c.K, c.Dv, c.sm_scale)
    rows = np.stack([c.kv_cache[c.block_table[0, s // 8], s % 8] for s in range(24)])
    ref = sdpa_gated(c.q, rows, c.gate, c.sm_scale, c.Dv, 24)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)
    assert all(idx[t].tolist() == list(range(t + 1)) + [-1] * (31 - t) for t in range(24))


def test_workloads_match_page_constants():
    g = json.load(open(os.path.join(GOLDEN, "page_constants.json")))
    K = g["top_k"]["value"]
    d = synth.decode_case(0, [8], HI=g["indexer_heads"]["value"], DI=g["indexer_dim"]["value"], K=K,
                          H=2, Dqk=8, Dv=8)
    assert (d.HI, d.DI, d.K) == (32, 128, 2048)
    h = synth.decode_case(0, [8], HI=g["hybrid_indexer_heads"]["value"], K=K, H=2, Dqk=8, Dv=8)
    assert h.HI == 16
    ratio = g["context_tokens"]["value"] / K
    assert ratio == 512 and abs(ratio - g["token_reduction"]["approx"]) / 500 < 0.05
    assert synth.swa_case(0, [4], H=1, D=8, window=g["swa_window"]["value"]).window == 128


def test_synth_is_deterministic_and_dyadic():
    a = synth.tiny_prefill(0, T=64)
    b = synth.tiny_prefill(0, T=64)
    for f in ("q_idx", "w", "k_cache", "q", "kv_cache", "gate", "block_table"):
        assert np.array_equal(getattr(a, f), getattr(b, f))
    v = dec_e4m3_torch(a.q_idx) * 16
    assert np.array_equal(v, np.round(v)) and np.abs(v).max() <= 4
    assert np.array_equal(a.w * 64, np.round(a.w * 64))
    assert sorted(set(a.block_table.ravel().tolist())) == list(range(a.num_pages))


def test_draft_query_inputs_follow_their_recipe():
    """Speculative-decoding queries: the last n positions of each sequence, in
    sequence order; with_queries keeps the caches and draws new dyadic query
    tensors, the same for the same seed."""
    c = synth.mtp_decode(0, B=3, L=[500, 90, 1300], n=4, HI=8)
    assert np.array_equal(c.q_seq, np.repeat(np.arange(3), 4))
    assert np.array_equal(c.q_pos, np.concatenate([np.arange(L - 4, L) for L in (500, 90, 1300)]))
    d = synth.with_queries(c, 7, c.q_seq[::-1].copy(), c.q_pos[::-1].copy(), "reversed")
    e = synth.with_queries(c, 7, c.q_seq[::-1].copy(), c.q_pos[::-1].copy(), "reversed")
    for f in ("k_cache", "kv_cache", "block_table", "seq_lens"):
        assert getattr(d, f) is getattr(c, f)
    for f in ("q_idx", "w", "q", "gate"):
        assert np.array_equal(getattr(d, f), getattr(e, f)) and getattr(d, f).shape == getattr(c, f).shape
    v = dec_e4m3_torch(d.q_idx) * 16
    assert np.array_equal(v, np.round(v)) and np.abs(v).max() <= 4
    assert np.array_equal(d.w * 64, np.round(d.w * 64)) and d.w.min() >= 0


# ---------------------------------------------------------------- the append step (FP8 quantisation)

def _finite_e4m3_codes():
    return [c for c in range(256) if (c & 0x7F) != 0x7F]


def test_e4m3_encoder_round_trips_every_finite_code(orc):
    for c in _finite_e4m3_codes():
        assert orc.e4m3_from_f64(orc.e4m3_to_f64(c)) == c, hex(c)


def test_e4m3_encoder_rounds_midpoints_to_even_and_neighbours_to_nearest(orc):
    # every pair of adjacent finite magnitudes, from the definition: the exact
    # midpoint goes to the code with the even mantissa, anything off it to the
    # nearer code
    for c in range(0x00, 0x7E):
        lo, hi = orc.e4m3_to_f64(c), orc.e4m3_to_f64(c + 1)
        mid = (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        for sgn, sbit in ((1.0, 0x00), (-1.0, 0x80)):
            assert orc.e4m3_from_f64(sgn * mid) == even | sbit, hex(c)
            assert orc.e4m3_from_f64(sgn * math.nextafter(mid, 0.0)) == c | sbit
            assert orc.e4m3_from_f64(sgn * math.nextafter(mid, math.inf)) == (c + 1) | sbit


def test_e4m3_encoder_matches_torch_within_range_and_saturates_beyond(orc):
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(200000) * np.exp2(rng.integers(-12, 9, 200000))).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([orc.e4m3_from_f64(float(v)) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)
    for v, code in ((448.0, 0x7E), (463.99, 0x7E), (464.0, 0x7E), (465.0, 0x7E), (1e30, 0x7E), (-1e30, 0xFE),
                    (-500.0, 0xFE), (0.0, 0x00), (-0.0, 0x80), (2.0 ** -10, 0x00), (2.0 ** -9, 0x01)):
        assert orc.e4m3_from_f64(v) == code, v


def test_append_places_rows_through_the_block_table_and_scales_before_rounding(orc):
    rng = np.random.default_rng(8)
    bt, npg = one_seq_pages(12, page_size=4, rng=rng, spare=2)
    seq_lens = np.array([12], np.int32)
    pg = orc.Paged(seq_lens, bt, 4, npg)
    k_cache = np.full((npg, 4, 8), 0x55, np.uint8)
    kv_cache = np.full((npg, 4, 6), 0x1234, np.uint16)
    kf = np.array([[1.0, -1.5, 0.3, 448.0, 600.0, 2.0 ** -10, -0.0, 7.0]] * 3, np.float32) * np.array([[1], [2], [3]],
                                                                                                     np.float32)
    k_new = bf16(kf)
    lat = rng.integers(0, 65536, (3, 6)).astype(np.uint16)
    pos = np.array([11, 0, 5], np.int32)
    kc, vc = orc.append_kv(k_new, 0.5, lat, np.zeros(3, np.int32), pos, pg, k_cache, kv_cache)
    touched = np.zeros((npg, 4), bool)
    for j, p in enumerate(pos):
        page, slot = bt[0, p // 4], p % 4
        touched[page, slot] = True
        xs = dec_bf16_torch(k_new[j]).astype(np.float32) * np.float32(0.5)
        expect = torch.from_numpy(np.clip(xs, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(kc[page, slot], expect)
        assert np.array_equal(vc[page, slot], lat[j])
    assert (kc[~touched] == 0x55).all() and (vc[~touched] == 0x1234).all()
    with pytest.raises(ValueError):  # position past the sequence
        orc.append_kv(k_new[:1], 1.0, lat[:1], np.zeros(1, np.int32), np.array([12], np.int32), pg, k_cache, kv_cache)


# ---------------------------------------------------------------- MXFP8 (32-element blocks sharing an E8M0 scale)

def test_e8m0_decoder_is_a_power_of_two_on_every_code(orc):
    for c in range(255):
        assert orc.e8m0_to_f64(c) == math.ldexp(1.0, c - 127), c
    assert math.isnan(orc.e8m0_to_f64(255))


def test_mx_encoder_hand_worked_blocks(orc):
    with open(os.path.join(GOLDEN, "mxfp8_blocks.json")) as f:
        blocks = json.load(f)["blocks"]
    for blk in blocks:
        x = np.zeros(32)
        x[:len(blk["values"])] = [float.fromhex(v) for v in blk["values"]]
        expect = np.zeros(32, np.uint8)
        expect[:len(blk["codes"])] = blk["codes"]
        codes, scale = orc.mx_encode(x[None])
        assert int(scale[0, 0]) == blk["scale"], blk["name"]
        assert np.array_equal(codes[0], expect), blk["name"]


def test_mx_encoder_round_trips_representable_blocks(orc):
    """A block whose largest magnitude is an E4M3 value in [256, 448] times
    2^k, all elements E4M3 values times 2^k, comes back exactly, scale 127+k."""
    rng = np.random.default_rng(21)
    finite = np.array(_finite_e4m3_codes(), np.uint8)
    for _ in range(200):
        codes = rng.choice(finite, 32).astype(np.uint8)
        codes[rng.integers(32)] = rng.integers(0x78, 0x7F) | (0x80 if rng.random() < 0.5 else 0)
        k = int(rng.integers(-100, 101))
        c2, s2 = orc.mx_encode(np.ldexp(dec_e4m3_torch(codes), k)[None])
        assert int(s2[0, 0]) == 127 + k
        assert np.array_equal(c2[0], codes)


def test_mx_encoder_elements_match_torch_and_the_scale_brackets_the_largest(orc):
    """Given the chosen scale, every element is torch's E4M3 cast of x / scale
    (clipped to the largest finite value), and the largest magnitude over the
    scale lies in [256, 512)."""
    rng = np.random.default_rng(22)
    x = (rng.standard_normal((500, 32)) * np.exp2(rng.integers(-30, 30, (500, 1)))).astype(np.float32)
    x[::7, 5] = 0.0
    x = x.astype(np.float64)
    codes, scales = orc.mx_encode(x)
    sh = scales.astype(np.int64) - 127
    r = np.abs(x).max(axis=1) * np.exp2(-sh[:, 0])
    assert np.all((r >= 256.0) & (r < 512.0))
    y = np.clip(x * np.exp2(-sh), -448.0, 448.0).astype(np.float32)  # exact: a power-of-two scaling of fp32 values
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_mx_encoder_sign_and_power_of_two_invariance(orc):
    rng = np.random.default_rng(24)
    x = (rng.standard_normal((200, 32)) * np.exp2(rng.integers(-20, 20, (200, 1)))).astype(np.float32)
    x = x.astype(np.float64)
    c, s = orc.mx_encode(x)
    cn, sn = orc.mx_encode(-x)
    assert np.array_equal(sn, s) and np.array_equal(cn, c ^ 0x80)
    for j in (-5, 3, 17):
        cj, sj = orc.mx_encode(np.ldexp(x, j))
        assert np.array_equal(cj, c) and np.array_equal(sj.astype(np.int64), s.astype(np.int64) + j)


def _mx_operands(rng, shape):
    """E4M3 elements in {-4..4}/16 and scale codes in [124, 130]: every sum below is exact in fp32."""
    codes = e4m3(rng.integers(-4, 5, size=shape).astype(np.float32) / 16)
    scales = rng.integers(124, 131, size=shape[:-1] + (shape[-1] // 32,)).astype(np.uint8)
    return codes, scales


def _mx_values(codes, scales):
    """Dequantised with library routines: torch's E4M3 cast and ldexp."""
    return dec_e4m3_torch(codes) * np.repeat(np.ldexp(1.0, scales.astype(np.int64) - 127), 32, axis=-1)


def test_mx_indexer_is_relu_matmul_of_the_dequantised_operands_per_head(orc):
    """One-hot weights pick each head in turn: I = w * max(0, Q_h K^T) on the
    dequantised operands (a numpy matmul).  Scales differ per head, per
    32-block and per key row; the cache's unused rows hold NaN scales."""
    rng = np.random.default_rng(23)
    T, HI, DI, L, P = 6, 3, 96, 40, 8
    qc, qs = _mx_operands(rng, (T, HI, DI))
    kc_rows, ks_rows = _mx_operands(rng, (L, DI))
    bt, npg = one_seq_pages(L, P, rng, spare=2)
    kc = scatter_rows(kc_rows, bt, P, npg)
    ks = scatter_rows(ks_rows, bt, P, npg, fill=255)
    pg = orc.Paged([L], bt, P, npg)
    qpos = rng.integers(0, L, T).astype(np.int32)
    Qd, Kd = _mx_values(qc, qs), _mx_values(kc_rows, ks_rows)
    for h in range(HI):
        w = np.zeros((T, HI), np.float32)
        w[:, h] = 0.75
        sc = orc.indexer_scores_mx(qc, qs, w, kc, ks, pg, np.zeros(T, np.int32), qpos, ld=L)
        ref = (0.75 * np.maximum(Qd[:, h, :] @ Kd.T, 0.0)).astype(np.float32)
        for t in range(T):
            n = qpos[t] + 1
            assert np.array_equal(sc[t, :n], ref[t, :n]), (h, t)
            assert np.all(np.isneginf(sc[t, n:]))


def test_mx_indexer_with_unit_scales_is_the_fp8_indexer_and_uniform_scales_shift_it(orc):
    rng = np.random.default_rng(26)
    T, HI, DI, L = 5, 4, 64, 30
    q, k, bt, npg, kc = _rand_indexer(rng, T, HI, DI, L)
    w = (rng.integers(-64, 65, (T, HI)) / 64).astype(np.float32)
    pg = orc.Paged([L], bt, 8, npg)
    qpos = rng.integers(0, L, T).astype(np.int32)
    z = np.zeros(T, np.int32)
    ref = orc.indexer_scores(e4m3(q), w, kc, pg, z, qpos, ld=L)

    def mx(qe, ke):
        return orc.indexer_scores_mx(e4m3(q), np.full((T, HI, DI // 32), 127 + qe, np.uint8), w, kc,
                                     np.full(kc.shape[:2] + (DI // 32,), 127 + ke, np.uint8), pg, z, qpos, ld=L)

    assert np.array_equal(mx(0, 0).view(np.uint32), ref.view(np.uint32))
    fin = np.isfinite(ref)
    assert np.array_equal(mx(2, -5)[fin], np.ldexp(ref[fin], -3))


def test_mx_append_places_encoded_blocks_and_scales_through_the_block_table(orc):
    rng = np.random.default_rng(25)
    DI, P, L = 64, 4, 12
    bt, npg = one_seq_pages(L, P, rng, spare=2)
    pg = orc.Paged(np.array([L], np.int32), bt, P, npg)
    k_cache = np.full((npg, P, DI), 0x55, np.uint8)
    k_scales = np.full((npg, P, DI // 32), 0xAA, np.uint8)
    kv_cache = np.full((npg, P, 6), 0x1234, np.uint16)
    kf = (rng.standard_normal((3, DI)) * np.exp2(rng.integers(-20, 20, (3, 2)).repeat(32, axis=1))).astype(np.float32)
    k_new = bf16(kf)
    lat = rng.integers(0, 65536, (3, 6)).astype(np.uint16)
    pos = np.array([11, 0, 5], np.int32)
    kc, ks, vc = orc.append_kv_mx(k_new, lat, np.zeros(3, np.int32), pos, pg, k_cache, k_scales, kv_cache)
    codes, scales = orc.mx_encode(dec_bf16_torch(k_new))
    touched = np.zeros((npg, P), bool)
    for j, p in enumerate(pos):
        page, slot = bt[0, p // P], p % P
        touched[page, slot] = True
        assert np.array_equal(kc[page, slot], codes[j])
        assert np.array_equal(ks[page, slot], scales[j])
        assert np.array_equal(vc[page, slot], lat[j])
    assert (kc[~touched] == 0x55).all() and (ks[~touched] == 0xAA).all() and (vc[~touched] == 0x1234).all()
    with pytest.raises(ValueError):  # position past the sequence
        orc.append_kv_mx(k_new[:1], lat[:1], np.zeros(1, np.int32), np.array([12], np.int32), pg, k_cache, k_scales,
                         kv_cache)
    with pytest.raises(ValueError):  # a row that is not whole blocks
        orc.append_kv_mx(k_new[:, :48], None, np.zeros(3, np.int32), pos, pg, k_cache[..., :48],
                         k_scales[..., :1], kv_cache)


# ---------------------------------------------------------------- context-parallel decode (one long sequence over G ranks)

def _decode_ref(orc, c):
    pg = orc.Paged(c.seq_lens, c.block_table, c.page_size, c.num_pages)
    B = len(c.seq_lens)
    _, idx, out = orc.layer_forward(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg,
                                    np.arange(B, dtype=np.int32), (c.seq_lens - 1).astype(np.int32), c.K, c.Dv,
                                    c.sm_scale)
    return pg, idx, out


def test_context_parallel_decode_is_the_single_device_layer(orc):
    """Splitting each sequence's history over G ranks (local top-K, union cut
    to K, per-rank attention merged by log-sum-exp weights) reproduces the
    one-device layer: indices exactly, outputs to fp64 rounding.  G = 40
    leaves most ranks of the short sequences empty."""
    for lens in ([700, 130, 2050], [40, 700]):  # the 40-token sequence is shorter than K: all of it is kept
        c = synth.decode_case(5, lens, HI=4, DI=64, K=64, H=4, Dqk=64, Dv=64)
        pg, idx, out = _decode_ref(orc, c)
        for G in (1, 2, 3, 5, 40):
            got_idx, got = orc.layer_forward_context_parallel(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg,
                                                              c.K, c.Dv, c.sm_scale, G)
            assert np.array_equal(got_idx, idx), (lens, G)
            np.testing.assert_allclose(got, out, rtol=1e-12, atol=1e-13)
    assert np.array_equal(idx[0, :40], np.arange(40)) and (idx[0, 40:] == -1).all()


@pytest.mark.parametrize("w_sign", [1.0, -1.0])
def test_context_parallel_decode_breaks_threshold_ties_across_ranks_by_position(orc, w_sign):
    """Every key row is one of three rows, so each query's scores take at
    most three values and the K-th best is shared by positions in several
    ranks: the union must keep the lowest of them, as one device does.  With
    negative weights every score is -0.0 or +0.0 or below."""
    c = synth.decode_case(9, [3000, 1300], HI=4, DI=64, K=64, H=4, Dqk=64, Dv=64)
    rng = np.random.default_rng(9)
    distinct = c.k_cache.reshape(-1, c.k_cache.shape[-1])[:3].copy()
    pick = rng.integers(0, 3, size=c.k_cache.shape[:2])
    c.k_cache = distinct[pick]
    c.w = (np.abs(c.w) * w_sign).astype(np.float32)
    pg, idx, out = _decode_ref(orc, c)
    sc = orc.indexer_scores(c.q_idx, c.w, c.k_cache, pg, np.arange(2, dtype=np.int32),
                            (c.seq_lens - 1).astype(np.int32))
    spans = []
    for G in (2, 3, 7):
        got_idx, got = orc.layer_forward_context_parallel(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg, c.K,
                                                          c.Dv, c.sm_scale, G)
        assert np.array_equal(got_idx, idx), G
        np.testing.assert_allclose(got, out, rtol=1e-12, atol=1e-13)
        for b in range(2):
            row = sc[b, :c.seq_lens[b]]
            kth = np.sort(row)[::-1][c.K - 1]
            rr = orc.rank_ranges(int(c.seq_lens[b]), c.page_size, G)
            spans.append(len({r for p in np.nonzero(row == kth)[0] for r, (lo, hi) in enumerate(rr) if lo <= p < hi}))
    assert max(spans) >= 2  # the case does put threshold ties in several ranks


def test_rank_ranges_cover_the_sequence_in_whole_pages(orc):
    for L, G in ((700, 3), (130, 5), (64, 2), (1, 4), (0, 2), (1 << 20, 8)):
        rr = orc.rank_ranges(L, 64, G)
        assert len(rr) == G and rr[0][0] == 0 and rr[-1][1] == L
        for (lo, hi), (lo2, _) in zip(rr, rr[1:]):
            assert lo <= hi == lo2
        assert all(lo % 64 == 0 for lo, hi in rr if hi > lo)  # a non-empty range starts on a page
