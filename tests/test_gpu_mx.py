"""MXFP8 indexer operands (E4M3 elements, one E8M0 scale per 32 along DI)
through the C ABI, against the oracle's block-scaled functions.

Inputs: every 32-element block draws its own scale code (117..132) and
stores its elements divided by that scale, so the decoded operands are the
dyadic indexer values n * 2^-4 and every sum is exact in fp32: scores and
indices must match bit for bit, and a scale applied to the wrong block or
row breaks that.  The append writes codes and scales byte for byte.
"""
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


def mx_case(seed, seq_lens, HI, **kw):
    """A decode case whose indexer operands are MXFP8 (see the module doc)."""
    c = synth.decode_case(seed, seq_lens, HI=HI, DI=128, **kw)
    r1, r2 = [np.random.default_rng(s) for s in np.random.SeedSequence(seed + 99).spawn(2)]
    c.q_idx, q_sc = synth.mx_dyadic(r1, c.q_idx.shape)
    c.k_cache, k_sc = synth.mx_dyadic(r2, c.k_cache.shape)
    return c, q_sc, k_sc


def oracle_scores(orc, c, q_sc, k_sc, q_seq, q_pos):
    pg = orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages)
    return orc.indexer_scores_mx(c.q_idx, q_sc, c.w, c.k_cache, k_sc, pg, q_seq, q_pos, ld=int(c.seq_lens.max()))


@pytest.mark.parametrize("HI,seq_lens,signed", [(32, [3000, 257, 131], True), (16, [70, 5000], False),
                                                 (32, [131072] * 8, False)],
                         ids=["32h_ragged_signed_w", "16h_ragged", "32h_8x131072"])
def test_mx_indexer_decode_bit_exact(L, orc, HI, seq_lens, signed):
    c, q_sc, k_sc = mx_case(3, seq_lens, HI, K=128, H=8, Dqk=64, Dv=64, w_signed=signed)
    B = len(c.seq_lens)
    ref = oracle_scores(orc, c, q_sc, k_sc, np.arange(B, dtype=np.int32), c.seq_lens - 1)
    ld = (int(c.seq_lens.max()) + 3) // 4 * 4
    scores = torch.full((B, ld), float("nan"), device="cuda")
    pg = L.paged(dev(c.seq_lens), dev(c.block_table), c.num_pages)
    L.indexer_scores_mx(dev(c.q_idx), dev(q_sc), dev(c.w), dev(c.k_cache), dev(k_sc), pg, None, None,
                        int(c.seq_lens.max()), scores)
    torch.cuda.synchronize()
    assert L.device_error(reset=True) == 0
    got = scores.cpu().numpy()
    for b in range(B):
        n = int(c.seq_lens[b])
        assert np.array_equal(got[b, :n].view(np.uint32), ref[b, :n].view(np.uint32)), b
        assert np.all(np.isnan(got[b, n:]))


def test_mx_indexer_explicit_queries_bit_exact(L, orc):
    """Several queries per sequence at chosen positions (draft tokens)."""
    c, _, k_sc = mx_case(5, [4000, 900], 32, K=128, H=8, Dqk=64, Dv=64)
    q_seq = np.array([0, 0, 0, 1, 1, 0], np.int32)
    q_pos = np.array([3999, 3998, 17, 899, 0, 2500], np.int32)
    r = np.random.default_rng(8)
    c.q_idx, q_sc = synth.mx_dyadic(r, (len(q_seq), 32, 128))
    c.w = synth.dyadic_weights(r, (len(q_seq), 32), signed=True)
    ref = oracle_scores(orc, c, q_sc, k_sc, q_seq, q_pos)
    scores = torch.full((len(q_seq), 4000), float("nan"), device="cuda")
    pg = L.paged(dev(c.seq_lens), dev(c.block_table), c.num_pages)
    L.indexer_scores_mx(dev(c.q_idx), dev(q_sc), dev(c.w), dev(c.k_cache), dev(k_sc), pg, dev(q_seq), dev(q_pos),
                        4000, scores)
    torch.cuda.synchronize()
    assert L.device_error(reset=True) == 0
    got = scores.cpu().numpy()
    for t in range(len(q_seq)):
        n = int(q_pos[t]) + 1
        assert np.array_equal(got[t, :n].view(np.uint32), ref[t, :n].view(np.uint32)), t


def test_mx_decode_layer_B8_L131072(L, orc):
    """The decode layer with MXFP8 indexer operands (dsa_layer_forward with
    scale pointers): indices bit for bit, outputs within the bf16 tolerance,
    on two calls that share one workspace."""
    from long_context_sparse_02_b200.runtime import LayerOnDevice
    c, q_sc, k_sc = mx_case(7, [131072] * 8, 32)
    B = c.T
    sc = oracle_scores(orc, c, q_sc, k_sc, np.arange(B, dtype=np.int32), c.seq_lens - 1)
    ref_idx = orc.topk(sc, c.seq_lens, c.K)
    pg = orc.Paged(c.seq_lens, c.block_table, 64, c.num_pages)
    ref = orc.sparse_attn(c.q, c.kv_cache, pg, np.arange(B, dtype=np.int32), ref_idx, c.gate, c.sm_scale, c.Dv)
    lay = LayerOnDevice(c, decode=True)
    qs, ks = dev(q_sc), dev(k_sc)
    args = L.layer_args(L.MODE_DECODE, lay.q_idx, lay.w, lay.k_cache, lay.q, lay.kv_cache, lay.gate, lay.pg, None,
                        None, c.K, c.Dv, c.sm_scale, lay.max_len, lay.out, lay.idx, None, qs, ks)
    ws = torch.zeros(L.layer_workspace_bytes(args), dtype=torch.uint8, device="cuda")
    for call in range(2):
        L.layer_forward(args, ws)
        torch.cuda.synchronize()
        assert L.device_error(reset=True) == 0
        assert np.array_equal(lay.idx.cpu().numpy(), ref_idx), f"call {call}: indices differ"
        got = lay.out.float().cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(got, ref, rtol=RTOL, atol=ATOL)
        assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= FRO


@pytest.mark.parametrize("DI,with_latent", [(128, True), (64, False)])
def test_mx_append_bytes_match_the_oracle(L, orc, DI, with_latent):
    """Blocks spanning 60 binades, an all-zero block (code 0) and blocks so
    small that the shared exponent clamps at -127; codes, scales and latent
    rows byte for byte."""
    rng = np.random.default_rng(4)
    seq_lens = np.array([3000, 1700], np.int32)
    bt, npg = synth.paged_layout(rng, seq_lens)
    n, Dqk = 300, 576
    tok_seq = rng.integers(0, 2, n).astype(np.int32)
    tok_pos = np.array([rng.integers(0, seq_lens[b]) for b in tok_seq], np.int32)
    _, first = np.unique(np.stack([tok_seq, tok_pos], 1), axis=0, return_index=True)  # one write per row
    keep = np.sort(first)
    tok_seq, tok_pos, n = tok_seq[keep], tok_pos[keep], len(keep)
    kf = (rng.standard_normal((n, DI)) * np.exp2(rng.integers(-30, 30, (n, DI // 32)).repeat(32, 1)))
    kf[0, :32] = 0.0                       # an all-zero block
    kf[1, 32:64] *= 2.0 ** -125            # amax near 2^-125: the shared exponent clamps at -127
    kf[2, :] = rng.integers(-448, 449, DI) * 2.0 ** 10  # saturation and ties to even
    k_new = synth.f32_to_bf16_bits(kf.astype(np.float32))
    latent = synth.normal_bf16(rng, (n, Dqk)) if with_latent else None
    k_cache = rng.integers(0, 256, (npg, 64, DI)).astype(np.uint8)
    k_sc = rng.integers(0, 256, (npg, 64, DI // 32)).astype(np.uint8)
    kv = rng.integers(0, 1 << 16, (npg, 64, Dqk)).astype(np.uint16)
    ref_k, ref_s, ref_kv = orc.append_kv_mx(k_new, latent, tok_seq, tok_pos, orc.Paged(seq_lens, bt, 64, npg),
                                            k_cache, k_sc, kv)
    dk, ds, dkv = dev(k_cache), dev(k_sc), dev(kv)
    pg = L.paged(dev(seq_lens), dev(bt), npg)
    L.append_kv_mx(dev(k_new), None if latent is None else dev(latent), dev(tok_seq), dev(tok_pos), pg, dk, ds,
                   dkv)
    torch.cuda.synchronize()
    assert L.device_error(reset=True) == 0
    assert np.array_equal(dk.cpu().numpy(), ref_k), "key codes differ"
    assert np.array_equal(ds.cpu().numpy(), ref_s), "scale codes differ"
    assert np.array_equal(dkv.view(torch.int16).cpu().numpy().view(np.uint16), ref_kv), "latent rows differ"
