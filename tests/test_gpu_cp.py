"""Context-parallel decode (one long sequence's history over G GPUs), with
the G ranks run one after another on this GPU through the same C-ABI calls
and exchange order as G GPUs: indices bit for bit and outputs within the
bf16 tolerance against the oracle's context-parallel layer (itself pinned to
the one-device layer)."""
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


def run_cp(L, orc, c, G):
    from long_context_sparse_02_b200 import cp
    k_cache, kv_cache = dev(c.k_cache), dev(c.kv_cache)
    ranks = [cp.CpRank(r, G, c.seq_lens, c.block_table, c.num_pages, k_cache, kv_cache, c.K, c.Dv, c.sm_scale)
             for r in range(G)]
    out, idx = cp.emulate(ranks, dev(c.q_idx), dev(c.w), dev(c.q), dev(c.gate))
    torch.cuda.synchronize()
    assert L.device_error(reset=True) == 0
    pg = orc.Paged(c.seq_lens, c.block_table, c.page_size, c.num_pages)
    ref_idx, ref = orc.layer_forward_context_parallel(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg, c.K,
                                                      c.Dv, c.sm_scale, G)
    assert np.array_equal(idx.cpu().numpy(), ref_idx), f"G={G}: indices differ"
    got = out.float().cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got, ref, rtol=RTOL, atol=ATOL)
    assert np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30) <= FRO


@pytest.mark.parametrize("G", [2, 3, 5])
def test_cp_decode_B1_L1048576(L, orc, G):
    run_cp(L, orc, synth.decode_1m(0), G)


@pytest.mark.parametrize("G", [1, 2, 3, 7])
@pytest.mark.parametrize("w_sign", [1.0, -1.0])
def test_cp_decode_threshold_ties_across_ranks(L, orc, G, w_sign):
    """Three distinct key rows only: the K-th best score is shared by
    positions held by several ranks (with negative weights every score is
    -0.0, +0.0 or below); the lower positions must win across ranks."""
    c = synth.decode_case(9, [3000, 1300], HI=4, DI=64, K=64, H=4, Dqk=64, Dv=64)
    rng = np.random.default_rng(9)
    distinct = c.k_cache.reshape(-1, c.k_cache.shape[-1])[:3].copy()
    c.k_cache = distinct[rng.integers(0, 3, size=c.k_cache.shape[:2])]
    c.w = (np.abs(c.w) * w_sign).astype(np.float32)
    run_cp(L, orc, c, G)


def test_cp_decode_ragged_batch_with_empty_ranks(L, orc):
    """Three sequences of different lengths, one shorter than K, over 5 ranks:
    some ranks hold nothing of the short ones."""
    c = synth.decode_case(4, [9000, 100, 2600], HI=16, DI=128, K=128, H=16, Dqk=576, Dv=512)
    run_cp(L, orc, c, 5)
