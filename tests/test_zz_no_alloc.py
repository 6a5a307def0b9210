"""dsa_topk_static: top-K for callers that cannot allocate device memory.

Such callers (an engine whose GPU memory is all reserved up front by its own
pool, or a latency-bound decode loop that cannot take cudaMalloc's implicit
device synchronisation) get the same selection as dsa_topk without passing a
workspace: the library keeps a fixed scratch array in each GPU's memory.  This
file runs last so that, if it fails, a run that stops at the first failure has
already run every other test; it passes both alone and after the others.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sparse_02_b200 import synth

pytestmark = pytest.mark.gpu

MAX_ROWS, MAX_LEN = 16, 1 << 20  # the limits include/dsa.h states


@pytest.fixture(scope="module")
def L():
    from long_context_sparse_02_b200 import build
    build.build()
    from long_context_sparse_02_b200 import _lib
    return _lib


def _static(L, scores, row_len, K, max_row_len, idx, ld=None):
    return L.lib.dsa_topk_static(ctypes.c_void_p(scores.data_ptr()), scores.shape[1] if ld is None else ld,
                                 ctypes.c_void_p(row_len.data_ptr()), scores.shape[0], K, max_row_len,
                                 ctypes.c_void_p(idx.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _tie_rows(seed, R, n, K):
    """Rows whose K-th largest score is shared by many positions on both sides
    of the cut (ties decided by position)."""
    rng = np.random.default_rng(seed)
    sc = rng.integers(0, 4, size=(R, n)).astype(np.float32)   # scores 0..3: thousands of equal keys
    sc[:, rng.integers(0, n, size=K // 3)] = 5.0                 # some clear winners
    return sc


CASES = [(8, 131072, 2048, "dyadic"), (3, 5000, 128, "ties"), (16, 70000, 2048, "normal"),
         (4, 40000, 2048, "heavy_ties"), (1, MAX_LEN, 2048, "normal")]


@pytest.mark.parametrize("R,n,K,kind", CASES, ids=[f"{c[0]}x{c[1]}_{c[3]}" for c in CASES])
def test_static_topk_matches_dsa_topk_and_oracle_on_two_calls(L, orc, R, n, K, kind):
    for call in range(2):   # the second call sees the first call's leftovers in the shared scratch
        sc_np = _tie_rows(100 + call, R, n, K) if kind == "heavy_ties" else synth.score_rows(100 + call, R, n, kind)
        rl_np = np.random.default_rng(200 + call).integers(0, n + 1, size=R).astype(np.int32)
        rl_np[0] = n
        sc, rl = torch.from_numpy(sc_np).cuda(), torch.from_numpy(rl_np).cuda()
        ref = L.topk(sc, rl, K, n)
        got = torch.full((R, K), -7, dtype=torch.int32, device="cuda")
        assert _static(L, sc, rl, K, n, got) == 0
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}: differs from dsa_topk"
        want = orc.topk(sc_np, rl_np, K)
        assert np.array_equal(got.cpu().numpy(), want), f"call {call}: differs from the oracle"
    assert L.device_error(reset=True) == 0


def test_static_topk_at_its_exact_limits(L, orc):
    """16 rows of 1,048,576 keys fill the scratch array to its last byte."""
    R, n, K = MAX_ROWS, MAX_LEN, 2048
    sc_np = synth.score_rows(300, R, n, "dyadic")
    rl_np = np.full(R, n, np.int32)
    rl_np[5] = n - 12345
    sc, rl = torch.from_numpy(sc_np).cuda(), torch.from_numpy(rl_np).cuda()
    ref = L.topk(sc, rl, K, n)
    for call in range(2):
        got = torch.full((R, K), -7, dtype=torch.int32, device="cuda")
        assert _static(L, sc, rl, K, n, got) == 0
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}"
    want = orc.topk(sc_np, rl_np, K)
    assert np.array_equal(got.cpu().numpy(), want)
    assert L.device_error(reset=True) == 0


def test_static_topk_rejects_sizes_beyond_its_scratch(L):
    sc = torch.zeros((MAX_ROWS + 1, 64), dtype=torch.float32, device="cuda")
    rl = torch.full((MAX_ROWS + 1,), 64, dtype=torch.int32, device="cuda")
    idx = torch.full((MAX_ROWS + 1, 8), -7, dtype=torch.int32, device="cuda")
    assert _static(L, sc, rl, 8, 64, idx) == 2                      # 17 rows > 16
    # exactly 16 rows but one key too many per row: rejected on the host, nothing launched
    big = torch.zeros((MAX_ROWS, 8), dtype=torch.float32, device="cuda")
    assert _static(L, big, rl, 8, MAX_LEN + 1, idx, ld=MAX_LEN + 4) == 2
    torch.cuda.synchronize()
    assert int((idx != -7).sum()) == 0, "a rejected call wrote its output"


def test_static_topk_allocates_no_device_memory(L):
    """After one warm-up call (the scratch address lookup), further calls leave
    the device's free memory unchanged: nothing is allocated behind the caller."""
    R, n, K = 8, 131072, 2048
    sc = torch.from_numpy(synth.score_rows(400, R, n, "normal")).cuda()
    rl = torch.full((R,), n, dtype=torch.int32, device="cuda")
    idx = torch.empty((R, K), dtype=torch.int32, device="cuda")
    assert _static(L, sc, rl, K, n, idx) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(5):
        assert _static(L, sc, rl, K, n, idx) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
