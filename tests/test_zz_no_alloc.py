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


@pytest.fixture(scope="module")
def L():
    from long_context_sparse_02_b200 import build
    build.build()
    from long_context_sparse_02_b200 import _lib
    return _lib


def _static(L, scores, row_len, K, max_row_len, idx):
    return L.lib.dsa_topk_static(ctypes.c_void_p(scores.data_ptr()), scores.shape[1],
                                 ctypes.c_void_p(row_len.data_ptr()), scores.shape[0], K, max_row_len,
                                 ctypes.c_void_p(idx.data_ptr()),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("R,n,K,kind", [(8, 131072, 2048, "dyadic"), (3, 5000, 128, "ties"),
                                        (16, 70000, 2048, "normal")])
def test_static_topk_matches_dsa_topk_on_two_calls(L, R, n, K, kind):
    for call in range(2):   # the second call sees the first call's leftovers in the shared scratch
        sc = torch.from_numpy(synth.score_rows(100 + call, R, n, kind)).cuda()
        rl_np = np.random.default_rng(200 + call).integers(0, n + 1, size=R).astype(np.int32)
        rl_np[0] = n
        rl = torch.from_numpy(rl_np).cuda()
        ref = L.topk(sc, rl, K, n)
        got = torch.full((R, K), -7, dtype=torch.int32, device="cuda")
        assert _static(L, sc, rl, K, n, got) == 0
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"call {call}"
    assert L.device_error(reset=True) == 0


def test_static_topk_rejects_sizes_beyond_its_scratch(L):
    sc = torch.zeros((17, 64), dtype=torch.float32, device="cuda")
    rl = torch.full((17,), 64, dtype=torch.int32, device="cuda")
    idx = torch.empty((17, 8), dtype=torch.int32, device="cuda")
    assert _static(L, sc, rl, 8, 64, idx) == 2                   # 17 rows > 16
    big = torch.zeros((1, 8), dtype=torch.float32, device="cuda")
    assert L.lib.dsa_topk_static(ctypes.c_void_p(big.data_ptr()), (1 << 20) + 4, ctypes.c_void_p(rl.data_ptr()),
                                 1, 8, (1 << 20) + 1, ctypes.c_void_p(idx.data_ptr()), None) == 2
