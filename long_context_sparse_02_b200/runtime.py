"""Device-side plumbing around the C ABI: uploads a layer's inputs, owns the
output and workspace buffers and issues dsa_layer_forward on the current
stream.  No arithmetic of the layer happens here."""
from __future__ import annotations

import numpy as np
import torch

from . import _lib


def to_dev(a: np.ndarray, device="cuda", dtype=None) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a)
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device, non_blocking=False)


class LayerOnDevice:
    """A Gated DSA layer call over one synthetic case, resident on the GPU."""

    def __init__(self, case, decode: bool, device: str = "cuda", want_idx: bool = True, want_lse: bool = False):
        self.case = case
        self.decode = decode
        d = device
        self.q_idx = to_dev(case.q_idx, d)
        self.w = to_dev(case.w, d)
        self.k_cache = to_dev(case.k_cache, d)
        self.q = to_dev(case.q, d)
        self.kv_cache = to_dev(case.kv_cache, d)
        self.gate = to_dev(case.gate, d)
        self.seq_lens = to_dev(case.seq_lens, d)
        self.block_table = to_dev(case.block_table, d)
        self.q_seq = None if decode else to_dev(case.q_seq, d)
        self.q_pos = None if decode else to_dev(case.q_pos, d)
        T, H = case.T, case.H
        self.out = torch.empty((T, H, case.Dv), dtype=torch.bfloat16, device=d)
        self.idx = torch.empty((T, case.K), dtype=torch.int32, device=d) if want_idx else None
        self.lse = torch.empty((T, H), dtype=torch.float32, device=d) if want_lse else None
        self.pg = _lib.paged(self.seq_lens, self.block_table, case.num_pages, case.page_size)
        self.max_len = int(case.seq_lens.max()) if decode else int(case.q_pos.max()) + 1
        self.args = _lib.layer_args(_lib.MODE_DECODE if decode else _lib.MODE_PREFILL, self.q_idx, self.w,
                                    self.k_cache, self.q, self.kv_cache, self.gate, self.pg, self.q_seq, self.q_pos,
                                    case.K, case.Dv, case.sm_scale, self.max_len, self.out, self.idx, self.lse)
        self.ws_bytes = _lib.layer_workspace_bytes(self.args)
        # zero-filled once: decode calls find the score histogram cleared and keep it so
        self.ws = torch.zeros(max(self.ws_bytes, 256), dtype=torch.uint8, device=d)

    def forward(self):
        _lib.layer_forward(self.args, self.ws)
        return self.out

    def forward_profiled(self, events):
        _lib.layer_forward_profiled(self.args, self.ws, events)
        return self.out

    @property
    def scores(self) -> torch.Tensor:
        """The fp32 scores the last forward left at the head of the workspace."""
        ld = (self.max_len + 3) // 4 * 4
        # the score histogram comes first in decode, or with up to 64 explicit queries
        off = (self.case.T * 2048 * 4 + 255) // 256 * 256 if (self.decode or self.case.T <= 64) else 0
        return self.ws[off: off + self.case.T * ld * 4].view(torch.float32).view(self.case.T, ld)
