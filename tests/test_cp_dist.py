"""The context-parallel decode step's exchanges on CPU: two gloo ranks run
cp.decode_step (rank ranges, local views, the two all-gathers in order) with
a stand-in for the GPU calls built from the oracle's per-rank functions, and
rank 0's result equals the oracle's context-parallel layer for G = 2."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class OracleRank:
    """cp.CpRank's interface over the oracle (CPU, fp64): test stand-in only."""

    def __init__(self, r, G, c, orc):
        from long_context_sparse_02_b200 import cp
        self.orc, self.c = orc, c
        self.lo, self.hi, self.n, bt = cp.local_view(c.seq_lens, c.block_table, c.page_size, G, r)
        self.pg = orc.Paged(self.n, bt, c.page_size, c.num_pages)

    def candidates(self, q_idx, w):
        c, orc = self.c, self.orc
        B = len(self.n)
        cs = np.full((B, c.K), -np.inf, np.float32)
        cpos = np.full((B, c.K), -1, np.int32)
        live = np.nonzero(self.n > 0)[0]
        if len(live):
            sc = orc.indexer_scores(q_idx[live], w[live], c.k_cache, self.pg, live.astype(np.int32),
                                    (self.n[live] - 1).astype(np.int32), ld=int(self.n.max()))
            kept = orc.topk(sc, self.n[live], c.K)
            for i, b in enumerate(live):
                k = kept[i] >= 0
                cs[b, k] = sc[i, kept[i][k]]
                cpos[b, k] = kept[i][k] + self.lo[b]
        return torch.from_numpy(cs), torch.from_numpy(cpos)

    def attend(self, all_s, all_p, q, gate):
        c, orc = self.c, self.orc
        s, p = all_s.numpy(), all_p.numpy()  # [G, B, K]
        B = s.shape[1]
        idx = np.full((B, c.K), -1, np.int32)
        for b in range(B):
            v = p[:, b].reshape(-1) >= 0
            ss, pp = s[:, b].reshape(-1)[v].astype(np.float64), p[:, b].reshape(-1)[v]
            keep = np.sort(pp[np.lexsort((pp, -ss))[:c.K]])
            idx[b, :len(keep)] = keep
        li = np.where((idx >= self.lo[:, None]) & (idx < self.hi[:, None]), idx - self.lo[:, None], -1)
        o, lse = orc.sparse_attn(q, c.kv_cache, self.pg, np.arange(B, dtype=np.int32), li.astype(np.int32), gate,
                                 c.sm_scale, c.Dv, return_lse=True)
        return torch.from_numpy(o), torch.from_numpy(lse), torch.from_numpy(idx)


def merge(all_o, all_l):
    o, lse = all_o.numpy(), all_l.numpy()
    m = lse.max(axis=0)
    w = np.where(np.isneginf(lse), 0.0, np.exp(lse - np.where(np.isneginf(m), 0.0, m)))
    return torch.from_numpy((w[..., None] * o).sum(axis=0) / np.maximum(w.sum(axis=0), 1e-300)[..., None])


def _case():
    from long_context_sparse_02_b200 import synth
    return synth.decode_case(5, [700, 130, 2050], HI=4, DI=64, K=64, H=4, Dqk=64, Dv=64)


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from long_context_sparse_02_b200 import cp
    from oracle import oracle as orc
    c = _case()
    calls = []

    def all_gather(t):
        calls.append(tuple(t.shape))
        parts = [torch.empty_like(t) for _ in range(world)]
        dist.all_gather(parts, t.contiguous())
        return torch.stack(parts)

    rk = OracleRank(rank, world, c, orc)
    out, idx = cp.decode_step(rk, c.q_idx, c.w, c.q, c.gate, all_gather, merge=merge)
    q.put((rank, out.numpy(), idx.numpy(), calls))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_cp_decode_step_matches_the_oracle(orc):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    c = _case()
    pg = orc.Paged(c.seq_lens, c.block_table, c.page_size, c.num_pages)
    ref_idx, ref = orc.layer_forward_context_parallel(c.q_idx, c.w, c.k_cache, c.q, c.kv_cache, c.gate, pg, c.K,
                                                      c.Dv, c.sm_scale, 2)
    for rank, out, idx, calls in res:
        assert np.array_equal(idx, ref_idx), rank
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
        # the two exchanges, in order: candidates (scores, positions), then outputs and log-sum-exps
        assert calls == [(3, 64), (3, 64), (3, 4, 64), (3, 4)], calls
