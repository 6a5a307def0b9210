"""The benchmark's multi-rank path on CPU: two gloo ranks, each timing its own
replica; the reported time is the max over ranks and the tokens are summed."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    local_ms = [12.5, 20.0][rank]
    local_tokens = [800, 800][rank]
    max_ms, tokens = bench.aggregate(local_ms, local_tokens, world)
    r, w, _ = bench.dist_env()
    q.put((rank, max_ms, tokens, r, w))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_aggregation_takes_max_time_and_sums_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, max_ms, tokens, r, w in res:
        assert max_ms == 20.0 and tokens == 1600 and r == rank and w == 2
    # value = tokens / max time, as bench.py reports it
    assert abs(1600 / (20.0 / 1e3) - 80000.0) < 1e-6


def test_single_rank_aggregation_is_identity():
    import bench
    assert bench.aggregate(3.0, 8, 1) == (3.0, 8)
    assert torch.__version__
