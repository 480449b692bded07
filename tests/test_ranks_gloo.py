"""The multi-GPU bench path without GPUs: two gloo ranks on CPU check the
max-over-ranks step time and the whole-job unit count the JSON line uses."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    step_ms = 1.5 + rank            # rank 1 is the slow one
    mx = bench.max_over_ranks(step_ms)
    units = bench.sum_over_ranks(100.0)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, units))


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [2.5, 2.5]
    assert [o[2] for o in out] == [200.0, 200.0]
