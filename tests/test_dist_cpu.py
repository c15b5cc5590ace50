"""World-size-2 check of the benchmark's multi-rank host logic on CPU (gloo):
the barrier and the max-over-ranks reduction that times a weak-scaling run."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    sys.path.insert(0, ROOT)
    os.environ["CUDA_VISIBLE_DEVICES"] = ""
    import bench
    import torch.distributed as dist
    ws, r, _ = bench.dist_setup()
    bench.dist_barrier(ws)
    m = bench.dist_max(10.0 * (r + 1), ws)
    q.put((r, ws, m, dist.get_backend()))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_and_barrier():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(100)
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 and r[2] == 20.0 and r[3] == "gloo" for r in res)
