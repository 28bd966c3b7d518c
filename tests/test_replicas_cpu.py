"""Multi-GPU runs split one layer over the ranks by kv-head group, and the layer's time is
the slowest rank's.  The host logic of that, on two and three gloo ranks on the CPU: the
max-over-ranks reduction every rank sees, and a rank that dies before the collective
ending its peer's wait with an error (no hang)."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def _timing_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    dist = _init(rank, world, port, 30)
    local = [3.25, 5.5, 4.0][rank]
    m = bench.max_over_ranks(local, dist, device="cpu")
    q.put((rank, m))
    dist.barrier()
    dist.destroy_process_group()


def _dying_worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    dist = _init(rank, world, port, 5)
    if rank == 1:
        os._exit(0)                       # leaves before the collective
    try:
        bench.max_over_ranks(1.0, dist, device="cpu")
        q.put((rank, "returned"))
    except Exception as e:                # the peer's wait ends with an error
        q.put((rank, type(e).__name__))


def _run(target, world, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout)
    alive = [p for p in procs if p.is_alive()]
    for p in alive:
        p.kill()
    assert not alive, "a rank did not finish"
    out = []
    while not q.empty():
        out.append(q.get())
    return out


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_report_the_slowest_rank(world):
    res = sorted(_run(_timing_worker, world))
    slowest = max([3.25, 5.5, 4.0][:world])
    assert [r[0] for r in res] == list(range(world))
    assert all(r[1] == slowest for r in res)


def test_a_rank_that_leaves_ends_its_peers_wait_with_an_error():
    res = _run(_dying_worker, 2)
    assert len(res) == 1 and res[0][0] == 0 and res[0][1] != "returned"
