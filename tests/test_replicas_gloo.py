"""Multi-process plumbing of the GPU replicas, exercised on the CPU with gloo (world size 2):
every rank runs its own replica of the workload and the ranks only meet to time the job."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

sys.path.insert(0, os.path.dirname(os.path.dirname(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank, world, port):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})


def _timing_worker(rank, world, port, q):
    _env(rank, world, port)
    from sparse_hierarchical_attention_pool_b200.replicas import Replicas
    r = Replicas(timeout_s=30.0, backend="gloo")
    r.barrier()
    mine = 1.0 + rank                       # rank 1 is the slow one
    slowest = r.max(mine)
    rate = r.job_throughput(units_per_rank=100.0, seconds_this_rank=mine)
    r.barrier()
    q.put((rank, r.leader, slowest, rate))
    r.close()


def _dropout_worker(rank, world, port, q):
    _env(rank, world, port)
    from sparse_hierarchical_attention_pool_b200.replicas import Replicas
    r = Replicas(timeout_s=4.0, backend="gloo")
    r.barrier()
    if rank == 1:
        q.put((rank, "left"))
        q.close()
        q.join_thread()                     # the message is out before the process goes
        os._exit(0)                         # leaves between steps, with nothing in flight
    try:
        r.max(1.0)
        q.put((rank, "no error"))
    except Exception as e:                  # the survivor learns of it through its collective
        q.put((rank, "error: " + type(e).__name__))


def _run(target, world=2, timeout=60):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=timeout) for _ in range(world)]
    for p in procs:
        p.join(timeout=timeout)
        if p.is_alive():
            p.kill()
    return sorted(out)


def test_replicas_time_the_job_by_the_slowest_rank():
    res = _run(_timing_worker)
    assert [r[0] for r in res] == [0, 1]
    assert [r[1] for r in res] == [True, False]            # rank 0 alone prints the line
    for _, _, slowest, rate in res:
        assert slowest == 2.0                               # max over ranks, on every rank
        assert rate == pytest.approx(2 * 100.0 / 2.0)      # all ranks' units / slowest time


def test_a_rank_that_leaves_surfaces_as_an_error_on_the_other():
    res = _run(_dropout_worker)
    assert res[1] == (1, "left")
    assert res[0][0] == 0 and res[0][1].startswith("error")
