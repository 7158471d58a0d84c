"""CPU: one prefill split by KV heads (and one decode step split by sequences) across gloo
ranks, gathered back along heads (sequences).  Each rank computes its shard with the fp64
oracle (the GPU kernels need a GPU); the gathered result must equal the oracle on the whole
problem exactly, since rows are independent and the oracle computes each row alone."""
import os
import queue
import socket
import sys
import time

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from sparse_hierarchical_attention_pool_b200.partition import shard_range  # noqa: E402


def test_shard_range_covers_every_unit_once():
    for n in (0, 1, 2, 3, 7, 8, 32):
        for world in (1, 2, 3, 4, 8):
            spans = [shard_range(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_prefill(q, k, v, alpha, cs):
    import oracle
    B, Hq, T, d = q.shape
    rows = [(b, h, t) for b in range(B) for h in range(Hq) for t in range(T)]
    out, _, _ = oracle.forward_rows(q.reshape(-1, d), k, v, rows, Hq, 64, alpha, cs, nthreads=2)
    return torch.from_numpy(out).float().reshape(B, Hq, T, d)


def _oracle_decode(q, kc, vc, ksum, kv_len, alpha, cs):
    import oracle
    B, Hq, d = q.shape
    rows = [(b, h, int(kv_len[b]) - 1) for b in range(B) for h in range(Hq)]
    out, _, _ = oracle.forward_rows(q.reshape(-1, d), kc, vc, rows, Hq, 64, alpha, cs, nthreads=2)
    return torch.from_numpy(out).float().reshape(B, Hq, d)


def _worker(rank, world, port, kind, q_out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world)})
    import datetime
    import torch.distributed as dist
    from sparse_hierarchical_attention_pool_b200 import inputs, partition
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        if kind == "prefill":
            _, (q, k, v) = inputs.make("16k", B=2, Hq=6, Hkv=3, T=200, d=64, n_topics=8, seed=31)
            out = partition.prefill_by_kv_heads(q, k, v, 1.5, 0.2, compute=_oracle_prefill,
                                               out_dtype=torch.float32)
        else:
            _, (q4, k, v) = inputs.make("16k", B=5, Hq=4, Hkv=2, T=300, d=64, n_topics=8, seed=32)
            lens = torch.tensor([300, 129, 64, 1, 250], dtype=torch.int32)
            q = torch.stack([q4[b, :, int(lens[b]) - 1] for b in range(5)]).contiguous()
            ksum = torch.zeros(5, 2, 300 // 64, 64)       # the oracle makes its own summaries
            out = partition.decode_by_sequences(q, k, v, ksum, lens, 1.5, 0.2, compute=_oracle_decode,
                                               out_dtype=torch.float32)
        q_out.put((rank, out.numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind,world", [("prefill", 2), ("prefill", 4), ("decode", 2), ("decode", 3)])
def test_partition_gathers_the_whole_problem(kind, world):
    import oracle
    from sparse_hierarchical_attention_pool_b200 import inputs
    oracle.build()
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, kind, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    deadline = time.monotonic() + 240
    try:
        while len(got) < world:
            try:
                r, out = q_out.get(timeout=2)
                got[r] = out
            except queue.Empty:
                dead = [p.exitcode for p in procs if p.exitcode not in (None, 0)]
                assert not dead, f"a rank exited with {dead}"
                assert time.monotonic() < deadline, "ranks did not finish"
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
    finally:
        for p in procs:
            if p.is_alive():
                p.kill()
    if kind == "prefill":
        _, (q, k, v) = inputs.make("16k", B=2, Hq=6, Hkv=3, T=200, d=64, n_topics=8, seed=31)
        ref = _oracle_prefill(q, k, v, 1.5, 0.2).numpy()
    else:
        _, (q4, k, v) = inputs.make("16k", B=5, Hq=4, Hkv=2, T=300, d=64, n_topics=8, seed=32)
        lens = torch.tensor([300, 129, 64, 1, 250], dtype=torch.int32)
        q = torch.stack([q4[b, :, int(lens[b]) - 1] for b in range(5)]).contiguous()
        ref = _oracle_decode(q, k, v, None, lens, 1.5, 0.2).numpy()
    for r in range(world):
        assert got[r].shape == ref.shape
        assert np.array_equal(got[r], ref), f"rank {r}"
