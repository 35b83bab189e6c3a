"""Multi-process host logic of the replica (data-parallel) path, on CPU with gloo.

Each rank runs its own independent input; the only collectives are the timing
barrier and the max / sum reductions that turn per-rank times into the whole-job
throughput.  World size 2, loopback rendezvous."""
import os
import socket

import pytest
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from linear_hybrid_attention_b200 import replicas
    r, lr, ws = replicas.env_rank()
    seconds = 1.0 + rank          # rank 1 is slower: the job time is the max
    tput, tmax = replicas.job_throughput(tokens_per_rank_step=100.0, steps=3, seconds_per_rank=seconds)
    replicas.barrier()
    q.put((r, ws, replicas.rank_seed(5000, r), tput, tmax))
    dist.destroy_process_group()


def test_two_rank_throughput_is_total_over_max_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, ws0, s0, t0, m0), (r1, ws1, s1, t1, m1) = res
    assert (ws0, ws1) == (2, 2)
    assert s0 == 5000 and s1 != s0                 # independent inputs per rank
    assert m0 == m1 == 2.0                         # max over ranks
    assert t0 == t1 == pytest.approx(2 * 300.0 / 2.0)


def test_single_process_identity():
    from linear_hybrid_attention_b200 import replicas
    assert replicas.max_over_ranks(3.5) == 3.5
    tput, tmax = replicas.job_throughput(10.0, 4, 2.0)
    assert tmax == 2.0 and tput == 20.0
