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


def _head_worker(rank, world, port, heads, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from linear_hybrid_attention_b200 import replicas
    g = torch.Generator().manual_seed(9)
    full_in = torch.randn(heads, 40, 8, generator=g)      # the same sample on every rank
    h0, h1 = replicas.head_range(heads, rank, world)
    local = full_in[h0:h1] * 2.0 + torch.arange(h0, h1, dtype=torch.float32)[:, None, None]
    out = replicas.gather_heads(local, heads)
    q.put((rank, h0, h1, out))
    dist.destroy_process_group()


@pytest.mark.parametrize("heads,world", [(16, 2), (5, 2), (16, 3)])
def test_head_partition_gathers_the_per_head_results_in_order(heads, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_head_worker, args=(r, world, port, heads, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    g = torch.Generator().manual_seed(9)
    full_in = torch.randn(heads, 40, 8, generator=g)
    want = full_in * 2.0 + torch.arange(heads, dtype=torch.float32)[:, None, None]
    assert res[0][1] == 0 and res[-1][2] == heads                     # the blocks tile the heads
    assert all(res[r][2] == res[r + 1][1] for r in range(world - 1))
    for _, _, _, out in res:
        assert torch.equal(out, want)


def test_head_range_balanced():
    from linear_hybrid_attention_b200 import replicas
    for H in (1, 5, 16, 17):
        for G in (1, 2, 3, 8):
            blocks = [replicas.head_range(H, r, G) for r in range(G)]
            assert blocks[0][0] == 0 and blocks[-1][1] == H
            assert all(blocks[r][1] == blocks[r + 1][0] for r in range(G - 1))
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1
