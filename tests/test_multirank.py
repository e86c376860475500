"""Host logic of the N-GPU benchmark path on CPU: two gloo ranks, each with its own batch,
timings reduced by max over ranks and accepted tokens by sum (no data-path collective)."""

import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from speculative_decoding_04_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = bench.rank_workload(inputs.TINY, rank)
    x0 = inputs.tokens(wl).tolist()
    times = [1.0 + rank, 2.0 * (rank + 1), 0.5, 0.25 + rank]
    t, acc = bench.combine_ranks(times, 10 * (rank + 1), world, "cpu")
    q.put((rank, wl.seed, x0, t, acc))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_weak_scaling_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict((r, (seed, x0, t, acc)) for r, seed, x0, t, acc in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (s0, x00, t0, a0), (s1, x01, t1, a1) = out[0], out[1]
    assert s0 != s1 and x00 != x01                  # each rank drafts its own batch
    assert t0 == t1 == [2.0, 4.0, 0.5, 1.25]         # max over ranks
    assert a0 == a1 == 30.0                          # tokens summed over ranks
