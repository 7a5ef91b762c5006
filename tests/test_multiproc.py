"""The N > 1 path of bench.py on CPU: two gloo ranks (no GPU).  Each rank gets its own
batch (distinct seeds, same shape) and the reported time is the maximum over ranks."""
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


def _worker(rank, world, port, out):
    import datetime
    import sys

    import torch.distributed as dist

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    base = synth.WORKLOADS["llama3_8b_32k"]
    w = bench.rank_workload(base, rank)
    k, _ = synth.gen_kv(w.with_(B=1, S=8), want_v=False)
    elapsed = [10.0 * (rank + 1), 3.0 - rank]
    got = bench.max_over_ranks(elapsed)
    out.put((rank, w.seed, int(k.sum()), w.B, w.S, got))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_take_the_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, s0, k0, B0, S0, g0), (r1, s1, k1, B1, S1, g1) = res
    assert s0 != s1 and k0 != k1            # different batches
    assert (B0, S0) == (B1, S1)              # same per-rank work (weak scaling)
    assert g0 == g1 == [20.0, 3.0]           # max over ranks, seen identically by both


def test_single_process_max_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
