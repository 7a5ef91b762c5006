"""The N > 1 path of bench.py on CPU: two gloo ranks (no GPU).  The batch is sharded over the
ranks (contiguous shards of the same job's samples), each step's decode outputs are all-gathered,
and the reported time is the maximum over ranks."""
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
    import torch

    from bit_kv_cache_26_b200.shard import gather_outputs
    base = synth.WORKLOADS["breadth_256x16k"].with_(B=5, S=8)
    b0, b1 = bench.rank_shard(base, rank, world)
    k, _ = synth.gen_kv(base, b0=b0, b1=b1, want_v=False)
    # the shard is exactly those samples of the whole job
    kall, _ = synth.gen_kv(base, want_v=False)
    assert (k == kall[b0:b1]).all()
    elapsed = [10.0 * (rank + 1), 3.0 - rank]
    got = bench.max_over_ranks(elapsed)
    # decode outputs: rank r contributes rows b0..b1 filled with their sequence index
    local = torch.arange(b0, b1, dtype=torch.float32)[:, None, None].expand(b1 - b0, 2, 4).contiguous()
    full = gather_outputs(local, base.B)
    out.put((rank, b0, b1, int(k.sum()), full[:, 0, 0].tolist(), got))
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
    (r0, a0, e0, k0, f0, g0), (r1, a1, e1, k1, f1, g1) = res
    assert (a0, e0, a1, e1) == (0, 3, 3, 5)           # contiguous shards, sizes differ by at most one
    assert f0 == f1 == [0.0, 1.0, 2.0, 3.0, 4.0]      # every rank holds the whole batch's output
    assert g0 == g1 == [20.0, 3.0]                    # max over ranks, seen identically by both


def test_shard_ranges_cover_the_batch():
    from bit_kv_cache_26_b200.shard import shard_range
    for B in (0, 1, 7, 256):
        for world in (1, 2, 3, 8):
            parts = [shard_range(B, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == B
            assert all(parts[i][1] == parts[i + 1][0] for i in range(world - 1))
            sizes = [b1 - b0 for b0, b1 in parts]
            assert max(sizes) - min(sizes) <= 1


def test_single_process_max_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
