"""The N>1 path on CPU: two gloo ranks split a batch of independent streams
with no data-path collective, each encodes its own share with the CPU
oracle (the GPU kernels need a GPU), and the job's time is the max over
ranks.  Checks that every unit is handled exactly once, that the shares are
balanced, and that the per-rank containers equal a single-rank run."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from lossless_bf16_kv_splitzip_b200.shard import partition


def test_partition_covers_and_balances():
    rng = np.random.default_rng(0)
    sizes = rng.integers(1, 1000, 257)
    for world in (1, 2, 3, 8):
        parts = partition(sizes, world)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(sizes)))
        loads = [int(sizes[p].sum()) for p in parts]
        assert max(loads) - min(loads) <= int(sizes.max())
    assert partition([5, 5, 5, 5], 2) == partition([5, 5, 5, 5], 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, result_dir):
    import time

    import torch.distributed as dist

    import kvgen
    import oracle
    from lossless_bf16_kv_splitzip_b200.shard import max_over_ranks, partition

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    cache = kvgen.contiguous_cache(1, layers=3, tokens=64)   # 6 small tensors
    parts = partition([c.nbytes for c in cache], world)
    t0 = time.perf_counter()
    blobs = {i: oracle.encode(cache[i]) for i in parts[rank]}
    dt = time.perf_counter() - t0
    worst = max_over_ranks(dt)
    assert worst >= dt
    for i, b in blobs.items():
        with open(os.path.join(result_dir, "r%d_u%d.bin" % (rank, i)), "wb") as f:
            f.write(b)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_split_the_batch(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    import kvgen
    import oracle
    cache = kvgen.contiguous_cache(1, layers=3, tokens=64)
    seen = {}
    for f in os.listdir(tmp_path):
        r, u = f[1:-4].split("_u")
        assert int(u) not in seen
        seen[int(u)] = open(tmp_path / f, "rb").read()
    assert sorted(seen) == list(range(len(cache)))
    for i, b in seen.items():
        assert b == oracle.encode(cache[i])
