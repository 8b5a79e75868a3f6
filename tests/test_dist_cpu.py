"""The multi-rank host path of bench.py on CPU: two gloo ranks, the timing
reduction takes the maximum over ranks and every rank takes the same
collective steps (replicas, no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench._dist()
    assert (w, r) == (world, rank)
    bench._barrier(w)
    mx = bench._max_over_ranks(10.0 + rank, w, "cpu")
    bench._barrier(w)
    q.put((rank, mx))
    dist.destroy_process_group()


def test_two_gloo_ranks_max_over_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert got == [(0, 11.0), (1, 11.0)]


def _amax_worker(rank, world, port, q):
    """Each rank holds a row shard; the MAX all-reduce of the shards' max|x|
    gives every rank the whole tensor's, hence its tensor-level scale."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np
    import oracle
    from nvfp4_w4a4_quantized_03_b200 import inputs
    from nvfp4_w4a4_quantized_03_b200.sharded import reduce_amax
    x = inputs.activation_bf16(96, 256, seed=5, outlier_channels=3, outlier_scale=50.0)
    shard = x[rank * 48:(rank + 1) * 48]
    b = shard.contiguous().view(torch.int16).numpy().view(np.uint16).astype(np.uint32) & 0x7FFF
    amax = torch.tensor([float((np.max(b) << 16).astype(np.uint32).view(np.float32))], dtype=torch.float32)
    reduce_amax(amax)
    alpha = float(np.float32(amax.item()) / np.float32(2688.0))
    whole = oracle.tensor_scale(x.contiguous().view(torch.int16).numpy().view(np.uint16))
    q.put((rank, alpha == whole, float(amax.item())))
    dist.destroy_process_group()


def test_two_gloo_ranks_share_the_global_amax():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_amax_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert got[0][1] and got[1][1] and got[0][2] == got[1][2]
