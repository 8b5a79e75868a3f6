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


def _column_shard_worker(rank, world, port, q):
    """Column sharding on the host: each rank holds a block of the weight's
    rows (a block of Y's columns); the MAX all-reduce of the shards' max|w|
    gives the whole weight's alpha, under which the oracle's quantization of
    the rank's rows equals those rows of the whole weight's quantization."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import numpy as np
    import oracle
    from nvfp4_w4a4_quantized_03_b200 import inputs
    from nvfp4_w4a4_quantized_03_b200.sharded import reduce_amax
    w = inputs.weight_bf16(160, 128, seed=9)
    w[3, 7] = 0.75             # the largest |w| sits in rank 0's rows only
    wb = w.contiguous().view(torch.int16).numpy().view(np.uint16)
    lo, hi = rank * 80, (rank + 1) * 80
    shard = wb[lo:hi]
    amax = torch.tensor([float(((np.max(shard.astype(np.uint32) & 0x7FFF)) << 16).astype(np.uint32).view(np.float32))],
                        dtype=torch.float32)
    local = float(amax.item())
    reduce_amax(amax)
    alpha = float(np.float32(amax.item()) / np.float32(2688.0))
    whole_alpha = oracle.tensor_scale(wb)
    codes, scales = oracle.quantize(np.ascontiguousarray(shard), alpha)
    wc, wsc = oracle.quantize(wb, whole_alpha)
    q.put((rank, alpha == whole_alpha, bool(np.array_equal(codes, wc[lo:hi]) and np.array_equal(scales, wsc[lo:hi])),
           local == float(amax.item())))
    dist.destroy_process_group()


def test_two_gloo_ranks_column_shards_match_the_whole_weight():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_column_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert all(g[1] and g[2] for g in got), got
    # rank 1's own max was below the whole weight's: the all-reduce changed it
    assert got[0][3] and not got[1][3], got
