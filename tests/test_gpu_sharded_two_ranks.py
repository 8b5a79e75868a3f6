"""The sharded linears end to end as two ranks: two processes on cuda:0 with a
gloo process group carrying the 4-byte MAX all-reduce (the step NCCL takes
between GPUs).  Nothing in either rank's kernels waits on the other rank;
only the host-side collective joins them.

  * token sharding (ShardedLinearW4A4, rows split 300 / 700, run on a side
    stream): each rank's rows equal the single-rank linear's bit for bit, and
    the all-reduced max|x| gives the oracle's tensor-level scale of the whole
    activation ("张量级尺度", section NVFP4 微缩放量化 of the paper.rainbus.top
    digest);
  * column sharding (ColumnShardedLinearW4A4, weight rows split 768 / 1280):
    each rank's weight alpha is the whole weight's, and its columns of Y equal
    the single-rank linear's bit for bit.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

M, K, N = 1000, 4096, 2048
ROW_CUT, COL_CUT = 300, 768


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import datetime

    import numpy as np
    import torch.distributed as dist

    import oracle
    from nvfp4_w4a4_quantized_03_b200 import inputs, mq
    from nvfp4_w4a4_quantized_03_b200.sharded import ColumnShardedLinearW4A4, ShardedLinearW4A4

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    out = {"rank": rank}
    try:
        torch.cuda.set_device(0)
        dev = torch.device("cuda:0")

        def b16(t):
            return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)

        x = inputs.activation_bf16(M, K, seed=31, outlier_channels=41, outlier_scale=50.0).to(dev)
        w = inputs.weight_bf16(N, K, seed=32).to(dev)
        whole = mq.LinearW4A4(w)
        y_whole = b16(whole(x))
        # token shards, on a side stream
        a, b = (0, ROW_CUT) if rank == 0 else (ROW_CUT, M)
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        lin = ShardedLinearW4A4(w)
        y = lin(x[a:b], stream=side)
        side.synchronize()
        out["rows_equal"] = bool(np.array_equal(b16(y), y_whole[a:b]))
        amax = float(lin._amax.item())
        alpha = float(np.float32(np.float32(amax) / np.float32(2688.0)))
        out["alpha_equal"] = alpha == oracle.tensor_scale(b16(x))
        # column shards
        c, d = (0, COL_CUT) if rank == 0 else (COL_CUT, N)
        col = ColumnShardedLinearW4A4(w[c:d].contiguous())
        yc = col(x)
        torch.cuda.synchronize()
        out["w_alpha_equal"] = float(col.w.alpha.item()) == float(whole.w.alpha.item())
        out["cols_equal"] = bool(np.array_equal(b16(yc), y_whole[:, c:d]))
    except Exception as e:   # reported to the parent, which fails the test
        out["error"] = repr(e)
    finally:
        dist.destroy_process_group()
    q.put(out)


def test_sharded_linears_as_two_ranks_on_one_gpu():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=600) for _ in range(world)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in sorted(results, key=lambda v: v["rank"]):
        assert "error" not in r, r
        assert r["rows_equal"] and r["alpha_equal"], r
        assert r["w_alpha_equal"] and r["cols_equal"], r
