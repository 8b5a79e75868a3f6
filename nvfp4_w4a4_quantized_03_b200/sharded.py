"""Sharded W4A4 linears, one process per GPU.

Token sharding (ShardedLinearW4A4): the rows (tokens) of an activation are
split across ranks, each holding the whole quantized weight.

Rows are independent in Y = X W^T, and so are their block scales and codes,
once every rank uses the tensor-level scale of the WHOLE activation
(alpha_x = fl32(max|x| / 2688), the pages' "张量级尺度", section NVFP4 微缩放量化
of the paper.rainbus.top digest).  The one exchange is therefore the 4-byte
maximum of the shards' max|x| (an all-reduce MAX over NCCL); with it, each
rank's output rows equal those of the single-GPU linear on the full
activation, bit for bit.

Column sharding (ColumnShardedLinearW4A4): the rows of the weight (output
columns of Y) are split across ranks, each holding the whole activation.
The weight's tensor scale is that of the WHOLE weight (one alpha per GEMM
operand), so preparing the shards takes the same 4-byte all-reduce (MAX) of
max|w|, once; each call then needs no exchange at all: every rank quantizes
the full activation identically and computes its columns of Y, which equal
those of the single-GPU linear bit for bit.  Gathering Y is left to the
consumer (an all-gather along the columns, if it needs the whole Y).

Plumbing only: max|x|, alpha, the codes/scales and the GEMM run in libmq.so's
kernels (mq_tensor_amax, mq_alpha_from_amax, mq_nvfp4_quantize,
mq_nvfp4_gemm, mq_linear_w4a4); torch.distributed carries the 4 bytes.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import mq


def reduce_amax(amax: torch.Tensor, group=None) -> torch.Tensor:
    """All-reduce (MAX) of a one-element fp32 max|x| over the ranks of `group`
    (max is exact in fp32, so every rank gets the same bits).  A no-op
    without an initialised process group or with one rank."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


class ShardedLinearW4A4:
    """y_shard = x_shard W^T with the activation quantized under the global
    alpha_x of all ranks' shards.  W is quantized once at construction (its
    alpha over the whole weight, as in the single-GPU linear)."""

    def __init__(self, weight: torch.Tensor, group=None):
        assert weight.dtype == torch.bfloat16 and weight.is_cuda
        self.N, self.K = weight.shape
        self.w = mq.quantize(weight.contiguous())
        self.group = group
        dev = weight.device
        self._ws = mq.workspace(mq.mq_workspace_bytes(), dev)
        self._amax = torch.zeros(1, dtype=torch.float32, device=dev)
        self._gemm_ws = mq.workspace(mq.mq_workspace_bytes(), dev)

    def __call__(self, x_shard: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Every step runs on `stream` (default: the current stream): the
        kernels, the all-reduce (torch.distributed orders a collective after
        the work of the stream that is current when it is called, and the
        work after it behind it), and the allocations of the call's buffers.
        The caller orders x_shard's producer (and any given `out`) before
        `stream`, as for any stream-ordered call."""
        M, K = x_shard.shape
        assert K == self.K
        s = torch.cuda.current_stream(x_shard.device) if stream is None else stream
        with torch.cuda.stream(s):
            mq.mq_tensor_amax(x_shard, self._amax, self._ws)
            reduce_amax(self._amax, self.group)
            qx = mq.QuantizedTensor(M, K, x_shard.device)
            mq.mq_alpha_from_amax(self._amax, qx.alpha)
            mq.mq_nvfp4_quantize(x_shard, qx.alpha, qx.codes, qx.scales)
            if out is None:
                out = torch.empty(M, self.N, dtype=torch.bfloat16, device=x_shard.device)
            mq.mq_nvfp4_gemm(qx.codes, qx.scales, qx.alpha, self.w.codes, self.w.scales, self.w.alpha, M, self.N,
                             K, out, self._gemm_ws)
        return out


def quantize_weight_shard(w_shard: torch.Tensor, group=None) -> mq.QuantizedTensor:
    """NVFP4 form of this rank's rows of a weight, under the tensor scale of
    the whole weight: max|w| of the shard, all-reduce (MAX), alpha from it,
    then the shard's codes and scales."""
    assert w_shard.dtype == torch.bfloat16 and w_shard.is_cuda and w_shard.dim() == 2
    rows, K = w_shard.shape
    dev = w_shard.device
    ws = mq.workspace(mq.mq_workspace_bytes(), dev)
    amax = torch.zeros(1, dtype=torch.float32, device=dev)
    mq.mq_tensor_amax(w_shard.contiguous(), amax, ws)
    reduce_amax(amax, group)
    q = mq.QuantizedTensor(rows, K, dev)
    mq.mq_alpha_from_amax(amax, q.alpha)
    mq.mq_nvfp4_quantize(w_shard.contiguous(), q.alpha, q.codes, q.scales)
    return q


class ColumnShardedLinearW4A4:
    """y[:, shard] = x W_shard^T with W_shard this rank's rows of the weight,
    quantized under the whole weight's alpha (quantize_weight_shard); the
    call is mq_linear_w4a4 on the full activation, with no exchange."""

    def __init__(self, w_shard: torch.Tensor, group=None):
        self.N, self.K = w_shard.shape
        self.w = quantize_weight_shard(w_shard, group)
        self._ws = None

    def __call__(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        M, K = x.shape
        assert K == self.K
        s = torch.cuda.current_stream(x.device) if stream is None else stream
        with torch.cuda.stream(s):
            need = mq.mq_linear_w4a4_workspace_bytes(M, K)
            if self._ws is None or self._ws.numel() < need:
                self._ws = mq.workspace(need, x.device)
            if out is None:
                out = torch.empty(M, self.N, dtype=torch.bfloat16, device=x.device)
            mq.mq_linear_w4a4(x, self.w.codes, self.w.scales, self.w.alpha, self.N, out, self._ws)
        return out
