"""Token-sharded W4A4 linear: the rows (tokens) of an activation are split
across ranks, one process per GPU, each holding the whole quantized weight.

Rows are independent in Y = X W^T, and so are their block scales and codes,
once every rank uses the tensor-level scale of the WHOLE activation
(alpha_x = fl32(max|x| / 2688), the pages' "张量级尺度", section NVFP4 微缩放量化
of the paper.rainbus.top digest).  The one exchange is therefore the 4-byte
maximum of the shards' max|x| (an all-reduce MAX over NCCL); with it, each
rank's output rows equal those of the single-GPU linear on the full
activation, bit for bit.

Plumbing only: max|x|, alpha, the codes/scales and the GEMM run in libmq.so's
kernels (mq_tensor_amax, mq_alpha_from_amax, mq_nvfp4_quantize,
mq_nvfp4_gemm); torch.distributed carries the 4 bytes.
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
        M, K = x_shard.shape
        assert K == self.K
        mq.mq_tensor_amax(x_shard, self._amax, self._ws, stream)
        reduce_amax(self._amax, self.group)
        qx = mq.QuantizedTensor(M, K, x_shard.device)
        mq.mq_alpha_from_amax(self._amax, qx.alpha, stream)
        mq.mq_nvfp4_quantize(x_shard, qx.alpha, qx.codes, qx.scales, stream)
        if out is None:
            out = torch.empty(M, self.N, dtype=torch.bfloat16, device=x_shard.device)
        mq.mq_nvfp4_gemm(qx.codes, qx.scales, qx.alpha, self.w.codes, self.w.scales, self.w.alpha, M, self.N, K,
                         out, self._gemm_ws, stream)
        return out
