"""The linear layers of a decoder stack's prefill, run as one CUDA graph.

Every layer applies the four projections of a Qwen3-8B-shaped decoder layer
(QKV, O, gate/up, down) through mq_linear_w4a4: the activation is quantized
to NVFP4 inside each call and multiplied with the layer's pre-quantized
weight.  The norms, attention and SwiGLU between the linears are not part of
this path, so each projection reads a fixed activation of its own shape.

All calls run in order on one stream and share one workspace (the library
requires only that calls sharing a workspace do not overlap on the GPU), so
the memory held is the weights, the activations, the outputs and a single
workspace sized for the largest activation.  `capture()` records the whole
sequence in a CUDA graph after one eager pass has set up every kernel's
launch attributes; `replay()` launches it.

Binding-level plumbing only: each step of the path runs in libmq.so's kernels.
"""
from __future__ import annotations

import torch

from . import inputs, mq


class PrefillSequence:
    def __init__(self, layers: int, tokens: int, device, weight_seed: int = 1000, act_seed: int = 2000,
                 projections=inputs.QWEN3_8B_PROJECTIONS):
        self.layers, self.tokens, self.device = layers, tokens, device
        self.projections = projections
        # one activation and one output per projection shape, reused by every layer
        self.x = [inputs.activation_bf16(tokens, p.K, seed=act_seed + i,
                                         outlier_channels=inputs.outlier_count(p.K), outlier_scale=50.0,
                                         device=device.type if hasattr(device, "type") else device)
                  for i, p in enumerate(projections)]
        self.y = [torch.empty(tokens, p.N, dtype=torch.bfloat16, device=device) for p in projections]
        # weights: quantized once, offline (their bf16 copies are dropped)
        self.w = []
        for layer in range(layers):
            row = []
            for i, p in enumerate(projections):
                wb = inputs.weight_bf16(p.N, p.K, seed=weight_seed + 16 * layer + i, device=device.type)
                row.append(mq.quantize(wb))
                del wb
            self.w.append(row)
        kmax = max(p.K for p in projections)
        self.ws = mq.workspace(mq.mq_linear_w4a4_workspace_bytes(tokens, kmax), device)
        self.graph = None

    def flops(self) -> float:
        return 2.0 * self.tokens * self.layers * sum(p.N * p.K for p in self.projections)

    def run(self, stream=None) -> None:
        """Every layer's four linears, eagerly, on `stream` (default: torch's current)."""
        for layer in range(self.layers):
            for i, p in enumerate(self.projections):
                q = self.w[layer][i]
                mq.mq_linear_w4a4(self.x[i], q.codes, q.scales, q.alpha, p.N, self.y[i], self.ws, stream)

    def capture(self) -> None:
        """Record run() in a CUDA graph (after an eager pass, so that every
        kernel's attributes and cached launch data are set up outside the
        capture)."""
        self.run()
        torch.cuda.synchronize()
        s = torch.cuda.Stream(device=self.device)
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                self.run(s)
        torch.cuda.current_stream().wait_stream(s)
        self.graph = g

    def replay(self) -> None:
        self.graph.replay()

    def status(self) -> int:
        return mq.mq_read_status(self.ws)
