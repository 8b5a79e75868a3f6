"""The linear layers of a decoder stack's prefill, run as one CUDA graph.

Every layer applies the four projections of a Qwen3-8B-shaped decoder layer
(QKV, O, gate/up, down) through mq_linear_w4a4: the activation is quantized
to NVFP4 inside each call and multiplied with the layer's pre-quantized
weight.  The norms, attention and SwiGLU between the linears are not part of
this path, so each projection reads a fixed activation of its own shape.

With `mlp=True` each layer runs the QKV and O linears and then its MLP as
one mq_mlp_w4a4 call: the gate/up GEMM with SwiGLU in its epilogue, H
quantized with its own tensor scale, and the down GEMM; the MLP reads the
gate/up activation and writes the down projection's output.

All calls run in order on one stream and share one workspace (the library
requires only that calls sharing a workspace do not overlap on the GPU), so
the memory held is the weights, the activations, the outputs and a single
workspace sized for the largest activation (the MLP's, with H, when `mlp`).
`capture()` records the whole sequence in a CUDA graph after one eager pass
has set up every kernel's launch attributes; `replay()` launches it.

Binding-level plumbing only: each step of the path runs in libmq.so's kernels.
"""
from __future__ import annotations

import torch

from . import inputs, mq


class PrefillSequence:
    def __init__(self, layers: int, tokens: int, device, weight_seed: int = 1000, act_seed: int = 2000,
                 projections=inputs.QWEN3_8B_PROJECTIONS, mlp: bool = False):
        self.layers, self.tokens, self.device = layers, tokens, device
        self.projections = projections
        self.mlp = mlp
        names = [p.name for p in projections]
        if mlp:
            self.i_gu, self.i_down = names.index("gate_up"), names.index("down")
            self.inter = projections[self.i_gu].N // 2
            assert projections[self.i_down].K == self.inter
        # one activation and one output per projection shape, reused by every layer
        # (with mlp, the down projection's input is the MLP's H, not a fixed activation)
        self.x = [None if mlp and i == self.i_down else
                  inputs.activation_bf16(tokens, p.K, seed=act_seed + i,
                                         outlier_channels=inputs.outlier_count(p.K), outlier_scale=50.0,
                                         device=device.type if hasattr(device, "type") else device)
                  for i, p in enumerate(projections)]
        self.y = [None if mlp and i == self.i_gu else torch.empty(tokens, p.N, dtype=torch.bfloat16, device=device)
                  for i, p in enumerate(projections)]
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
        nbytes = mq.mq_linear_w4a4_workspace_bytes(tokens, kmax)
        if mlp:
            nbytes = max(nbytes, mq.mq_mlp_w4a4_workspace_bytes(tokens, projections[self.i_gu].K, self.inter))
        self.ws = mq.workspace(nbytes, device)
        self.graph = None

    def flops(self) -> float:
        return 2.0 * self.tokens * self.layers * sum(p.N * p.K for p in self.projections)

    def run(self, stream=None) -> None:
        """Every layer's linears (or linears and MLP), eagerly, on `stream`
        (default: torch's current)."""
        for layer in range(self.layers):
            for i, p in enumerate(self.projections):
                q = self.w[layer][i]
                if self.mlp and i == self.i_gu:
                    d, pd = self.w[layer][self.i_down], self.projections[self.i_down]
                    mq.mq_mlp_w4a4(self.x[i], q.codes, q.scales, q.alpha, self.inter, d.codes, d.scales, d.alpha,
                                   pd.N, self.y[self.i_down], self.ws, stream)
                elif self.mlp and i == self.i_down:
                    continue
                else:
                    mq.mq_linear_w4a4(self.x[i], q.codes, q.scales, q.alpha, p.N, self.y[i], self.ws, stream)

    def launches(self) -> int:
        """Kernel launches of one run(): two per linear, five per MLP."""
        return self.layers * (2 * (len(self.projections) - 2) + 5 if self.mlp else 2 * len(self.projections))

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
