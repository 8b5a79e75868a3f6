"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI
(binding in nvfp4_w4a4_quantized_03_b200.mq) and bring results back to numpy."""
import numpy as np
import torch

from nvfp4_w4a4_quantized_03_b200 import mq


def dev():
    return torch.device("cuda:0")


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def gpu_quantize(x_cpu: torch.Tensor, alpha: float | None = None):
    """alpha (from mq_tensor_scale unless given), codes [rows, K/2], stored scales."""
    rows, K = x_cpu.shape
    x = x_cpu.to(dev())
    q = mq.QuantizedTensor(rows, K, dev())
    q.scales.fill_(0xAB)   # the quantizer must overwrite padding too
    if alpha is None:
        ws = mq.workspace(mq.mq_workspace_bytes(), dev())
        mq.mq_tensor_scale(x, q.alpha, ws)
    else:
        q.alpha.fill_(alpha)
    mq.mq_nvfp4_quantize(x, q.alpha, q.codes, q.scales)
    torch.cuda.synchronize()
    return (float(q.alpha.item()), q.codes.cpu().numpy().reshape(rows, K // 2), q.scales.cpu().numpy(), q)


def rel_frobenius(y: np.ndarray, ref: np.ndarray) -> float:
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(y - ref) / den) if den > 0 else float(np.linalg.norm(y))


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
