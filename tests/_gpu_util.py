"""Shared helpers of the GPU tests: seeded inputs on the device and the
oracle's view of them.  Inputs come only from the seeded generator; expected
values only from the oracle."""
import numpy as np
import torch

import workloads as W


def to_dev_bf16(x_u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_u16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return W.bf16_bits_to_f64(from_dev_bf16(t))


def inputs(wl):
    q, k, v = W.generate(wl)
    return (q, k, v), (to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v))


def scores_close(gpu: np.ndarray, ref64: np.ndarray, rtol=1e-5, atol=1e-30):
    """|g - o| <= rtol*|o| + atol elementwise; returns the worst ratio."""
    err = np.abs(gpu.astype(np.float64) - ref64)
    bound = rtol * np.abs(ref64) + atol
    return float((err / bound).max())


def garbage_like(shape, dtype=torch.bfloat16):
    """Buffer pre-filled with NaN bit patterns, to show unwritten rows are not read."""
    t = torch.empty(shape, dtype=dtype, device="cuda")
    t.view(torch.int16).fill_(0x7FC1)
    return t
