"""Helpers shared by the GPU tests: moving the seeded bf16 bit arrays to the
device and back, and the error measures the parity bar is stated in."""
import numpy as np
import torch

from synth import bf16_bits_to_f32

DEV = "cuda"

# Parity bar: normwise max error ||g - o||_inf / ||o||_inf per row/request.
TOL_BF16 = 1e-2
TOL_F32 = 1e-5


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    return torch.from_numpy(bits.view(np.int16)).to(DEV).view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def to_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f32(host_bits(t)).astype(np.float64)
    return t.detach().cpu().numpy().astype(np.float64)


def normwise(g: np.ndarray, o: np.ndarray) -> float:
    """||g - o||_inf / ||o||_inf (0 if both vanish)."""
    den = np.max(np.abs(o))
    num = np.max(np.abs(g - o))
    if den == 0:
        return float(num)
    return float(num / den)


def rowwise_normwise(g: np.ndarray, o: np.ndarray) -> np.ndarray:
    g = g.reshape(g.shape[0], -1)
    o = o.reshape(o.shape[0], -1)
    den = np.max(np.abs(o), axis=1)
    den[den == 0] = 1.0
    return np.max(np.abs(g - o), axis=1) / den


def same_bytes(a: torch.Tensor, b: torch.Tensor) -> bool:
    if a.shape != b.shape or a.dtype != b.dtype:
        return False
    return bool(torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8)))
