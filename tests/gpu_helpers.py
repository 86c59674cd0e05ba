"""Shared helpers of the GPU parity tests: bf16 bits -> device tensors with
NaN padding past the logical end, outputs with NaN guard bands, and the
comparison against the fp64 oracle."""
import numpy as np
import torch

import inputgen

BF16_NAN = 0x7FC0
GUARD = 64  # elements of guard band before and after every output (>= 16 B)

# Tolerances for bf16 inputs with fp32 accumulation (problem statement)
TOL_O = 1e-2
TOL_LSE = 1e-3
TOL_GRAD_REL = 2e-2


def f64(bits: np.ndarray) -> np.ndarray:
    return inputgen.bf16_bits_to_f32(bits).astype(np.float64)


def bf16_device(bits: np.ndarray, pad: int = 256) -> torch.Tensor:
    """Device bf16 tensor of the given bits, followed in memory by `pad`
    NaN elements, so a kernel that reads past the logical end sees NaN."""
    flat = np.full(bits.size + pad, BF16_NAN, dtype=np.uint16)
    flat[: bits.size] = bits.reshape(-1)
    t = torch.from_numpy(flat.view(np.int16)).cuda().view(torch.bfloat16)
    return t[: bits.size].view(bits.shape)


def f32_device(x: np.ndarray, pad: int = 256) -> torch.Tensor:
    flat = np.full(x.size + pad, np.nan, dtype=np.float32)
    flat[: x.size] = x.reshape(-1)
    t = torch.from_numpy(flat).cuda()
    return t[: x.size].view(x.shape)


class Guarded:
    """An output tensor with NaN guard bands on both sides."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape))
        self.n = n
        self.buf = torch.full((n + 2 * GUARD,), float("nan"), dtype=dtype, device="cuda")
        self.t = self.buf[GUARD: GUARD + n].view(shape)

    def guards_intact(self) -> bool:
        g = torch.cat([self.buf[:GUARD], self.buf[GUARD + self.n:]])
        return bool(torch.isnan(g.float()).all())


def max_abs(a: torch.Tensor, ref: np.ndarray) -> float:
    x = a.detach().float().cpu().numpy().astype(np.float64)
    if x.shape != ref.shape:
        raise ValueError(f"shape {x.shape} vs {ref.shape}")
    if not np.all(np.isfinite(x)):
        return float("inf")
    return float(np.max(np.abs(x - ref))) if x.size else 0.0


def rel_fro(a: torch.Tensor, ref: np.ndarray) -> float:
    x = a.detach().float().cpu().numpy().astype(np.float64)
    if not np.all(np.isfinite(x)):
        return float("inf")
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-30))
