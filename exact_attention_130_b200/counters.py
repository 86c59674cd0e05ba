"""Algorithmic FLOP and byte counts used for throughput and roofline figures.

Conventions ("Bellek Duvarinin Fizigi", webturing Principia):

* "Attention'in Cebiri": the two matrix products cost 2 N^2 d_k FLOPs each
  per head, 4 N^2 d_k in total; softmax work (~3 N^2) is not counted.
  Causal attention visits half the score matrix, so its count is halved
  ("Maskeleme ve Dropout").
* "Geri Yayilim": the backward pass costs about 2.5x the forward FLOPs.
* "O(N^2) Cikmazi" / "Bellek Duvarinin Fizigi": a standard (materialising)
  forward moves about 8 N^2 bytes of fp16 score traffic per head, the
  probability matrix alone is N^2 * 2 bytes, and the roofline ridge point is
  peak FLOP/s divided by bandwidth.
* "Duvarin Otesi": the KV cache costs 2 (K and V) * d_model * layers *
  bytes-per-element per token.

Bytes for the fused kernels are the compulsory HBM traffic: every input read
once and every output written once.
"""
from __future__ import annotations

__all__ = [
    "fwd_flops", "bwd_flops", "fwd_bytes", "bwd_bytes", "decode_bytes",
    "decode_flops", "naive_matmul_time_s", "naive_io_time_s",
    "prob_matrix_bytes", "naive_intensity", "ridge_point",
    "kv_cache_bytes_per_token",
]


def fwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """4 B H N^2 d, halved under the causal mask."""
    f = 4.0 * B * H * N * N * d
    return f / 2.0 if causal else f


def bwd_flops(B: int, H: int, N: int, d: int, causal: bool) -> float:
    """2.5x the forward count."""
    return 2.5 * fwd_flops(B, H, N, d, causal)


def fwd_bytes(B: int, H: int, N: int, d: int, elem: int = 2) -> float:
    """Read Q, K, V; write O (elem bytes each) and the fp32 LSE."""
    return 4.0 * B * H * N * d * elem + 4.0 * B * H * N


def bwd_bytes(B: int, H: int, N: int, d: int, elem: int = 2) -> float:
    """Read Q, K, V, O, dO and LSE; write dQ, dK, dV."""
    return 8.0 * B * H * N * d * elem + 4.0 * B * H * N


def decode_bytes(H: int, seqlens, d: int, elem: int = 2) -> float:
    """Read every visible cached K and V row once, plus q; write O and LSE."""
    B = len(seqlens)
    cache = sum(2.0 * H * int(L) * d * elem for L in seqlens)
    return cache + 2.0 * B * H * d * elem + 4.0 * B * H


def decode_flops(H: int, seqlens, d: int) -> float:
    """q.k and p.v over every visible key: 4 H L d per sequence."""
    return sum(4.0 * H * int(L) * d for L in seqlens)


def naive_matmul_time_s(N: int, d: int, peak_flops: float) -> float:
    """Time of the 4 N^2 d matmul FLOPs of one head at peak throughput."""
    return 4.0 * N * N * d / peak_flops


def naive_io_time_s(N: int, bandwidth: float, elem: int = 2) -> float:
    """Time of the ~4 N^2 element score traffic (8 N^2 bytes in fp16)."""
    return 4.0 * N * N * elem / bandwidth


def prob_matrix_bytes(N: int, elem: int = 2) -> float:
    """Size of one head's N x N probability matrix."""
    return float(N) * N * elem


def naive_intensity(d: int, elem: int = 2) -> float:
    """FLOPs per byte of a materialising forward: 4 N^2 d / (4 N^2 elem)."""
    return 4.0 * d / (4.0 * elem)


def ridge_point(peak_flops: float, bandwidth: float) -> float:
    return peak_flops / bandwidth


def kv_cache_bytes_per_token(d_model: int, layers: int, elem: int = 2) -> float:
    return 2.0 * d_model * layers * elem
