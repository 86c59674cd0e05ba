"""CPU oracle for the FP8 forward with incoherent processing.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this
module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it. It shares no code with the CUDA library.

What it follows:

* "FlashAttention-3 (TR)", section "FlashAttention-3'un Teknik
  Yenilikleri", item 3 "Kuantizasyon Hatasini Azaltarak Dusuk Hassasiyet
  (FP8) Kullanimi": before attention, Q and K are multiplied by a random
  orthogonal matrix (a Hadamard matrix, for instance), which spreads
  outlier coordinates over all coordinates; then they are quantised to FP8;
  since the matrix is orthogonal it cancels in Q K^T. The page reports about
  2.6x lower attention error than plain FP8.
* "Bellek Duvarinin Fizigi", section "FlashAttention-2, -3 ve -4:
  Utilizasyon Savasi", the FlashAttention-3 paragraph: the FP8 path keeps
  its accuracy with block-wise scaling and random sign factors.

Readings taken where the pages stop (each one listed with the design notes):

* the orthogonal matrix is diag(sigma) H_d / sqrt(d): random signs sigma
  (passed in; only the sign of each entry counts) times the Sylvester
  Hadamard matrix. The CUDA path applies the unnormalised H_d and folds
  the 1/d into Q's block scales, which is exact (d is a power of two);
* FP8 is e4m3 (4 exponent bits, bias 7, 3 mantissa bits, no infinities,
  largest finite 448), rounding to nearest even with saturation to +-448;
* block-wise scaling: one fp32 scale per 128-row block of each head of the
  rotated Q and K, scale = max|x| / 448 (1 when the block is all zero), the
  code of x being e4m3(x / scale) with the fp32 quotient; V is not rotated
  and has one scale per head, max|v| / 448;
* the fp32 rotation is the butterfly form of the Walsh-Hadamard transform,
  strides 1, 2, 4, ..., d/2 in that order, each pair (i, i + h) (bit h of i
  clear) becoming (x_i + x_{i+h}, x_i - x_{i+h}) in fp32, so that both
  sides reach the same fp32 values and hence the same codes;
* the attention itself is then the exact attention of the dequantised
  tensors (the definition the bf16 oracle computes); rounding P to e4m3
  inside the kernel is an approximation whose size the tests measure with
  ``attention_fp8_rounded_p``.

Pinned by ``tests/test_oracle_fp8.py``: the e4m3 codec against torch's
float8_e4m3fn conversion and hand-decoded codes, the butterfly against
scipy's Hadamard matrix, H H = d I, exact reconstruction of inputs that lie
on the e4m3 grid, and the error reduction on inputs with outliers.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_fwd

__all__ = [
    "E4M3_MAX",
    "e4m3_encode",
    "e4m3_decode",
    "hadamard_rotate_f32",
    "quantize_blocks",
    "fp8_prepare",
    "fp8_dequantize",
    "attention_fp8",
    "attention_fp8_rounded_p",
]

E4M3_MAX = 448.0
_BLOCK = 128


def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 code (uint8) as float64.

    Bit 7 sign, bits 6..3 exponent field E, bits 2..0 mantissa field M.
    E = 0: subnormal M * 2^-9. Otherwise (1 + M/8) * 2^(E-7), except
    E = 15 with M = 7, which is NaN (the format has no infinities).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x) -> np.ndarray:
    """Round float32 values to e4m3 codes: nearest, ties to even, magnitudes
    above 448 saturate to 448, NaN gives 0x7F; the sign of zero is kept.
    """
    x = np.asarray(x, dtype=np.float32)
    a = np.abs(x.astype(np.float64))
    out = np.zeros(x.shape, dtype=np.uint8)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    # exponent of the binade (normals from 2^-6 up); below, the subnormal step
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)
    step = np.exp2(e - 3)  # spacing of the e4m3 values in the binade
    q = np.round(a / step) * step  # np.round rounds half to even
    q = np.minimum(q, E4M3_MAX)
    # encode the (now exactly representable) magnitude
    is_sub = q < 2.0 ** -6
    m_sub = np.round(q / 2.0 ** -9).astype(np.int64)
    with np.errstate(divide="ignore"):
        eq = np.floor(np.log2(np.where(q > 0, q, 1.0))).astype(np.int64)
    m_norm = np.round((q / np.exp2(eq) - 1.0) * 8).astype(np.int64)
    code = np.where(is_sub, m_sub, ((eq + 7) << 3) | m_norm)
    code = code | np.where(np.signbit(x), 0x80, 0)
    code = np.where(nan, 0x7F, code)
    out[...] = code.astype(np.uint8)
    return out


def hadamard_rotate_f32(x, signs) -> np.ndarray:
    """(x * sign(signs)) H_d in float32 by butterflies, strides 1, 2, ..., d/2.

    x [..., d] (any float type, converted to float32), signs [d]. Returns
    float32 [..., d], equal to the fp64 product up to fp32 rounding.
    """
    y = np.asarray(x, dtype=np.float32).copy()
    d = y.shape[-1]
    if d & (d - 1):
        raise ValueError("d must be a power of two")
    neg = np.signbit(np.asarray(signs, dtype=np.float32))
    y = np.where(neg, -y, y).astype(np.float32)
    h = 1
    while h < d:
        idx = np.arange(d)
        lo = idx[(idx & h) == 0]
        a = y[..., lo].copy()
        b = y[..., lo + h].copy()
        y[..., lo] = a + b
        y[..., lo + h] = a - b
        h *= 2
    return y


def quantize_blocks(x, block: int = _BLOCK):
    """Block-scaled e4m3 codes of x [heads, N, d] (float32 values).

    Each run of ``block`` rows of a head (the last may be shorter) gets
    scale = fp32(max|x|) / fp32(448) (1 when the block is zero) and codes
    e4m3(fp32(x / scale)). Returns (codes uint8 [heads, N, d], scales fp32
    [heads, ceil(N / block)]).
    """
    x = np.asarray(x, dtype=np.float32)
    nh, n, _ = x.shape
    nb = -(-n // block)
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty((nh, nb), dtype=np.float32)
    for h in range(nh):
        for b in range(nb):
            blk = x[h, b * block:(b + 1) * block]
            amax = np.float32(np.max(np.abs(blk)))
            s = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
            scales[h, b] = s
            codes[h, b * block:(b + 1) * block] = e4m3_encode(blk / s)
    return codes, scales


def fp8_prepare(q, k, v, signs=None):
    """The prepared FP8 operands of one forward call.

    q, k, v [B, H, N, d] (the bf16 values, as float32 or float64); signs
    [d] or None (None: no rotation). Rotated (or not) Q and K are
    block-quantised; V gets one scale per head. Q's block scales carry the
    1/d of the unnormalised Hadamard (exact for d a power of two), so
    dequantised Q K^T equals Q K^T up to rounding. Returns a dict with
    q8, k8, v8 (uint8 [B, H, N, d]), q_scale, k_scale (fp32 [B, H, nblk]),
    v_amax (fp32 [B, H]).
    """
    q = np.asarray(q, dtype=np.float32)
    k = np.asarray(k, dtype=np.float32)
    v = np.asarray(v, dtype=np.float32)
    B, H, N, d = q.shape
    if signs is not None:
        q = hadamard_rotate_f32(q, signs)
        k = hadamard_rotate_f32(k, signs)
    q8, qs = quantize_blocks(q.reshape(B * H, N, d))
    k8, ks = quantize_blocks(k.reshape(B * H, N, d))
    if signs is not None:
        qs = (qs * np.float32(1.0 / d)).astype(np.float32)  # exact: d = 2^k
    vf = v.reshape(B * H, N, d)
    v_amax = np.max(np.abs(vf), axis=(1, 2)).astype(np.float32)
    sv = np.where(v_amax > 0, v_amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    v8 = np.empty(vf.shape, dtype=np.uint8)
    for h in range(B * H):
        v8[h] = e4m3_encode(vf[h] / sv[h])
    nb = qs.shape[1]
    return {
        "q8": q8.reshape(B, H, N, d), "k8": k8.reshape(B, H, N, d), "v8": v8.reshape(B, H, N, d),
        "q_scale": qs.reshape(B, H, nb), "k_scale": ks.reshape(B, H, nb),
        "v_amax": v_amax.reshape(B, H),
    }


def fp8_dequantize(prep):
    """float64 (Q^, K^, V^) that the prepared codes stand for."""
    q8, k8, v8 = prep["q8"], prep["k8"], prep["v8"]
    n = q8.shape[2]
    rows = np.arange(n) // _BLOCK

    def blocks(codes, scales):
        return e4m3_decode(codes) * scales.astype(np.float64)[:, :, rows][..., None]

    va = prep["v_amax"].astype(np.float32)
    sv = np.where(va > 0, va / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float64)
    return (blocks(q8, prep["q_scale"]), blocks(k8, prep["k_scale"]),
            e4m3_decode(v8) * sv[:, :, None, None])


def attention_fp8(prep, scale: float, causal: bool):
    """Exact attention (float64) of the dequantised operands: (O, LSE)."""
    qd, kd, vd = fp8_dequantize(prep)
    return attention_fwd(qd, kd, vd, scale, causal)


def attention_fp8_rounded_p(prep, scale: float, causal: bool):
    """As ``attention_fp8`` but with P~ = exp(S - rowmax) rounded to e4m3
    before the product with V (the row sum keeps the unrounded values): the
    size of the deviation that rounding P to FP8 alone causes."""
    qd, kd, vd = fp8_dequantize(prep)
    B, H, N, d = qd.shape
    o = np.empty((B, H, N, vd.shape[-1]))
    for b in range(B):
        for h in range(H):
            s = scale * (qd[b, h] @ kd[b, h].T)
            if causal:
                s = np.where(np.arange(N)[None, :] <= np.arange(N)[:, None], s, -np.inf)
            m = np.max(s, axis=1, keepdims=True)
            p = np.exp(s - m)
            l = np.sum(p, axis=1, keepdims=True)
            pq = e4m3_decode(e4m3_encode(p.astype(np.float32)))
            o[b, h] = (pq @ vd[b, h]) / l
    return o
