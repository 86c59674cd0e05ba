"""CPU oracle for attention with an additive bias and dropout on P.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this
module: only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` use it. It shares no code with the CUDA library.

What it follows:

* "FlashAttention'i Anlamak Bolum 1", section 0.2 Notasyon:
  S = Q K^T / sqrt(d) + B with B an optional mask or bias, P = softmax_row(S),
  O = P V.
* "Bellek Duvarinin Fizigi", section "Maskeleme ve Dropout": dropout acts on
  P; the kernel cannot store the mask, so it drives a counter-based random
  generator (Philox on CUDA) from a seed and a sequence offset and the
  backward regenerates the same mask from the same pair; the causal mask
  (-inf) goes in before the row maximum.
* "Geri Yayilim" of the same page for the backward (P = exp(S - L),
  D = rowsum(dO * O), dS = P * (dP - D)), with dropout's mask applied to
  P in dV and to dP.

Readings taken where the pages stop (listed with the design notes):

* the generator is Philox4x32-10 (Salmon, Moraes, Dror and Shaw, "Parallel
  random numbers: as easy as 1, 2, 3", SC 2011): 10 rounds on a 4 x 32-bit
  counter with a 2 x 32-bit key; per round (c0, c1, c2, c3) ->
  (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2), hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)) with
  M0 = 0xD2511F53, M1 = 0xCD9E8D57, and the key bumped by the Weyl
  constants W0 = 0x9E3779B9, W1 = 0xBB67AE85 between rounds;
* one call covers 16 consecutive keys of one query row: counter =
  (j // 16, i, b * H + h, offset), key = (seed mod 2^32, seed >> 32); the
  byte of pair (i, j) is byte (j % 16) % 4 (least significant first) of
  output word (j % 16) // 4;
* keep iff that byte < t with t = round(256 (1 - p)) (1 <= t <= 256), and
  a kept P is scaled by 256 / t, so the expected P is unchanged;
* the bias is read as bias[b, h, i, j] with broadcasting over b and h
  allowed, and is an input only (no gradient for it);
* the LSE is that of the undropped softmax, O = (P * keep * 256/t) V, and
  D = rowsum(dO * O) with that O.

Pins (``tests/test_oracle_dropout_bias.py``): the generator against the
known-answer vectors its authors publish with the Random123 library
(``tests/golden/philox4x32_10_kat.json``: zero, all-ones and pi-digit
counter/key pairs, every output word bit for bit); the Weyl constants
against their closed forms (golden ratio and sqrt(3)); byte uniformity and
the keep fraction within binomial bounds; independence of the mask from the
seed and offset; p = 0 giving plain attention; a bias of -inf above the
diagonal giving causal attention; a bias equal to scale * Q' K'^T giving
the attention of the concatenated [Q, Q'] and [K, K']; a per-row constant
bias leaving O unchanged and shifting the LSE; the mean of O over many
seeds approaching the undropped O; and the backward against central finite
differences of the forward at a fixed mask. The CUDA side is compared with
this generator bit for bit through the dropout mask.
"""
from __future__ import annotations

import numpy as np

from .attention import softmax_rows

__all__ = [
    "PHILOX_M0",
    "PHILOX_M1",
    "PHILOX_W0",
    "PHILOX_W1",
    "philox4x32_10",
    "keep_threshold",
    "dropout_keep",
    "attention_fwd_ex",
    "attention_bwd_ex",
]

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
_MASK32 = np.uint64(0xFFFFFFFF)


def philox4x32_10(c0, c1, c2, c3, k0: int, k1: int):
    """Philox4x32-10 of counters (arrays of uint32-valued ints, broadcast
    together) under the key (k0, k1). Returns four uint32 arrays."""
    c = [np.asarray(x, dtype=np.uint64) & _MASK32 for x in (c0, c1, c2, c3)]
    c = np.broadcast_arrays(*c)
    c0, c1, c2, c3 = (x.copy() for x in c)
    k0 = np.uint64(k0 & 0xFFFFFFFF)
    k1 = np.uint64(k1 & 0xFFFFFFFF)
    m0, m1 = np.uint64(PHILOX_M0), np.uint64(PHILOX_M1)
    for r in range(10):
        p0 = m0 * c0  # < 2^64: exact in uint64
        p1 = m1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & _MASK32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _MASK32
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
        if r < 9:
            k0 = (k0 + np.uint64(PHILOX_W0)) & _MASK32
            k1 = (k1 + np.uint64(PHILOX_W1)) & _MASK32
    return tuple(x.astype(np.uint32) for x in (c0, c1, c2, c3))


def keep_threshold(p_drop: float) -> int:
    """t = round(256 (1 - p)), clamped to [1, 256]: a byte b keeps iff b < t."""
    if not (0.0 <= p_drop < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    return int(min(256, max(1, round(256.0 * (1.0 - p_drop)))))


def dropout_keep(B: int, H: int, N: int, seed: int, offset: int, p_drop: float):
    """Boolean keep mask [B, H, N (query), N (key)] and the scale 256 / t."""
    t = keep_threshold(p_drop)
    nb = -(-N // 16)
    jb = np.arange(nb)[None, :]
    rows = np.arange(N)[:, None]
    keep = np.empty((B, H, N, nb * 16), dtype=bool)
    for b in range(B):
        for h in range(H):
            w = philox4x32_10(jb, rows, b * H + h, offset, seed & 0xFFFFFFFF, seed >> 32)
            # bytes[i, jb, word, byte] -> pair (i, 16 jb + 4 word + byte)
            words = np.stack(w, axis=-1)                       # [N, nb, 4]
            by = (words[..., None] >> (8 * np.arange(4, dtype=np.uint32))) & 0xFF
            keep[b, h] = (by < t).reshape(N, nb * 16)
    return keep[:, :, :, :N], 256.0 / t


def _scores_ex(q, k, scale, causal, bias):
    s = scale * (q @ k.T)
    if bias is not None:
        s = s + bias
    if causal:
        n = q.shape[0]
        s = np.where(np.arange(n)[None, :] <= np.arange(n)[:, None], s, -np.inf)
    return s


def _head_bias(bias, b, h):
    if bias is None:
        return None
    bb = bias[b if bias.shape[0] > 1 else 0]
    return np.asarray(bb[h if bb.shape[0] > 1 else 0], dtype=np.float64)


def attention_fwd_ex(q, k, v, scale: float, causal: bool, bias=None, keep=None,
                     keep_scale: float = 1.0):
    """O, LSE of softmax(scale Q K^T + bias [causal]) with dropout on P.

    q, k, v [B, H, N, d]; bias broadcastable [B or 1, H or 1, N, N] or None;
    keep [B, H, N, N] bool or None (no dropout). LSE is that of the
    undropped softmax; O = (P * keep * keep_scale) V.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    B, H, N, _ = q.shape
    o = np.empty(q.shape[:3] + (v.shape[-1],))
    lse = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            p, lse[b, h] = softmax_rows(_scores_ex(q[b, h], k[b, h], scale, causal,
                                                   _head_bias(bias, b, h)))
            if keep is not None:
                p = p * keep[b, h] * keep_scale
            o[b, h] = p @ v[b, h]
    return o, lse


def attention_bwd_ex(q, k, v, do, scale: float, causal: bool, bias=None, keep=None,
                     keep_scale: float = 1.0):
    """dQ, dK, dV of sum(O * dO) for ``attention_fwd_ex`` (the bias and the
    mask are constants). With Z = keep * keep_scale: dV = (P Z)^T dO,
    dP = (dO V^T) Z, D = rowsum(dO * O), dS = P (dP - D), dQ = scale dS K,
    dK = scale dS^T Q."""
    q, k, v, do = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
    B, H, _, _ = q.shape
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    for b in range(B):
        for h in range(H):
            p, _ = softmax_rows(_scores_ex(q[b, h], k[b, h], scale, causal,
                                           _head_bias(bias, b, h)))
            z = keep[b, h] * keep_scale if keep is not None else 1.0
            pz = p * z
            o = pz @ v[b, h]
            dv[b, h] = pz.T @ do[b, h]
            dp = (do[b, h] @ v[b, h].T) * z
            dsum = np.sum(do[b, h] * o, axis=1)
            ds = p * (dp - dsum[:, None])
            dq[b, h] = scale * (ds @ k[b, h])
            dk[b, h] = scale * (ds.T @ q[b, h])
    return dq, dk, dv
