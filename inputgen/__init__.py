"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module holds no attention arithmetic. It only draws iid N(0,1) values
with a fixed seed, rounds them to bf16 with round-to-nearest-even, and knows
the shapes of the five workloads. Both the fp64 oracle and the GPU path read
the *same* bf16 bit patterns from here, so any difference between them comes
from the attention computation alone.

Workloads (sizes, dtypes, masks) follow the problem statement of the build;
the values are synthetic because the pages measure on no dataset.

Recipe
------
* workload ``k`` (0..4) draws from ``numpy.random.default_rng(20260 + k)``;
* draws are float32 standard normals, taken in the order Q, K, V, dO;
* the split-KV decode workload first draws its per-sequence cache lengths
  with ``rng.integers(16384, 32769, size=B)``, then q; the K (V) cache rows
  of sequence b come from their own generator,
  ``default_rng(SeedSequence([seed, 1 (2 for V), b]))``, drawn head by
  head as [seqlen[b], d] blocks, so sequences can be drawn in parallel; cache
  positions at or past ``seqlen[b]`` are filled with NaN so that a kernel
  that reads past the logical end poisons its own result;
* the paged, grouped-query decode inputs (``make_paged_decode_inputs``)
  draw q from ``default_rng(seed)`` after the lengths (as above), the K (V)
  rows of sequence b and KV head h from
  ``default_rng(SeedSequence([seed, 1 (2 for V), b]))`` as [seqlen[b], d]
  blocks head by head, and scatter them into pages whose order is a seeded
  permutation (``default_rng(seed + 7)``); rows past a sequence's end, and
  pages no sequence uses, hold NaN, and block-table entries past a
  sequence's last page hold -1, so a kernel that reads any of them is caught;
* the FP8 inputs (``make_fp8_inputs``) draw, from ``default_rng(seed)`` in
  this order, the d random signs of the rotation (``rng.choice([-1, 1])``
  as float32), then for each of Q, K, V in turn a float32 N(0,1) array, a
  uniform array that marks a fraction ``outlier_frac`` of the entries, and
  a float32 N(0,1) array whose marked entries, times ``outlier_std``, are
  added (outliers; 0.1% with std 10 in the tests); the sum is rounded to
  bf16;
* bf16 rounding is round-to-nearest-even on the fp32 bit pattern.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "Workload",
    "WORKLOADS",
    "bf16_round_bits",
    "bf16_bits_to_f32",
    "standard_normal_bf16",
    "make_attention_inputs",
    "make_decode_inputs",
    "make_paged_decode_inputs",
    "make_small_inputs",
    "make_fp8_inputs",
    "sample_row_blocks",
]

SEED_BASE = 20260


@dataclass(frozen=True)
class Workload:
    """One workload: shapes, dtype and masks, named by what it is."""

    name: str
    index: int
    B: int
    H: int
    N: int  # sequence length (prefill) or cache capacity Lmax (decode)
    d: int
    dtype: str  # "f32" or "bf16"
    causal: tuple = (False,)
    kind: str = "fwd"  # "fwd", "bwd" or "decode"
    seqlen_range: tuple | None = None
    extra: dict = field(default_factory=dict)

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.d))


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 0, B=1, H=1, N=128, d=64, dtype="f32",
                         causal=(False, True)),
    "prefill": Workload("prefill", 1, B=4, H=16, N=2048, d=128, dtype="bf16",
                        causal=(False, True)),
    "long_causal": Workload("long_causal", 2, B=1, H=32, N=16384, d=128,
                            dtype="bf16", causal=(True,)),
    "backward": Workload("backward", 3, B=2, H=16, N=4096, d=128, dtype="bf16",
                         causal=(True,), kind="bwd"),
    "decode": Workload("decode", 4, B=8, H=32, N=32768, d=128, dtype="bf16",
                       kind="decode", seqlen_range=(16384, 32768)),
}


def bf16_round_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even).

    Returns the 16-bit patterns as uint16. Inputs here are finite normals,
    so no NaN/Inf special-casing is needed; NaN payloads are preserved
    anyway by the quiet-bit OR below.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    rounded = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = ((u[nan] >> np.uint32(16)) | np.uint32(0x40)).astype(np.uint16)
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact float32 value of each bf16 bit pattern."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def standard_normal_bf16(rng: np.random.Generator, shape) -> np.ndarray:
    """Draw float32 N(0,1) values and return their bf16 bit patterns."""
    return bf16_round_bits(rng.standard_normal(shape, dtype=np.float32))


def make_attention_inputs(w: Workload, with_grad: bool = False):
    """Q, K, V (and dO) for a prefill / backward workload.

    Returns a dict. For bf16 workloads the arrays are uint16 bit patterns
    of shape [B, H, N, d]; for the fp32 workload they are float32.
    """
    rng = np.random.default_rng(w.seed)
    shape = (w.B, w.H, w.N, w.d)
    names = ["q", "k", "v"] + (["do"] if with_grad else [])
    out = {}
    for n in names:
        if w.dtype == "f32":
            out[n] = rng.standard_normal(shape, dtype=np.float32)
        else:
            out[n] = standard_normal_bf16(rng, shape)
    return out


def make_decode_inputs(w: Workload, seqlens=None):
    """q [B,H,d], K/V caches [B,H,Lmax,d] (bf16 bits) and seqlens int32 [B].

    Cache entries at or past ``seqlens[b]`` hold bf16 NaN (0x7FC0).
    ``seqlens`` may be given to override the drawn lengths (edge cases);
    the draw still happens so the stream of values is unchanged.
    """
    rng = np.random.default_rng(w.seed)
    lo, hi = w.seqlen_range
    drawn = rng.integers(lo, hi + 1, size=w.B).astype(np.int32)
    lens = drawn if seqlens is None else np.asarray(seqlens, dtype=np.int32)
    q = standard_normal_bf16(rng, (w.B, w.H, w.d))
    kc = np.empty((w.B, w.H, w.N, w.d), dtype=np.uint16)
    vc = np.empty((w.B, w.H, w.N, w.d), dtype=np.uint16)

    def fill(job):
        which, b = job
        cache = kc if which == 1 else vc
        n = int(lens[b])
        g = np.random.default_rng(np.random.SeedSequence([w.seed, which, b]))
        cache[b, :, n:] = 0x7FC0
        for h in range(w.H):  # one head at a time keeps the fp32 draw small
            cache[b, h, :n] = standard_normal_bf16(g, (n, w.d))

    jobs = [(which, b) for which in (1, 2) for b in range(w.B)]
    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        list(ex.map(fill, jobs))
    return {"q": q, "kcache": kc, "vcache": vc, "seqlens": lens}


def make_paged_decode_inputs(seed: int, B: int, Hq: int, Hkv: int, d: int, page: int,
                             seqlen_range=None, seqlens=None, spare_pages: int = 3,
                             max_pages: int | None = None):
    """q [B,Hq,d]; K/V pages [num_pages, Hkv, page, d] (bf16 bits); block table
    int32 [B, max_pages]; seqlens int32 [B]. See the recipe above."""
    rng = np.random.default_rng(seed)
    if seqlens is None:
        lo, hi = seqlen_range
        lens = rng.integers(lo, hi + 1, size=B).astype(np.int32)
    else:
        lens = np.asarray(seqlens, dtype=np.int32)
    q = standard_normal_bf16(rng, (B, Hq, d))
    used = [(int(n) + page - 1) // page for n in lens]
    mp = max(max(used), 1) if max_pages is None else max_pages
    num_pages = sum(used) + spare_pages
    order = np.random.default_rng(seed + 7).permutation(num_pages)
    table = np.full((B, mp), -1, dtype=np.int32)
    kp = np.full((num_pages, Hkv, page, d), 0x7FC0, dtype=np.uint16)
    vp = np.full((num_pages, Hkv, page, d), 0x7FC0, dtype=np.uint16)
    nxt = 0
    for b in range(B):
        n = int(lens[b])
        pages_b = order[nxt:nxt + used[b]]
        nxt += used[b]
        table[b, :used[b]] = pages_b
        for which, dst in ((1, kp), (2, vp)):
            g = np.random.default_rng(np.random.SeedSequence([seed, which, b]))
            for h in range(Hkv):
                rows = standard_normal_bf16(g, (n, d))
                for i, pg in enumerate(pages_b):
                    r0, r1 = i * page, min((i + 1) * page, n)
                    dst[pg, h, :r1 - r0] = rows[r0:r1]
    return {"q": q, "kpages": kp, "vpages": vp, "block_table": table, "seqlens": lens}


def make_small_inputs(seed: int, B: int, H: int, N: int, d: int,
                      with_grad: bool = False, dtype: str = "bf16"):
    """Seeded inputs of any shape, for the small parity cases."""
    rng = np.random.default_rng(seed)
    shape = (B, H, N, d)
    names = ["q", "k", "v"] + (["do"] if with_grad else [])
    out = {}
    for n in names:
        if dtype == "f32":
            out[n] = rng.standard_normal(shape, dtype=np.float32)
        else:
            out[n] = standard_normal_bf16(rng, shape)
    return out


def make_fp8_inputs(seed: int, B: int, H: int, N: int, d: int,
                    outlier_frac: float = 0.0, outlier_std: float = 10.0):
    """Q, K, V (bf16 bit patterns, [B, H, N, d]) with optional outliers, and
    the d random signs of the rotation (float32 +-1)."""
    rng = np.random.default_rng(seed)
    signs = rng.choice(np.array([-1.0, 1.0], dtype=np.float32), size=d)
    shape = (B, H, N, d)
    out = {"signs": signs.astype(np.float32)}
    for n in ("q", "k", "v"):
        x = rng.standard_normal(shape, dtype=np.float32)
        mark = rng.random(shape) < outlier_frac
        extra = rng.standard_normal(shape, dtype=np.float32) * np.float32(outlier_std)
        out[n] = bf16_round_bits(np.where(mark, x + extra, x).astype(np.float32))
    return out


def sample_row_blocks(w: Workload, count: int = 64, block: int = 128,
                      seed_offset: int = 100):
    """Seeded sample of (batch, head, row-block) triples for large workloads.

    Draws from ``default_rng(seed + seed_offset)``; returns a sorted list of
    distinct triples ``(b, h, blk)`` where rows ``blk*block .. +block`` form
    the sampled query block.
    """
    rng = np.random.default_rng(w.seed + seed_offset)
    nblk = (w.N + block - 1) // block
    total = w.B * w.H * nblk
    picks = rng.choice(total, size=min(count, total), replace=False)
    out = []
    for p in sorted(int(x) for x in picks):
        b, rem = divmod(p, w.H * nblk)
        h, blk = divmod(rem, nblk)
        out.append((b, h, blk))
    return out
