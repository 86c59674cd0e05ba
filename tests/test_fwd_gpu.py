"""Forward parity on the GPU: fa_fwd / fa_fwd_f32 against the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation): max |O - O_ref| <= 1e-2 and
max |LSE - LSE_ref| <= 1e-3, compared element by element. Inputs carry NaN
past their logical end and outputs carry NaN guard bands, so an
out-of-bounds read or write shows up as a failure.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
import oracle
from gpu_helpers import (TOL_LSE, TOL_O, Guarded, bf16_device, f32_device, f64,
                         max_abs)

pytestmark = pytest.mark.gpu

SMALL = [
    (1, 2, 128, 64), (2, 2, 256, 128), (1, 3, 384, 128), (1, 2, 130, 64),
    (1, 2, 1000, 128), (1, 1, 1, 128), (2, 1, 200, 64), (1, 1, 640, 128),
    (1, 2, 513, 64), (3, 1, 255, 128),
]


def run_fwd(x, causal, scale=None):
    B, H, N, d = x["q"].shape
    q, k, v = (bf16_device(x[n]) for n in ("q", "k", "v"))
    o = Guarded((B, H, N, d), torch.bfloat16)
    lse = Guarded((B, H, N), torch.float32)
    fa.fa_fwd(q, k, v, causal=causal, scale=scale, o=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.guards_intact() and lse.guards_intact()
    return o.t, lse.t


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", SMALL, ids=lambda s: "x".join(map(str, s)))
def test_fwd_small(shape, causal):
    B, H, N, d = shape
    x = inputgen.make_small_inputs(1000 + N + d, B, H, N, d)
    o, lse = run_fwd(x, causal)
    ref_o, ref_l = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]),
                                        1 / math.sqrt(d), causal)
    assert max_abs(o, ref_o) <= TOL_O
    assert max_abs(lse, ref_l) <= TOL_LSE


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_fwd_prefill_workload_every_head(causal):
    """B=4, H=16, N=2048, d=128, compared in full for every head."""
    w = inputgen.WORKLOADS["prefill"]
    x = inputgen.make_attention_inputs(w)
    o, lse = run_fwd(x, causal)
    ref_o, ref_l = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]),
                                        w.scale, causal)
    assert max_abs(o, ref_o) <= TOL_O
    assert max_abs(lse, ref_l) <= TOL_LSE


def test_fwd_long_causal_sampled_row_blocks():
    """B=1, H=32, N=16384 causal; oracle on 64 seeded (b, h, row-block)s."""
    w = inputgen.WORKLOADS["long_causal"]
    x = inputgen.make_attention_inputs(w)
    o, lse = run_fwd(x, True)
    o_np = o.float().cpu().numpy()
    l_np = lse.cpu().numpy()
    for b, h, blk in inputgen.sample_row_blocks(w, 64):
        r0, r1 = blk * 128, min((blk + 1) * 128, w.N)
        ro, rl = oracle.attention_fwd_rows(f64(x["q"][b, h]), f64(x["k"][b, h]),
                                           f64(x["v"][b, h]), w.scale, True, r0, r1)
        assert np.max(np.abs(o_np[b, h, r0:r1] - ro)) <= TOL_O, (b, h, blk)
        assert np.max(np.abs(l_np[b, h, r0:r1] - rl)) <= TOL_LSE, (b, h, blk)
    assert np.all(np.isfinite(o_np)) and np.all(np.isfinite(l_np))


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", [(1, 25, 2048, 128), (1, 40, 2048, 64), (2, 3, 1500, 128)],
                         ids=lambda s: "x".join(map(str, s)))
def test_fwd_partial_last_round(shape, causal):
    """More work units (one per 128-row query tile and head) than SMs, with
    the last round of the persistent CTAs partly filled: H=25 gives 400
    units on 148 SMs, H=40 at d=64 gives 640, and B=2, H=3, N=1500 (a
    ragged last tile) gives 72 units, fewer than the SMs. Every row of the
    last heads (whose units fall in the last rounds) is compared, plus the
    first and last row blocks of every other head."""
    B, H, N, d = shape
    x = inputgen.make_small_inputs(77 + H + (1000 if causal else 0), B, H, N, d)
    o, lse = run_fwd(x, causal)
    o_np, l_np = o.float().cpu().numpy(), lse.cpu().numpy()
    nblk = (N + 127) // 128
    blocks = [(b, h, blk) for b in range(B) for h in range(H)
              for blk in (range(nblk) if (b == B - 1 and h >= H - 2) else (0, nblk - 1))]
    for b, h, blk in blocks:
        r0, r1 = blk * 128, min((blk + 1) * 128, N)
        ro, rl = oracle.attention_fwd_rows(f64(x["q"][b, h]), f64(x["k"][b, h]), f64(x["v"][b, h]),
                                           1 / math.sqrt(d), causal, r0, r1)
        assert np.max(np.abs(o_np[b, h, r0:r1] - ro)) <= TOL_O, (b, h, blk)
        assert np.max(np.abs(l_np[b, h, r0:r1] - rl)) <= TOL_LSE, (b, h, blk)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", [(4, 40, 384, 128), (2, 75, 260, 64), (3, 70, 200, 128)],
                         ids=lambda s: "x".join(map(str, s)))
def test_fwd_many_short_units_per_cta(shape, causal):
    """Hundreds of heads of one to three Q tiles: every CTA of the
    persistent grid runs several units back to back, of every length from
    one to three K/V steps in turn (under the mask), so every hand-over
    between consecutive units (the epilogue of one, the first steps of the
    next) occurs many times per CTA.

    These shapes are outside the stated workloads: under the mask the first
    rows average a few keys, so |O| reaches 2-3, where the bf16 rounding of
    P and of O (each up to the unit roundoff 2^-8 relative) can alone come
    close to 1e-2; the bound is 1e-2 + 2^-8 |O_ref| element-wise, as for the
    non-default scale."""
    B, H, N, d = shape
    x = inputgen.make_small_inputs(4242 + H + N + (1000 if causal else 0), B, H, N, d)
    o, lse = run_fwd(x, causal)
    ref_o, ref_l = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), 1 / np.sqrt(d), causal)
    err = np.abs(o.float().cpu().numpy() - ref_o)
    assert np.all(err <= TOL_O + 2.0 ** -8 * np.abs(ref_o))
    assert max_abs(lse, ref_l) <= TOL_LSE


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_fwd_tiny_f32_workload(causal):
    """B=1, H=1, N=128, d=64, fp32 Q/K/V in, fp32 O out."""
    w = inputgen.WORKLOADS["tiny_f32"]
    x = inputgen.make_attention_inputs(w)
    q, k, v = (f32_device(x[n]) for n in ("q", "k", "v"))
    o = Guarded((w.B, w.H, w.N, w.d), torch.float32)
    lse = Guarded((w.B, w.H, w.N), torch.float32)
    fa.fa_fwd_f32(q, k, v, causal=causal, o=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.guards_intact() and lse.guards_intact()
    ref_o, ref_l = oracle.attention_fwd(x["q"].astype(np.float64), x["k"].astype(np.float64),
                                        x["v"].astype(np.float64), w.scale, causal)
    assert max_abs(o.t, ref_o) <= TOL_O
    assert max_abs(lse.t, ref_l) <= TOL_LSE
    # fp32 arithmetic end to end: far inside the bf16 tolerances
    assert max_abs(o.t, ref_o) <= 1e-4
    assert max_abs(lse.t, ref_l) <= 1e-4


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [100, 333])
def test_fwd_f32_other_shapes(N, d):
    rng = np.random.default_rng(N * d)
    x = {n: rng.standard_normal((2, 2, N, d), dtype=np.float32) for n in "qkv"}
    for causal in (False, True):
        o, lse = fa.fa_fwd_f32(*(f32_device(x[n]) for n in "qkv"), causal=causal)
        ref_o, ref_l = oracle.attention_fwd(*(x[n].astype(np.float64) for n in "qkv"),
                                            1 / math.sqrt(d), causal)
        assert max_abs(o, ref_o) <= 1e-4 and max_abs(lse, ref_l) <= 1e-4


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_fwd_tiny_tf32_workload(causal):
    """The fp32 workload (B=1, H=1, N=128, d=64) through fa_fwd_tf32, the
    TF32 tensor-core variant: within the bf16 forward's bars (O 1e-2, LSE
    1e-3), and, its inputs being rounded to nearest, within 2e-3 / 1e-3
    where truncation would bias the LSE by ~1e-3."""
    w = inputgen.WORKLOADS["tiny_f32"]
    x = inputgen.make_attention_inputs(w)
    q, k, v = (f32_device(x[n]) for n in ("q", "k", "v"))
    o = Guarded((w.B, w.H, w.N, w.d), torch.float32)
    lse = Guarded((w.B, w.H, w.N), torch.float32)
    fa.fa_fwd_tf32(q, k, v, causal=causal, o=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.guards_intact() and lse.guards_intact()
    ref_o, ref_l = oracle.attention_fwd(x["q"].astype(np.float64), x["k"].astype(np.float64),
                                        x["v"].astype(np.float64), w.scale, causal)
    assert max_abs(o.t, ref_o) <= 2e-3
    assert max_abs(lse.t, ref_l) <= TOL_LSE


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 63, 100, 333, 1000])
def test_fwd_tf32_other_shapes(N, d):
    """Ragged lengths over one and several 64-key and 128-row tiles, both
    head dims, both masks: O within 1e-2 and LSE within 1e-3 of the oracle,
    and the two masks agree on the last row (which sees every key)."""
    rng = np.random.default_rng(N * d + 5)
    x = {n: rng.standard_normal((2, 2, N, d), dtype=np.float32) for n in "qkv"}
    outs = {}
    for causal in (False, True):
        o, lse = fa.fa_fwd_tf32(*(f32_device(x[n]) for n in "qkv"), causal=causal)
        torch.cuda.synchronize()
        ref_o, ref_l = oracle.attention_fwd(*(x[n].astype(np.float64) for n in "qkv"),
                                            1 / math.sqrt(d), causal)
        assert max_abs(o, ref_o) <= TOL_O and max_abs(lse, ref_l) <= TOL_LSE
        outs[causal] = (o, lse)
    assert torch.equal(outs[False][0][:, :, -1], outs[True][0][:, :, -1])


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_growing_scores_rescale_path(d):
    """Keys grow along the sequence so the running maximum keeps rising by
    far more than the lazy-rescale threshold: exercises the O~ rescale."""
    B, H, N = 1, 2, 1024
    rng = np.random.default_rng(77)
    q = rng.standard_normal((B, H, N, d), dtype=np.float32) * 0.2 + 1.0
    growth = np.linspace(0.0, 6.0, N, dtype=np.float32)[None, None, :, None]
    k = rng.standard_normal((B, H, N, d), dtype=np.float32) * 0.2 + growth
    v = rng.standard_normal((B, H, N, d), dtype=np.float32)
    x = {"q": inputgen.bf16_round_bits(q), "k": inputgen.bf16_round_bits(k),
         "v": inputgen.bf16_round_bits(v)}
    for causal in (False, True):
        o, lse = run_fwd(x, causal, scale=1.0 / math.sqrt(d))
        ref_o, ref_l = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]),
                                            1 / math.sqrt(d), causal)
        assert max_abs(o, ref_o) <= TOL_O
        assert max_abs(lse, ref_l) <= TOL_LSE


def test_fwd_deterministic():
    x = inputgen.make_small_inputs(5, 2, 4, 1000, 128)
    for causal in (False, True):
        o1, l1 = run_fwd(x, causal)
        o2, l2 = run_fwd(x, causal)
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
        assert torch.equal(l1, l2)


def test_fwd_nondefault_scale_and_stream():
    """scale = 0.3 (2.4x the default): peakier rows, |O| up to ~3.5.

    Outside the stated workloads the O tolerance is derived from the
    arithmetic: P enters the PV product rounded to bf16 and O is stored in
    bf16, each with relative error at most the unit roundoff 2^-8 (8
    significant bits, round to nearest even). The bound used is
    1e-2 + 2^-8 |O_ref| element-wise: the two roundings of one element
    rarely align, and the 1e-2 base covers the remainder.
    """
    x = inputgen.make_small_inputs(9, 1, 2, 300, 64)
    s = torch.cuda.Stream()
    q, k, v = (bf16_device(x[n]) for n in ("q", "k", "v"))
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        o, lse = fa.fa_fwd(q, k, v, causal=True, scale=0.3)
    s.synchronize()
    ref_o, ref_l = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), 0.3, True)
    err = np.abs(o.float().cpu().numpy() - ref_o)
    assert np.all(err <= TOL_O + 2.0 ** -8 * np.abs(ref_o))
    assert max_abs(lse, ref_l) <= TOL_LSE
