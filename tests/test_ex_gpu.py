"""Bias and dropout (fa_fwd_ex / fa_bwd_ex) on the GPU against the oracle.

* the dropout mask is compared bit for bit: with V = identity rows the
  output row is the dropped P row itself, so its zeros are exactly the
  dropped pairs (a kept P is > 0 here);
* O within 1e-2 + 2^-8 |O_ref| and LSE within 1e-3 of the oracle's
  ``attention_fwd_ex`` with the oracle's own mask (a kept P is scaled by
  256/t, so |O| reaches ~3 in early causal rows, where the bf16 rounding
  of P and O, each up to the unit roundoff 2^-8 relative, exceeds a flat
  1e-2); the gradients
  within the backward's relative Frobenius tolerance of
  ``attention_bwd_ex``;
* biases broadcast over batch and head, rows of 16-byte and 2-byte loads
  (N a multiple of 8 or not), causal and not, d = 64 and 128.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
import oracle
from gpu_helpers import TOL_GRAD_REL, TOL_LSE, TOL_O, Guarded, bf16_device, f64, max_abs, rel_fro

pytestmark = pytest.mark.gpu


def _bias_bits(seed, shape, std=1.0):
    rng = np.random.default_rng(seed)
    return inputgen.bf16_round_bits((rng.standard_normal(shape) * std).astype(np.float32))


def _run_fwd(x, causal, bias_bits=None, p_drop=0.0, seed=0, offset=0):
    B, H, N, d = x["q"].shape
    q, k, v = (bf16_device(x[n]) for n in ("q", "k", "v"))
    bias = bf16_device(bias_bits) if bias_bits is not None else None
    o = Guarded((B, H, N, d), torch.bfloat16)
    lse = Guarded((B, H, N), torch.float32)
    fa.fa_fwd_ex(q, k, v, causal=causal, bias=bias, p_drop=p_drop, seed=seed, offset=offset,
                 o=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.guards_intact() and lse.guards_intact()
    assert fa.fa_device_status()[0] == 0
    return o.t, lse.t


def test_dropout_mask_bit_exact():
    """V = identity rows, key tile by key tile: O's zeros are the dropped pairs."""
    B, H, N, d = 1, 2, 300, 128
    seed, offset, p_drop = 0x1234_5678_9ABC, 5, 0.3
    x = inputgen.make_small_inputs(61, B, H, N, d)
    x["q"] = inputgen.bf16_round_bits(inputgen.bf16_bits_to_f32(x["q"]) * np.float32(0.1))
    keep, _ = oracle.dropout_keep(B, H, N, seed, offset, p_drop)
    for t0 in range(0, N, 128):
        vv = np.zeros((B, H, N, d), dtype=np.float32)
        n = min(128, N - t0)
        vv[:, :, t0 + np.arange(n), np.arange(n)] = 1.0
        x["v"] = inputgen.bf16_round_bits(vv)
        for causal in (False, True):
            o, _ = _run_fwd(x, causal, p_drop=p_drop, seed=seed, offset=offset)
            got = o.float().cpu().numpy()[..., :n] != 0
            want = keep[..., t0:t0 + n].copy()
            if causal:
                want &= (np.arange(t0, t0 + n)[None, :] <= np.arange(N)[:, None])
            assert np.array_equal(got, want), (t0, causal, int((got != want).sum()))


CASES = [((1, 2, 256, 128), "full"), ((2, 2, 200, 64), "batch"), ((1, 1, 77, 128), "head"),
         ((1, 2, 640, 128), "both"), ((2, 1, 130, 64), "full")]


@pytest.mark.parametrize("p_drop", [0.0, 0.2], ids=["nodrop", "drop"])
@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[0])) + "-" + c[1])
def test_fwd_bwd_ex(case, causal, p_drop):
    (B, H, N, d), bcast = case
    x = inputgen.make_small_inputs(90 + N + d, B, H, N, d, with_grad=True)
    bshape = {"full": (B, H, N, N), "batch": (1, H, N, N), "head": (B, 1, N, N),
              "both": (1, 1, N, N)}[bcast]
    bb = _bias_bits(7 + N, bshape, 1.5)
    seed, offset = 987654321 + N, 11
    scale = 1 / math.sqrt(d)
    o, lse = _run_fwd(x, causal, bb, p_drop, seed, offset)
    keep, ks = oracle.dropout_keep(B, H, N, seed, offset, p_drop) if p_drop else (None, 1.0)
    args = (f64(x["q"]), f64(x["k"]), f64(x["v"]))
    ro, rl = oracle.attention_fwd_ex(*args, scale, causal, bias=f64(bb), keep=keep, keep_scale=ks)
    og = o.float().cpu().numpy().astype(np.float64)
    assert np.all(np.abs(og - ro) <= TOL_O + 2.0 ** -8 * np.abs(ro))
    assert max_abs(lse, rl) <= TOL_LSE
    # backward with the GPU's own O and LSE
    q, k, v, do = (bf16_device(x[n]) for n in ("q", "k", "v", "do"))
    dq, dk, dv = fa.fa_bwd_ex(q, k, v, o, lse, do, causal=causal, bias=bf16_device(bb),
                              p_drop=p_drop, seed=seed, offset=offset)
    torch.cuda.synchronize()
    assert fa.fa_device_status()[0] == 0
    ref = oracle.attention_bwd_ex(*args, f64(x["do"]), scale, causal, bias=f64(bb), keep=keep,
                                  keep_scale=ks)
    for g, r in zip((dq, dk, dv), ref):
        assert rel_fro(g, r) <= TOL_GRAD_REL


def test_ex_without_options_matches_plain():
    """fa_fwd_ex / fa_bwd_ex with no bias and p = 0 run the plain kernels:
    bitwise equal to fa_fwd / fa_bwd."""
    x = inputgen.make_small_inputs(77, 1, 2, 384, 128, with_grad=True)
    q, k, v, do = (bf16_device(x[n]) for n in ("q", "k", "v", "do"))
    o1, l1 = fa.fa_fwd(q, k, v, causal=True)
    o2, l2 = fa.fa_fwd_ex(q, k, v, causal=True)
    g1 = fa.fa_bwd(q, k, v, o1, l1, do, causal=True)
    g2 = fa.fa_bwd_ex(q, k, v, o2, l2, do, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("mask", ["left_pad", "window"])
def test_bias_as_mask(mask, causal):
    """-inf bias entries hide keys; for a left padding of 200 keys every row's
    first key tile is hidden entirely. Rows keep at least one visible key."""
    B, H, N, d = 1, 2, 520, 128
    x = inputgen.make_small_inputs(401, B, H, N, d, with_grad=True)
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    if mask == "left_pad":
        hide = (j < 200) & (i >= 0)
        if causal:
            hide &= i >= 200  # rows before 200 would have no visible key
    else:
        hide = j < i - 150
    bias = np.where(hide, -np.inf, 0.25 * np.sin(i + 2 * j)).astype(np.float32)[None, None]
    bb = inputgen.bf16_round_bits(np.repeat(bias, H, axis=1))
    o, lse = _run_fwd(x, causal, bb, 0.1, 5, 0)
    keep, ks = oracle.dropout_keep(B, H, N, 5, 0, 0.1)
    args = (f64(x["q"]), f64(x["k"]), f64(x["v"]))
    ro, rl = oracle.attention_fwd_ex(*args, 1 / math.sqrt(d), causal, bias=f64(bb), keep=keep,
                                     keep_scale=ks)
    og = o.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(og))
    assert np.all(np.abs(og - ro) <= TOL_O + 2.0 ** -8 * np.abs(ro))
    assert max_abs(lse, rl) <= TOL_LSE
    q, k, v, do = (bf16_device(x[n]) for n in ("q", "k", "v", "do"))
    grads = fa.fa_bwd_ex(q, k, v, o, lse, do, causal=causal, bias=bf16_device(bb), p_drop=0.1,
                         seed=5, offset=0)
    torch.cuda.synchronize()
    ref = oracle.attention_bwd_ex(*args, f64(x["do"]), 1 / math.sqrt(d), causal, bias=f64(bb),
                                  keep=keep, keep_scale=ks)
    for g, r in zip(grads, ref):
        assert rel_fro(g, r) <= TOL_GRAD_REL


def test_dropout_extreme_keep_threshold():
    """p = 0.997: t = round(256 * 0.003) = 1, a pair is kept iff its byte is 0
    (1 in 256) and scaled by 256. A row of O is then a sum of a few large
    terms (often one), so the error is bounded by the roundings of P and of
    O to bf16 (unit roundoff 2^-8 each): 2^-7 (P Z)|V|, not a multiple of |O|
    alone."""
    B, H, N, d = 1, 1, 384, 64
    x = inputgen.make_small_inputs(402, B, H, N, d, with_grad=True)
    o, lse = _run_fwd(x, False, None, 0.997, 77, 3)
    keep, ks = oracle.dropout_keep(B, H, N, 77, 3, 0.997)
    assert ks == 256.0
    ro, rl = oracle.attention_fwd_ex(f64(x["q"]), f64(x["k"]), f64(x["v"]), 1 / math.sqrt(d), False,
                                     keep=keep, keep_scale=ks)
    mag, _ = oracle.attention_fwd_ex(f64(x["q"]), f64(x["k"]), np.abs(f64(x["v"])), 1 / math.sqrt(d),
                                     False, keep=keep, keep_scale=ks)
    og = o.float().cpu().numpy().astype(np.float64)
    bad = np.abs(og - ro) - (TOL_O + 2.0 ** -7 * mag)
    w = np.unravel_index(np.argmax(bad), bad.shape)
    assert bad[w] <= 0, (w, og[w], ro[w], mag[w], int((bad > 0).sum()),
                         int(keep[0, 0, w[2]].sum()))
    assert max_abs(lse, rl) <= TOL_LSE
