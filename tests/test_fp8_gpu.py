"""FP8 forward with incoherent processing on the GPU, against the oracle.

* fa_fp8_prepare: codes, block scales and V amax bit for bit equal to the
  oracle's (both sides take every rounding decision in fp32 the same way).
* fa_fwd_fp8: O against the exact attention of the dequantised operands.
  The kernel rounds P~ to e4m3 before P V (the method's approximation), so
  the bar is the deviation that rounding P alone gives in the oracle
  (``attention_fp8_rounded_p``): RMS within 1.5x of it, largest entry
  within 4x of its largest, each plus the bf16 rounding of the output
  (2^-8 of the reference's RMS, resp. largest magnitude, + 1e-4). The LSE
  has no P rounding in it: max |LSE - LSE_ref| <= 1e-3.
* the page's accuracy claim on the GPU path: with 0.1% outliers the rotation
  lowers the RMS error against the exact bf16 attention.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
import oracle
from gpu_helpers import TOL_LSE, Guarded, bf16_device, f32_device, f64, max_abs

pytestmark = pytest.mark.gpu

D = 128


def _prepare(x, rotate):
    q, k, v = (bf16_device(x[n]) for n in ("q", "k", "v"))
    signs = f32_device(x["signs"]) if rotate else None
    prep = fa.fa_fp8_prepare(q, k, v, signs)
    torch.cuda.synchronize()
    return prep


def _np(t):
    return t.cpu().numpy()


@pytest.mark.parametrize("rotate", [False, True], ids=["plain", "rotated"])
@pytest.mark.parametrize("shape", [(1, 2, 128), (2, 2, 1000), (1, 3, 77), (1, 1, 300)],
                         ids=lambda s: "x".join(map(str, s)))
def test_prepare_bit_exact(shape, rotate):
    B, H, N = shape
    x = inputgen.make_fp8_inputs(700 + N, B, H, N, D, outlier_frac=0.001)
    prep = _prepare(x, rotate)
    ref = oracle.fp8_prepare(inputgen.bf16_bits_to_f32(x["q"]), inputgen.bf16_bits_to_f32(x["k"]),
                             inputgen.bf16_bits_to_f32(x["v"]), x["signs"] if rotate else None)
    for n in ("q8", "k8"):
        assert np.array_equal(_np(prep[n]), ref[n]), n
    for n in ("q_scale", "k_scale", "v_amax"):
        assert np.array_equal(_np(prep[n]), ref[n]), n
    nv = fa.fa_fp8_vt_keys(N)
    vt = _np(prep["vt8"])
    assert vt.shape == (B, H, D, nv)
    assert np.array_equal(vt[..., :N], np.swapaxes(ref["v8"], 2, 3))
    assert not vt[..., N:].any()  # zero codes past N


def _rms(a, b):
    return float(np.sqrt(np.mean((np.asarray(a, dtype=np.float64) - b) ** 2)))


def run_fp8(prep, causal):
    B, H, N, d = prep["q8"].shape
    o = Guarded((B, H, N, d), torch.bfloat16)
    lse = Guarded((B, H, N), torch.float32)
    fa.fa_fwd_fp8(prep, causal=causal, o=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.guards_intact() and lse.guards_intact()
    assert fa.fa_device_status()[0] == 0
    return o.t, lse.t


def _oracle_prep(prep):
    """The oracle's view of the GPU's prepared operands (they are bit-exact
    with the oracle's own preparation, tested above)."""
    N = prep["q8"].shape[2]
    out = {n: _np(prep[n]) for n in ("q8", "k8", "q_scale", "k_scale", "v_amax")}
    out["v8"] = np.ascontiguousarray(np.swapaxes(_np(prep["vt8"])[..., :N], 2, 3))
    return out


def _check_against_oracle(prep, causal, o, lse):
    op = _oracle_prep(prep)
    scale = 1 / math.sqrt(D)
    ro, rl = oracle.attention_fp8(op, scale, causal)
    rp = oracle.attention_fp8_rounded_p(op, scale, causal)
    og = o.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(og))
    rms_p, max_p = _rms(rp, ro), float(np.max(np.abs(rp - ro)))
    rms_g, max_g = _rms(og, ro), float(np.max(np.abs(og - ro)))
    out_rms, out_max = float(np.sqrt(np.mean(ro ** 2))), float(np.max(np.abs(ro)))
    assert rms_g <= 1.5 * rms_p + 2.0 ** -8 * out_rms + 1e-4, (rms_g, rms_p, out_rms)
    assert max_g <= 4 * max_p + 2.0 ** -8 * out_max + 1e-4, (max_g, max_p, out_max)
    assert max_abs(lse, rl) <= TOL_LSE


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", [(1, 2, 128), (2, 2, 1000), (1, 1, 77), (1, 2, 640), (1, 1, 1)],
                         ids=lambda s: "x".join(map(str, s)))
def test_fwd_fp8_small(shape, causal):
    B, H, N = shape
    x = inputgen.make_fp8_inputs(800 + N, B, H, N, D)
    prep = _prepare(x, True)
    o, lse = run_fp8(prep, causal)
    _check_against_oracle(prep, causal, o, lse)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_fwd_fp8_prefill_sampled_heads(causal):
    """The prefill shape (B=4, H=16, N=2048) as bench.py runs it; four heads
    compared in full."""
    B, H, N = 4, 16, 2048
    x = inputgen.make_fp8_inputs(20262, B, H, N, D)
    prep = _prepare(x, True)
    o, lse = run_fp8(prep, causal)
    for b, h in ((0, 0), (1, 7), (2, 13), (3, 15)):
        sub = {n: prep[n][b:b + 1, h:h + 1] for n in prep}
        _check_against_oracle(sub, causal, o[b:b + 1, h:h + 1], lse[b:b + 1, h:h + 1])


def test_rotation_lowers_error_on_gpu():
    """0.1% outliers of std 10: the GPU's FP8 attention with the rotation is
    closer to the exact bf16 attention than without it."""
    B, H, N = 1, 4, 1024
    x = inputgen.make_fp8_inputs(31, B, H, N, D, outlier_frac=0.001, outlier_std=10.0)
    ro, _ = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), 1 / math.sqrt(D), False)
    errs = {}
    for rotate in (False, True):
        o, _ = run_fp8(_prepare(x, rotate), False)
        errs[rotate] = _rms(o.float().cpu().numpy(), ro)
    assert errs[False] / errs[True] > 1.2, errs
