"""fa_fwd_pair (the forward on CTA pairs, tcgen05 .cta_group::2) on the GPU
against the fp64 oracle.

The same contract as fa_fwd for d = 128: O within 1e-2 and LSE within 1e-3
of the oracle on the stated workloads (the prefill workload for every head,
without and with the causal mask); other shapes cover pair tiles of 256
query rows that end inside the sequence (ragged N, N below 128 where the
second CTA of a pair holds no row, N = 1), many units per pair, and a
repeat run that must be bitwise identical. Outputs carry NaN guard bands
and inputs NaN padding, so any access past either end shows.
"""
import numpy as np
import pytest
import torch

import exact_attention_130_b200 as fa
import inputgen
import oracle
from gpu_helpers import TOL_LSE, TOL_O, Guarded, bf16_device, f64, max_abs

pytestmark = pytest.mark.gpu

SHAPES = [
    (1, 2, 128, 128), (2, 3, 256, 128), (1, 2, 384, 128), (1, 1, 1, 128), (2, 2, 100, 128),
    (1, 2, 1000, 128), (1, 3, 513, 128), (3, 5, 200, 128), (4, 40, 384, 128),
]


def run_pair(x, causal):
    B, H, N, d = x["q"].shape
    q, k, v = (bf16_device(x[n]) for n in ("q", "k", "v"))
    o = Guarded((B, H, N, d), torch.bfloat16)
    lse = Guarded((B, H, N), torch.float32)
    fa.fa_fwd_pair(q, k, v, causal=causal, o=o.t, lse=lse.t)
    torch.cuda.synchronize()
    assert o.guards_intact() and lse.guards_intact()
    return o.t, lse.t


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_fwd_pair_small(shape, causal):
    """Outside the stated workloads the O bound is 1e-2 + 2^-8 |O_ref|
    (bf16 rounding of P and O, unit roundoff 2^-8, where the first causal
    rows average few keys and |O| reaches 2-3)."""
    B, H, N, d = shape
    x = inputgen.make_small_inputs(7000 + N + H + (1000 if causal else 0), B, H, N, d)
    o, lse = run_pair(x, causal)
    ref_o, ref_l = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), 1 / np.sqrt(d), causal)
    err = np.abs(o.float().cpu().numpy() - ref_o)
    assert np.all(err <= TOL_O + 2.0 ** -8 * np.abs(ref_o))
    assert max_abs(lse, ref_l) <= TOL_LSE
    st, word = fa.fa_device_status()
    assert st == 0, hex(word)


@pytest.mark.parametrize("causal", [False, True], ids=["full", "causal"])
def test_fwd_pair_prefill_workload_every_head(causal):
    w = inputgen.WORKLOADS["prefill"]
    x = inputgen.make_attention_inputs(w)
    o, lse = run_pair(x, causal)
    ref_o, ref_l = oracle.attention_fwd(f64(x["q"]), f64(x["k"]), f64(x["v"]), w.scale, causal)
    assert max_abs(o, ref_o) <= TOL_O
    assert max_abs(lse, ref_l) <= TOL_LSE


def test_fwd_pair_deterministic_and_refuses_d64():
    x = inputgen.make_small_inputs(17, 2, 4, 1000, 128)
    a = run_pair(x, True)
    b = run_pair(x, True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    q = torch.zeros((1, 1, 128, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(fa.FAError):
        fa.fa_fwd_pair(q, q, q)
